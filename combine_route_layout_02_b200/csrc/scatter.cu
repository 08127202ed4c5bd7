// Atomic-scatter combine: the weighted top-k reduction driven from the pool
// side (StreamEP README, "What's in the box": kernel_y's AtomicScatterStore
// does per-warp coalesced bf16 atomic scatter into the output; ptx_helpers'
// red_add_bf16x2).
//
// out[t] += bf16( w[t, j] * y[r] ) for every valid pool row r, with
// t = pool_recv_token[r] and j = pool_recv_slot[r], into an out that starts at
// zero.  A warp owns (pool row, segment of the row): it reads its slice of
// y[r] once, coalesced, scales it in fp32, rounds each product to bf16 and adds
// it to out[t] with 16-byte bf16x2 reductions performed at L2
// (red.global.add.noftz.v4.bf16x2).  Rows are walked in pool order, so the
// reads are sequential and the k reductions a token receives come from k
// different warps in no fixed order: the result is not deterministic, and its
// rounding is bf16 at every partial sum (a token's k terms each rounded once,
// then k - 1 bf16 additions in arrival order) instead of the gather combine's
// single fp32 sum.  Padding rows and rows past the pool size P (read from the
// handle's device size word, so an unsynced layout needs no host round trip)
// are skipped.
#include <cuda_bf16.h>

#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

__device__ __forceinline__ uint32_t scale_word(uint32_t word, float w)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(w, __uint_as_float(word << 16)),
                                                   __fmul_rn(w, __uint_as_float(word & 0xffff0000u)));
    return static_cast<uint32_t>(__bfloat16_as_ushort(r.x)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(r.y)) << 16);
}

// eight bf16 additions at L2, one 16-byte request
__device__ __forceinline__ void red_add_bf16x8(uint4 *dst, uint4 v)
{
    asm volatile("red.relaxed.gpu.global.add.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};"
                 ::"l"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__global__ void __launch_bounds__(kWarps * 32) combine_scatter_kernel(ScatterParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t P = *p.num_pool_rows;              // rows past P may hold a previous layout's maps
    const int64_t items = (P < p.rows_cap ? P : p.rows_cap) * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t r = it / p.segs;
        const int s = (int)(it - r * p.segs);
        const int t = __ldg(p.pool_recv_token + r);
        if (t < 0)
            continue;                                    // padding row, warp-uniform
        const int j = __ldg(p.pool_recv_slot + r);
        const float w = __ldg(p.w + (int64_t)t * p.k + j);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const uint4 *src = static_cast<const uint4 *>(p.y) + r * V;
        uint4 *dst = static_cast<uint4 *>(p.out) + (int64_t)t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += 32 * kUnroll) {
            uint4 buf[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                buf[u] = v < v_end ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < v_end)
                    red_add_bf16x8(dst + v, make_uint4(scale_word(buf[u].x, w), scale_word(buf[u].y, w),
                                                       scale_word(buf[u].z, w), scale_word(buf[u].w, w)));
            }
        }
    }
}

// Bulk variant: the warp stages its scaled bf16 slice in shared memory and lane
// 0 hands it to the TMA unit as one bulk reduction
// (cp.reduce.async.bulk .add.noftz.bf16, shared -> global, no multicast).  Two
// staging buffers per warp; a buffer is rewritten only after the bulk
// operation that read it has finished reading (wait_group.read).
constexpr bool kBulkScatter = false;
constexpr int kStageBytes = 2048;                        // one 128-vector step

__device__ __forceinline__ uint32_t smem_u32(const void *ptr)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__global__ void __launch_bounds__(kWarps * 32) combine_scatter_bulk_kernel(ScatterParams p)
{
    __shared__ __align__(128) uint8_t stage[kWarps][2][kStageBytes];
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int V = p.H / 8;
    const int64_t P = *p.num_pool_rows;
    const int64_t items = (P < p.rows_cap ? P : p.rows_cap) * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int b = 0;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t r = it / p.segs;
        const int s = (int)(it - r * p.segs);
        const int t = __ldg(p.pool_recv_token + r);
        if (t < 0)
            continue;
        const int j = __ldg(p.pool_recv_slot + r);
        const float w = __ldg(p.w + (int64_t)t * p.k + j);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);  // seg_len <= 128 vectors: one stage
        const uint4 *src = static_cast<const uint4 *>(p.y) + r * V;
        uint4 buf[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int v = v_begin + u * 32 + lane;
            buf[u] = v < v_end ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
        }
        // the bulk reduction issued two items ago read this buffer: wait until it has
        if (lane == 0)
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
        uint4 *st = reinterpret_cast<uint4 *>(stage[warp][b]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int v = v_begin + u * 32 + lane;
            if (v < v_end)
                st[u * 32 + lane] = make_uint4(scale_word(buf[u].x, w), scale_word(buf[u].y, w),
                                               scale_word(buf[u].z, w), scale_word(buf[u].w, w));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            uint8_t *dst = static_cast<uint8_t *>(p.out) + ((int64_t)t * V + v_begin) * 16;
            asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.noftz.bf16 [%0], [%1], %2;"
                         ::"l"(dst), "r"(smem_u32(st)), "r"((uint32_t)(v_end - v_begin) * 16u) : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        b ^= 1;
    }
    if (lane == 0)
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
}

}  // namespace

cudaError_t launch_combine_scatter(const ScatterParams &p, cudaStream_t s)
{
    const int64_t items = p.rows_cap * p.segs;
    if (items == 0)
        return cudaSuccess;
    const int64_t want = (items + kWarps - 1) / kWarps;
    if (kBulkScatter && p.seg_len <= kStageBytes / 16)
        return launch_kernel(combine_scatter_bulk_kernel, dim3((int)want), dim3(kWarps * 32), 0, s, p);
    return launch_kernel(combine_scatter_kernel, dim3((int)want), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_scatter_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_scatter_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_scatter_bulk_kernel));
    return e;
}

}  // namespace sep
