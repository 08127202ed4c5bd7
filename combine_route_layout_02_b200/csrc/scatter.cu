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

}  // namespace

cudaError_t launch_combine_scatter(ScatterParams p, cudaStream_t s, int num_sms)
{
    if (p.rows_cap == 0)
        return cudaSuccess;
    // a pool row splits into steps of 32 * kUnroll vectors, one work item each
    int64_t steps = 1;
    split_rows(p.rows_cap, ((p.H / 8) + 32 * kUnroll - 1) / (32 * kUnroll), (int64_t)num_sms * 32, 1 << 20, &p.segs,
               &steps);
    p.seg_len = (int)(steps * 32 * kUnroll);
    const int64_t items = p.rows_cap * p.segs;
    if (items == 0)
        return cudaSuccess;
    const int64_t want = (items + kWarps - 1) / kWarps;
    return launch_kernel(combine_scatter_kernel, dim3((int)want), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_scatter_kernels()
{
    cudaFuncAttributes a;
    return cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_scatter_kernel));
}

}  // namespace sep
