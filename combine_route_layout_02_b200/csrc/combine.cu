// Combine: weighted top-k reduction from the pool back to token order.
//
// out[t] = bf16( sum_j w[t, j] * y[src_pool_row[t, j]] )  ("DeepEP MoE
// dispatch/combine" blog, "Router 权重什么时候应用": y_t = sum_j p_{t,j} o_{t,j};
// "一轮 DeepEP 数据流": combine restores the source token / top-k slot and
// reduces the routing-weighted expert outputs).
//
// Accumulation is fp32 in ascending j, a rounded multiply followed by a
// rounded add (no fused multiply-add), starting at +0: exactly the fp32
// arithmetic of the definition, so the result is bit-identical to it; the
// final bf16 rounding is to nearest even.  Masked assignments (row < 0) are
// skipped.
//
// Two implementations:
//  * register path: a warp owns (token, segment); the token's k row indices
//    and weights are broadcast once into every lane's registers, then each lane
//    walks its 16-byte columns issuing kRowBatch row loads at a time.  Tokens
//    are taken in descending order, which reads first the pool rows a preceding
//    dispatch wrote last (still resident in L2);
//  * bulk path (used when k <= 32 and two stages of k rows fit in shared
//    memory): warp 0 of a CTA bulk-loads the token's k rows into a two-stage
//    shared-memory ring with cp.async.bulk (completion on an mbarrier), every
//    thread waits on the barrier (bounded), reduces its columns from shared
//    memory and stores the bf16 result; the stage is refilled with the CTA's
//    next-but-one token after a CTA barrier.
#include <cuda_bf16.h>

#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kRowBatch = 4;         // rows loaded before they are summed (register path)
constexpr int kKMax = 8;             // row indices / weights held in registers
constexpr bool kBulkCombine = false;
constexpr int kBulkStages = 2;
constexpr int kBulkThreads = 256;
constexpr int kBulkMaxSmem = 200 * 1024;

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

__device__ __forceinline__ void accumulate_word(float &lo, float &hi, uint32_t word, float w)
{
    lo = __fadd_rn(lo, __fmul_rn(w, __uint_as_float(word << 16)));
    hi = __fadd_rn(hi, __fmul_rn(w, __uint_as_float(word & 0xffff0000u)));
}

__device__ __forceinline__ void accumulate(float *acc, uint4 v, float w)
{
    accumulate_word(acc[0], acc[1], v.x, w);
    accumulate_word(acc[2], acc[3], v.y, w);
    accumulate_word(acc[4], acc[5], v.z, w);
    accumulate_word(acc[6], acc[7], v.w, w);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

__device__ __forceinline__ uint4 pack_out(const float *acc)
{
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// ------------------------------------------------------------ register path

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(CombineParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        // tokens are visited in descending order: a dispatch that ran just before
        // wrote the highest tokens' rows last, so those are the rows still in L2
        const int64_t t = p.T - 1 - it / p.segs;
        const int s = (int)(it - (p.T - 1 - t) * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        const float my_w = lane < p.k ? __ldg(p.w + t * p.k + lane) : 0.f;
        uint4 *out = static_cast<uint4 *>(p.out) + t * V;
        if (p.k <= kKMax) {
            int rows[kKMax];
            float ws[kKMax];
#pragma unroll
            for (int j = 0; j < kKMax; ++j) {
                rows[j] = __shfl_sync(kFullMask, my_row, j);
                ws[j] = __shfl_sync(kFullMask, my_w, j);
            }
            for (int v = v_begin + lane; v < v_end; v += 32) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j0 = 0; j0 < kKMax; j0 += kRowBatch) {
                    uint4 buf[kRowBatch];
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u)
                        buf[u] = rows[j0 + u] >= 0 ? ld_stream(y + (int64_t)rows[j0 + u] * V + v)
                                                   : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u)
                        if (rows[j0 + u] >= 0)
                            accumulate(acc, buf[u], ws[j0 + u]);
                }
                out[v] = pack_out(acc);
            }
        } else {
            for (int v0 = v_begin; v0 < v_end; v0 += 32) {
                const int v = v0 + lane;
                const bool act = v < v_end;
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int j0 = 0; j0 < p.k; j0 += kRowBatch) {
                    uint4 buf[kRowBatch];
                    int rows[kRowBatch];
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u) {
                        const int j = j0 + u;
                        const int row = __shfl_sync(kFullMask, my_row, j & 31);
                        rows[u] = j < p.k ? row : -1;
                        buf[u] = (rows[u] >= 0 && act) ? ld_stream(y + (int64_t)rows[u] * V + v)
                                                       : make_uint4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u) {
                        const float w = __shfl_sync(kFullMask, my_w, (j0 + u) & 31);
                        if (rows[u] >= 0)
                            accumulate(acc, buf[u], w);
                    }
                }
                if (act)
                    out[v] = pack_out(acc);
            }
        }
    }
}

// ---------------------------------------------------------------- bulk path

__device__ __forceinline__ uint32_t smem_u32(const void *ptr)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns)
{
    const uint64_t t0 = now_ns();
    for (uint32_t it = 0; it < (1u << 24); ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (now_ns() - t0 > limit_ns)
            return false;
    }
    return false;
}

// Warp 0: fetch token t's rows and weights into the stage's tables and start
// the bulk loads of its valid rows (one expect_tx for their total size).
__device__ __forceinline__ void issue_token(const CombineParams &p, int64_t t, uint32_t stage_smem,
                                            uint32_t bar, int *s_rows, float *s_w, uint32_t row_bytes)
{
    const int lane = threadIdx.x & 31;
    const int row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
    if (lane < p.k) {
        s_rows[lane] = row;
        s_w[lane] = __ldg(p.w + t * p.k + lane);
    }
    const unsigned valid = __ballot_sync(kFullMask, row >= 0);
    if (lane == 0)
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                     ::"r"(bar), "r"((uint32_t)__popc(valid) * row_bytes) : "memory");
    for (int j = 0; j < p.k; ++j) {
        const int r = __shfl_sync(kFullMask, row, j);
        if (lane == 0 && r >= 0)
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                         ::"r"(stage_smem + (uint32_t)j * row_bytes),
                           "l"(static_cast<const uint8_t *>(p.y) + (int64_t)r * row_bytes), "r"(row_bytes),
                           "r"(bar) : "memory");
    }
}

__global__ void __launch_bounds__(kBulkThreads) combine_bulk_kernel(CombineParams p)
{
    extern __shared__ __align__(128) uint8_t stage_mem[];   // [stages][k][row bytes]
    __shared__ __align__(8) uint64_t bars[kBulkStages];
    __shared__ int s_rows[kBulkStages][32];
    __shared__ float s_w[kBulkStages][32];
    grid_dependency_wait();
    allow_dependents();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int V = p.H / 8;
    const uint32_t row_bytes = (uint32_t)p.H * 2u;
    const uint32_t stage_bytes = (uint32_t)p.k * row_bytes;
    const uint32_t base = smem_u32(stage_mem);
    const int64_t n = p.T > blockIdx.x ? (p.T - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    auto token = [&](int64_t i) { return (int64_t)blockIdx.x + i * gridDim.x; };

    if (warp == 0) {
        if (tid == 0) {
            for (int s = 0; s < kBulkStages; ++s)
                asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[s])));
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        for (int64_t i = 0; i < n && i < kBulkStages; ++i)
            issue_token(p, token(i), base + (uint32_t)i * stage_bytes, smem_u32(&bars[i]), s_rows[i], s_w[i],
                        row_bytes);
    }
    __syncthreads();
    int64_t issued = n < kBulkStages ? n : kBulkStages;
    const uint4 *stage16 = reinterpret_cast<const uint4 *>(stage_mem);
    for (int64_t i = 0; i < n; ++i) {
        const int s = (int)(i % kBulkStages);
        const bool ok = mbar_wait_bounded(smem_u32(&bars[s]), (uint32_t)((i / kBulkStages) & 1), 100000000ull);
        if (!__syncthreads_and(ok)) {
            if (tid == 0) {
                atomicMax(p.error_epoch, p.epoch);
                for (int64_t q = i; q < issued; ++q)        // let issued loads land before exiting
                    mbar_wait_bounded(smem_u32(&bars[q % kBulkStages]), (uint32_t)((q / kBulkStages) & 1),
                                      100000000ull);
            }
            return;
        }
        const int64_t t = token(i);
        const uint4 *st = stage16 + (size_t)s * (stage_bytes / 16);
        uint4 *out = static_cast<uint4 *>(p.out) + t * V;
        for (int v = tid; v < V; v += kBulkThreads) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < p.k; ++j)
                if (s_rows[s][j] >= 0)
                    accumulate(acc, st[(size_t)j * V + v], s_w[s][j]);
            out[v] = pack_out(acc);
        }
        __syncthreads();                                 // the stage and its tables are free again
        if (warp == 0 && issued < n) {
            issue_token(p, token(issued), base + (uint32_t)s * stage_bytes, smem_u32(&bars[s]), s_rows[s],
                        s_w[s], row_bytes);
        }
        if (issued < n)
            ++issued;
    }
}

}  // namespace

cudaError_t launch_combine(const CombineParams &p, cudaStream_t s, int num_sms)
{
    const int64_t items = p.T * p.segs;
    if (items == 0)
        return cudaSuccess;
    const int64_t smem = (int64_t)kBulkStages * p.k * p.H * 2;
    if (kBulkCombine && p.k <= 32 && smem <= kBulkMaxSmem) {
        static int attr_set = 0;
        if (!attr_set) {
            cudaError_t e = cudaFuncSetAttribute(combine_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kBulkMaxSmem);
            if (e != cudaSuccess)
                return e;
            attr_set = 1;
        }
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_bulk_kernel, kBulkThreads,
                                                          (size_t)smem) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const int64_t cap = (int64_t)num_sms * per_sm;
        return launch_kernel(combine_bulk_kernel, dim3((int)(p.T < cap ? p.T : cap)), dim3(kBulkThreads),
                             (size_t)smem, s, p);
    }
    const int64_t want = (items + kWarps - 1) / kWarps;
    return launch_kernel(combine_kernel, dim3((int)want), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_combine_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_bulk_kernel));
    return e;
}

}  // namespace sep
