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
// skipped.  With no weights (w == nullptr) every weight is 1: that is the
// backward of dispatch, combine_grads (StreamEP README, "What's in the box"),
// and 1 * y is exact, so it too is bit-identical to its definition.
//
// A warp owns (token, segment); the token's k row indices and weights are
// broadcast once into every lane's registers, then each lane walks its
// 16-byte columns issuing kRowBatch row loads at a time.  Tokens are taken in
// descending order, which reads first the pool rows a preceding dispatch wrote
// last (still resident in L2).
//
// Gated combine (StreamEP README, opening section: the per-recv-token gate
// y_done_per_token lets combine start on a token as soon as that token's
// compute has drained).  The grid is persistent and bounded by the caller so
// that the producer keeps SMs; tokens are taken in ascending order, the order
// in which a tile-ordered producer finishes them.  Lane 0 waits (acquire load,
// bounded by %globaltimer and a poll budget) for y_done[t] >= done_seq, the
// warp barrier passes the acquired view to the other lanes, and the rows are
// read through L2 (they are written by a kernel that is still running, so the
// non-coherent path is not used).  A token without valid assignments is not
// waited for (its output is +0).  A wait that gives up sets status[0] =
// SEP_ERR_TIMEOUT; every warp then stops waiting and counts the tokens it did
// not reduce in status[1].
#include <cuda_bf16.h>

#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kRowBatch = 4;         // rows loaded before they are summed
constexpr int kKMax = 8;             // row indices / weights held in registers

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

template <bool GATED>
__device__ __forceinline__ uint4 ld_row(const uint4 *ptr)
{
    return GATED ? __ldcg(ptr) : ld_stream(ptr);
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *ptr)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_time_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 1 once y_done[t] has reached done_seq; 0 if this or another warp gave up.
__device__ int wait_token(const CombineParams &p, int64_t t)
{
    const uint64_t t0 = global_time_ns();
    for (uint32_t polls = 0;; ++polls) {
        if ((int32_t)(ld_acquire_gpu(p.y_done + t) - p.done_seq) >= 0)
            return 1;
        if (*reinterpret_cast<volatile const uint32_t *>(p.status) != 0u)
            return 0;
        if (polls >= p.max_polls || global_time_ns() - t0 > p.timeout_ns) {
            atomicCAS(p.status, 0u, (uint32_t)SEP_ERR_TIMEOUT);
            return 0;
        }
        __nanosleep(128);
    }
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

template <bool GATED, int WARPS = kWarps>
__global__ void __launch_bounds__(WARPS * 32) combine_kernel(CombineParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        // ungated, tokens are visited in descending order: a dispatch that ran just
        // before wrote the highest tokens' rows last, so those are still in L2
        const int64_t t = GATED ? it / p.segs : p.T - 1 - it / p.segs;
        const int s = (int)(GATED ? it - t * p.segs : it - (p.T - 1 - t) * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        if (GATED && __any_sync(kFullMask, my_row >= 0)) {   // a token with no rows has nothing to wait for
            int go = 0;
            if (lane == 0) {
                go = wait_token(p, t);
                if (!go)
                    atomicAdd(p.status + 1, 1u);
            }
            go = __shfl_sync(kFullMask, go, 0);
            __syncwarp();
            if (!go)
                continue;
        }
        const float my_w = lane < p.k ? (p.w ? __ldg(p.w + t * p.k + lane) : 1.f) : 0.f;
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
                        buf[u] = rows[j0 + u] >= 0 ? ld_row<GATED>(y + (int64_t)rows[j0 + u] * V + v)
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
                        buf[u] = (rows[u] >= 0 && act) ? ld_row<GATED>(y + (int64_t)rows[u] * V + v)
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

}  // namespace

cudaError_t launch_combine(CombineParams p, cudaStream_t s, int num_sms, int num_ctas)
{
    if (p.T == 0)
        return cudaSuccess;
    if (p.y_done) {
        p.segs = 1;                                      // a token is either reduced or left unwritten
        p.seg_len = p.H / 8;
    } else {
        // steps of 32 vectors (one per lane); rows split only when tokens are too few to fill the GPU
        int64_t steps = 1;
        split_rows(p.T, ((p.H / 8) + 31) / 32, (int64_t)num_sms * 32, 1, &p.segs, &steps);
        p.seg_len = (int)(steps * 32);
    }
    const int64_t items = p.T * p.segs;
    const int64_t want = (items + kWarps - 1) / kWarps;
    if (p.y_done) {
        // persistent: at most num_ctas CTAs, so that the producer keeps its SMs
        const int64_t n = want < num_ctas ? want : num_ctas;
        return launch_kernel(combine_kernel<true>, dim3((int)n), dim3(kWarps * 32), 0, s, p);
    }
    if (p.max_ctas > 0 && want > p.max_ctas) {
        // a CTA budget below the default grid: at most max_ctas CTAs of kBudgetWarps warps (about one per
        // SM; a small grid of 8-warp CTAs keeps too few row loads in flight per SM)
        const int64_t b = (items + kBudgetWarps - 1) / kBudgetWarps;
        return launch_kernel(combine_kernel<false, kBudgetWarps>, dim3((int)(b < p.max_ctas ? b : p.max_ctas)),
                             dim3(kBudgetWarps * 32), 0, s, p);
    }
    return launch_kernel(combine_kernel<false>, dim3((int)want), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_combine_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_kernel<false>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_kernel<true>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_kernel<false, kBudgetWarps>));
    return e;
}

}  // namespace sep
