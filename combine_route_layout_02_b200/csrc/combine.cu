// Combine: weighted top-k reduction from the pool back to token order.
//
// out[t] = bf16( sum_j w[t, j] * y[src_pool_row[t, j]] )  ("DeepEP MoE
// dispatch/combine" blog, "Router 权重什么时候应用": y_t = sum_j p_{t,j} o_{t,j};
// "一轮 DeepEP 数据流": combine restores the source token / top-k slot and
// reduces the routing-weighted expert outputs).
//
// A warp owns (token, segment).  Lane j < k holds the token's row index and
// weight; each lane then loads 16 bytes from up to 8 rows at once (8 loads in
// flight per lane), and accumulates in fp32 in ascending j with a rounded
// multiply followed by a rounded add (no fused multiply-add), starting at +0.
// That is exactly the fp32 arithmetic of the definition, so the result is
// bit-identical to it; the final bf16 rounding is to nearest even.
#include <cuda_bf16.h>

#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kRowBatch = 8;         // rows loaded before they are summed

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

__device__ __forceinline__ void accumulate(float *acc, const uint4 &v, float w)
{
    const uint32_t word[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(w, __uint_as_float(word[i] << 16)));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(w, __uint_as_float(word[i] & 0xffff0000u)));
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

__global__ void __launch_bounds__(kWarps * 32) combine_kernel(CombineParams p)
{
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const uint4 *y = static_cast<const uint4 *>(p.y);
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.segs;
        const int s = (int)(it - t * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        const float my_w = lane < p.k ? __ldg(p.w + t * p.k + lane) : 0.f;
        uint4 *out = static_cast<uint4 *>(p.out) + t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += 32) {
            const int v = v0 + lane;
            const bool act = v < v_end;
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                acc[q] = 0.f;
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
                out[v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineParams &p, cudaStream_t s, int num_sms)
{
    const int64_t items = p.T * p.segs;
    if (items == 0)
        return cudaSuccess;
    const int per_sm = occupancy_blocks_per_sm(reinterpret_cast<const void *>(combine_kernel), kWarps * 32, 0);
    const int64_t want = (items + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)num_sms * per_sm;
    combine_kernel<<<(int)(want < cap ? want : cap), kWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t preload_combine_kernels()
{
    cudaFuncAttributes a;
    return cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(combine_kernel));
}

}  // namespace sep
