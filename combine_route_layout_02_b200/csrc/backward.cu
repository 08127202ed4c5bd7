// Backward of combine: dispatch_grads (StreamEP README, "What's in the box":
// Buffer.dispatch_grads / combine_grads give the backward symmetry of the
// forward pair).
//
// The forward combine is out[t] = sum_j w[t, j] * y[row(t, j)] ("DeepEP MoE
// dispatch/combine" blog, "Router 权重什么时候应用").  Its gradients are
//   grad_y[row(t, j)] = bf16( w[t, j] * grad_out[t] )
//   grad_w[t, j]      = sum_h grad_out[t, h] * y[row(t, j), h]
// so dispatch_grads is a dispatch of grad_out that scales each copy by its
// routing weight, plus one dot product per assignment.  Masked assignments get
// no row and grad_w = 0; padding rows of grad_y are never touched.  The
// backward of dispatch (combine_grads) is the combine kernel with unit weights.
//
// Arithmetic: the product w * g is rounded once to fp32 (a plain multiply),
// then to bf16 to nearest even, exactly as the definition reads, so grad_y is
// bit-exact.  The product of two bf16 values is exact in fp32, so grad_w's
// only rounding is in the fp32 sums: a lane adds its columns in ascending
// order, then the warp adds the 32 lane sums by a fixed xor tree.  The order
// depends on H alone, never on scheduling.
//
// Work items.  Without grad_w a warp owns (token, segment) as the forward
// dispatch does: it reads its slice of grad_out[t] once and writes the k scaled
// rows.  With grad_w a warp owns one assignment (t, j) and the whole row; the k
// warps of a token run side by side in one CTA, so grad_out[t] comes from HBM
// once and from L1/L2 for the other k - 1.
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

__device__ __forceinline__ float lo_f32(uint32_t word) { return __uint_as_float(word << 16); }
__device__ __forceinline__ float hi_f32(uint32_t word) { return __uint_as_float(word & 0xffff0000u); }

// bf16(w * g) for the two bf16 values packed in one word
__device__ __forceinline__ uint32_t scale_word(uint32_t word, float w)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(__fmul_rn(w, lo_f32(word)), __fmul_rn(w, hi_f32(word)));
    return static_cast<uint32_t>(__bfloat16_as_ushort(r.x)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(r.y)) << 16);
}

__device__ __forceinline__ uint4 scale_vec(uint4 v, float w)
{
    return make_uint4(scale_word(v.x, w), scale_word(v.y, w), scale_word(v.z, w), scale_word(v.w, w));
}

// acc += sum of the eight products of g and y (ascending channel order)
__device__ __forceinline__ float dot_vec(float acc, uint4 g, uint4 y)
{
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
    const uint32_t yw[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc = __fadd_rn(acc, __fmul_rn(lo_f32(gw[i]), lo_f32(yw[i])));
        acc = __fadd_rn(acc, __fmul_rn(hi_f32(gw[i]), hi_f32(yw[i])));
    }
    return acc;
}

// grad_y only: a work item is (token, segment of seg_len 16-byte vectors).
__global__ void __launch_bounds__(kWarps * 32) dispatch_grads_kernel(DispatchGradsParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.segs;
        const int s = (int)(it - t * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        const float my_w = lane < p.k ? __ldg(p.w + t * p.k + lane) : 0.f;
        const uint4 *src = static_cast<const uint4 *>(p.g) + t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += 32 * kUnroll) {
            uint4 buf[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                buf[u] = v < v_end ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
            }
            for (int j = 0; j < p.k; ++j) {
                const int row = __shfl_sync(kFullMask, my_row, j);
                const float w = __shfl_sync(kFullMask, my_w, j);
                if (row < 0)
                    continue;                            // warp-uniform
                uint4 *dst = static_cast<uint4 *>(p.grad_y) + (int64_t)row * V;
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < v_end)
                        dst[v] = scale_vec(buf[u], w);
                }
            }
        }
    }
}

// grad_y and grad_w: a work item is one assignment (t, j), the whole row.
__global__ void __launch_bounds__(kWarps * 32) dispatch_grads_dot_kernel(DispatchGradsParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.k;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.k;
        const int row = __ldg(p.src_pool_row + it);
        float acc = 0.f;
        if (row >= 0) {
            const float w = __ldg(p.w + it);
            const uint4 *g = static_cast<const uint4 *>(p.g) + t * V;
            const uint4 *y = static_cast<const uint4 *>(p.y) + (int64_t)row * V;
            uint4 *dst = static_cast<uint4 *>(p.grad_y) + (int64_t)row * V;
            for (int v0 = 0; v0 < V; v0 += 32 * kUnroll) {
                uint4 gb[kUnroll], yb[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * 32 + lane;
                    gb[u] = v < V ? __ldg(g + v) : make_uint4(0, 0, 0, 0);
                    yb[u] = v < V ? ld_stream(y + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < V) {
                        dst[v] = scale_vec(gb[u], w);
                        acc = dot_vec(acc, gb[u], yb[u]);
                    }
                }
            }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1)
            acc = __fadd_rn(acc, __shfl_xor_sync(kFullMask, acc, m));
        if (lane == 0)
            p.grad_w[it] = acc;                          // 0 for a masked assignment
    }
}

// one warp per work item, as the forward dispatch launches
int blocks_for(int64_t warp_items)
{
    const int64_t want = (warp_items + kWarps - 1) / kWarps;
    return (int)(want < 1 ? 1 : want);
}

}  // namespace

cudaError_t launch_dispatch_grads(DispatchGradsParams p, cudaStream_t s, int num_sms)
{
    if (p.T == 0)
        return cudaSuccess;
    // without grad_w, rows split into the forward dispatch's 128-vector steps, one item each
    int64_t steps = 1;
    split_rows(p.T, ((p.H / 8) + 127) / 128, (int64_t)num_sms * 32, 1 << 20, &p.segs, &steps);
    p.seg_len = (int)(steps * 128);
    if (p.grad_w)
        return launch_kernel(dispatch_grads_dot_kernel, dim3(blocks_for(p.T * p.k)), dim3(kWarps * 32), 0, s, p);
    return launch_kernel(dispatch_grads_kernel, dim3(blocks_for(p.T * p.segs)), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_backward_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(dispatch_grads_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(dispatch_grads_dot_kernel));
    return e;
}

}  // namespace sep
