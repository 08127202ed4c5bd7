// Dispatch permute: token rows into the expert-major pool.
//
// recv[src_pool_row[t, j]] = x[t] for every valid (t, j) (StreamEP README,
// "Streaming dispatch in one paragraph": each landed (token, k) pair lands in
// its pool slot; PR #769 "Description": the activation copy of the dispatch
// epilogue).  Token-major: a warp reads its slice of x[t] once with 16-byte
// loads and stores it to the token's k pool rows, so HBM sees the algorithmic
// minimum (read T*H once, write N_a rows).  Padding rows are never touched.
//
// FP8 (DeepEP low-latency article, "FP8 and Quantization Support"; blog, "FP8
// Dispatch 减少的是 payload"): a lane holds 16 channels, 8 lanes one 128-channel
// group; amax by shuffles, one scale per group, codes from the hardware
// e4m3x2 round-to-nearest-even satfinite conversion; each token is quantised
// once and its codes written k times.
//
// Streaming (StreamEP README, same section): after its rows are stored, a
// warp fences, then lane j atomically adds one arrival to the tile of row j
// (acq_rel, gpu scope); the arrival that reaches the tile's target (valid rows
// x warps per row) release-stores dispatch_seq into tile_ready[tile].
#include <cstdlib>

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fp8_quant.cuh"
#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned *ptr, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_release_gpu(unsigned *ptr, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// Store of one 16-byte piece of a pool row.
constexpr bool kStreamingStores = false;
__device__ __forceinline__ void st_row(uint4 *ptr, uint4 v)
{
    if (kStreamingStores)
        asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x), "r"(v.y), "r"(v.z),
                     "r"(v.w) : "memory");
    else
        *ptr = v;
}

// Publish the rows this warp just finished for token t (one arrival per row).
__device__ __forceinline__ void publish_rows(const DispatchParams &p, int my_row, int lane)
{
    __threadfence();
    __syncwarp();
    if (lane < p.k && my_row >= 0) {
        const int tile = my_row / p.B;
        const unsigned need = (unsigned)p.pool_arrival_target[tile] * (unsigned)p.segs;
        const unsigned old = atom_add_acq_rel_gpu(p.pool_arrival_count + tile, 1u);
        if (old + 1u == need)
            st_release_gpu(p.tile_ready + tile, p.seq);
    }
}

// bf16: a work item is (token, segment of seg_len 16-byte vectors).
template <int UNROLL, bool PUBLISH, int WARPS = kWarps>
__global__ void __launch_bounds__(WARPS * 32) dispatch_bf16_kernel(DispatchParams p)
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
        const uint4 *src = static_cast<const uint4 *>(p.x) + t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += 32 * UNROLL) {
            uint4 buf[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = v0 + u * 32 + lane;
                buf[u] = v < v_end ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
            }
            for (int j = 0; j < p.k; ++j) {
                const int row = __shfl_sync(kFullMask, my_row, j);
                if (row < 0)
                    continue;                            // warp-uniform
                uint4 *dst = static_cast<uint4 *>(p.recv) + (int64_t)row * V;
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < v_end)
                        st_row(dst + v, buf[u]);
                }
            }
        }
        if (PUBLISH)
            publish_rows(p, my_row, lane);
    }
}

// fp8: a work item is (token, segment of seg_len 512-channel iterations).
// The default grid's 8-warp CTAs are held to 40 registers, so 6 of them fit
// an SM (42 registers, allocated as 48, allowed 5): more warps waiting on x
// at once (prefill_skew dispatch 193.6 against 194.0 us, decode step 26.2
// against 26.8 us).
template <int SCALE, bool PUBLISH, int WARPS = kWarps>
__global__ void __launch_bounds__(WARPS * 32, WARPS == kWarps ? 6 : 1) dispatch_fp8_kernel(DispatchParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int H = p.H;
    const int G = H / 128;
    const int iters = (H + 511) / 512;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.segs;
        const int s = (int)(it - t * p.segs);
        const int i_begin = s * p.seg_len;
        const int i_end = min(iters, i_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        const __nv_bfloat16 *xrow = static_cast<const __nv_bfloat16 *>(p.x) + t * H;
        for (int i = i_begin; i < i_end; ++i) {
            const int c0 = i * 512 + lane * 16;          // H % 128 == 0: whole groups are in or out
            const bool active = c0 < H;
            float f[16];
            if (active) {
                const uint4 *src = reinterpret_cast<const uint4 *>(xrow + c0);
                bf16x8_to_f32(ld_stream(src), f);
                bf16x8_to_f32(ld_stream(src + 1), f + 8);
            } else {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    f[q] = 0.f;
            }
            float scale_f;
            int expo;
            const uint4 codes = quantize_lane16<SCALE>(f, scale_f, expo);
            const int g = c0 / 128;
            for (int j = 0; j < p.k; ++j) {
                const int row = __shfl_sync(kFullMask, my_row, j);
                if (row < 0)
                    continue;                            // warp-uniform
                if (active) {
                    uint8_t *dst = static_cast<uint8_t *>(p.recv) + (int64_t)row * H + c0;
                    *reinterpret_cast<uint4 *>(dst) = codes;
                    if ((lane & 7) == 0) {
                        if (SCALE == SEP_SCALE_UE8M0)
                            static_cast<uint8_t *>(p.recv_scales)[(int64_t)row * G + g] = (uint8_t)(expo + 127);
                        else
                            static_cast<float *>(p.recv_scales)[(int64_t)row * G + g] = scale_f;
                    }
                }
            }
        }
        if (PUBLISH)
            publish_rows(p, my_row, lane);
    }
}

// bf16 pool stores handed to the bulk-copy (TMA) unit.  The warp writes its
// 2 KB step of x[t] (128 vectors, one per lane and unroll slot) into one of
// two shared-memory stages, makes it visible to the async proxy
// (fence.proxy.async), and lane 0 issues one cp.async.bulk store of the stage
// per pool row of the token (no multicast; addresses and sizes are 16-byte
// multiples).  A stage is rewritten only after the bulk group that read it
// has finished reading (cp.async.bulk.wait_group.read).  This replaces
// k x 32 lane stores per step by k bulk operations: measured on train8k, 71.8
// against 73.1 us alone and 152.6 against 153.5 us per step, with the
// store-issue stalls (lg_throttle, short scoreboard) gone.  It is the bf16
// default wherever no tile publication follows the stores;
// SEP_DISPATCH_STAGED=0 in the environment (read once per process) selects
// the register stores, for comparison.  (The same staging of the FP8 codes,
// 512 bytes per bulk store, measured slower: prefill_skew dispatch 217.4
// against 205.8 us; the FP8 dispatch stores from registers.)
constexpr int kStageVecs = 128;                  // one 2 KB step
constexpr int kStages = 2;

__global__ void __launch_bounds__(kWarps * 32) dispatch_bf16_staged_kernel(DispatchParams p)
{
    __shared__ __align__(128) uint4 s_stage[kWarps][kStages][kStageVecs];
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    int stage = 0;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.segs;
        const int s = (int)(it - t * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        const uint4 *src = static_cast<const uint4 *>(p.x) + t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += kStageVecs) {
            const int n = min(kStageVecs, v_end - v0);
            uint4 buf[kStageVecs / 32];
#pragma unroll
            for (int u = 0; u < kStageVecs / 32; ++u) {
                const int v = v0 + u * 32 + lane;
                buf[u] = v < v0 + n ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
            }
            if (lane == 0)                                   // the stage's previous bulk reads are done
                asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kStages - 1) : "memory");
            __syncwarp();
            uint4 *st = s_stage[warp][stage];
#pragma unroll
            for (int u = 0; u < kStageVecs / 32; ++u)
                st[u * 32 + lane] = buf[u];
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            const uint32_t saddr = static_cast<uint32_t>(__cvta_generic_to_shared(st));
            for (int j = 0; j < p.k; ++j) {
                const int row = __shfl_sync(kFullMask, my_row, j);
                if (row >= 0 && lane == 0) {
                    uint4 *dst = static_cast<uint4 *>(p.recv) + (int64_t)row * V + v0;
                    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                                 ::"l"(dst), "r"(saddr), "r"(n * 16) : "memory");
                }
            }
            if (lane == 0)
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            stage ^= 1;
        }
    }
    if (lane == 0)
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

bool staged_dispatch_selected()
{
    static const bool on = [] {
        const char *v = std::getenv("SEP_DISPATCH_STAGED");
        return !(v != nullptr && v[0] == '0' && v[1] == '\0');
    }();
    return on;
}

// One warp per work item and no cap at the resident CTA count: CTAs that
// finish early make room for the rest, which balances the tail across SMs.
// A caller's CTA budget (max_ctas) below that grid launches at most max_ctas
// CTAs of kBudgetWarps warps instead (about one per SM: a small grid of
// 8-warp CTAs keeps too few loads in flight per SM); the kernels walk their
// items with a grid stride, so any grid covers them.
int64_t default_blocks(int64_t items)
{
    return (items + kWarps - 1) / kWarps;
}

int budget_blocks(int64_t items, int max_ctas)
{
    const int64_t b = (items + kBudgetWarps - 1) / kBudgetWarps;
    return (int)(b > max_ctas ? max_ctas : b);
}

template <bool PUBLISH, int WARPS>
cudaError_t launch_fp8(const DispatchParams &p, cudaStream_t s, dim3 grid)
{
    const dim3 block(WARPS * 32);
    switch (p.scale) {
    case SEP_SCALE_F32:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_F32, PUBLISH, WARPS>, grid, block, 0, s, p);
    case SEP_SCALE_UE8M0:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_UE8M0, PUBLISH, WARPS>, grid, block, 0, s, p);
    default:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, PUBLISH, WARPS>, grid, block, 0, s, p);
    }
}

}  // namespace

// Row splitting.  A bf16 step is 128 vectors of 16 bytes (one pass of the
// kernel's 4-deep unroll); without tile publication every step is its own work
// item, so the items divide finely over the waves of CTAs (measured faster
// than whole rows per warp).  With tile publication a row stays on one warp
// where possible, since every item pays a fence and one arrival per row.  FP8
// steps are 512 channels, and a row splits over up to 14 warps (prefill_skew,
// H = 7168: one step per warp, so no warp waits on a second load of x after
// its first step's stores; dispatch 194.0 against 206.3 us with up to 7).
constexpr int64_t kStepVecs = 128;
constexpr int64_t kMinSegs = 1 << 20;
constexpr int64_t kPublishMinSegs = 1;
constexpr int64_t kFp8MinSegs = 14;

cudaError_t launch_dispatch(DispatchParams p, int payload, cudaStream_t s, int num_sms)
{
    if (p.T == 0)
        return cudaSuccess;
    const bool fp8 = payload != SEP_PAYLOAD_BF16;
    const int64_t units = fp8 ? (p.H + 511) / 512 : ((p.H / 8) + kStepVecs - 1) / kStepVecs;
    int64_t steps = 1;
    split_rows(p.T, units, (int64_t)num_sms * 32, fp8 ? kFp8MinSegs : (p.tile_ready ? kPublishMinSegs : kMinSegs),
               &p.segs, &steps);
    p.seg_len = (int)(fp8 ? steps : steps * kStepVecs);
    const int64_t items = p.T * p.segs;
    if (p.max_ctas > 0 && p.max_ctas < default_blocks(items)) {
        const dim3 grid(budget_blocks(items, p.max_ctas)), block(kBudgetWarps * 32);
        if (payload == SEP_PAYLOAD_BF16)
            return p.tile_ready != nullptr
                       ? launch_kernel(dispatch_bf16_kernel<4, true, kBudgetWarps>, grid, block, 0, s, p)
                       : launch_kernel(dispatch_bf16_kernel<4, false, kBudgetWarps>, grid, block, 0, s, p);
        return p.tile_ready != nullptr ? launch_fp8<true, kBudgetWarps>(p, s, grid)
                                       : launch_fp8<false, kBudgetWarps>(p, s, grid);
    }
    const dim3 grid((int)default_blocks(items)), block(kWarps * 32);
    if (payload == SEP_PAYLOAD_BF16) {
        if (p.tile_ready == nullptr && p.seg_len % kStageVecs == 0 && staged_dispatch_selected())
            return launch_kernel(dispatch_bf16_staged_kernel, grid, block, 0, s, p);
        if (p.tile_ready != nullptr)
            return launch_kernel(dispatch_bf16_kernel<4, true>, grid, block, 0, s, p);
        return launch_kernel(dispatch_bf16_kernel<4, false>, grid, block, 0, s, p);
    }
    return p.tile_ready != nullptr ? launch_fp8<true, kWarps>(p, s, grid) : launch_fp8<false, kWarps>(p, s, grid);
}

cudaError_t preload_dispatch_kernels()
{
    const void *k[] = {
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, false>),
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, true>),
        reinterpret_cast<const void *>(dispatch_bf16_staged_kernel),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, true>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, true>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, true>),
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, false, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, true, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, false, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, true, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, false, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, true, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, false, kBudgetWarps>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, true, kBudgetWarps>)};
    cudaFuncAttributes a;
    for (const void *f : k) {
        const cudaError_t e = cudaFuncGetAttributes(&a, f);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace sep
