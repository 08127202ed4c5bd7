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
#include <cuda_bf16.h>
#include <cuda_fp8.h>

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
template <int UNROLL, bool PUBLISH>
__global__ void __launch_bounds__(kWarps * 32) dispatch_bf16_kernel(DispatchParams p)
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

// ---------------------------------------------------------------- bulk copy
//
// bf16 dispatch through the TMA unit (non-streaming only): a CTA is one warp
// whose lane 0 bulk-loads x[t] into one stage of a shared-memory ring
// (cp.async.bulk global->shared, completion on an mbarrier), then issues k
// bulk stores from that stage to the token's pool rows (cp.async.bulk
// shared->global, one bulk group per token).  A stage is refilled once the
// stores of the token before have finished reading it.  Every wait is bounded;
// a wait that gives up records the layout epoch in the handle's timeout word
// (reported by sep_handle_sync), drains the copies it issued and returns.
constexpr bool kBulkDispatch = false;
constexpr int kBulkStages = 4;
constexpr int kBulkMaxSmem = 96 * 1024;

__device__ __forceinline__ uint32_t smem_u32(const void *ptr)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
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

__device__ __forceinline__ uint64_t now_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// true once the barrier's phase `parity` completed; false after ~limit_ns
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

__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst_smem), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, uint32_t src_smem, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(dst), "r"(src_smem), "r"(bytes) : "memory");
}

__global__ void __launch_bounds__(32) dispatch_bf16_bulk_kernel(DispatchParams p)
{
    extern __shared__ __align__(128) uint8_t stage_mem[];
    __shared__ __align__(8) uint64_t bars[kBulkStages];
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x;
    const bool leader = lane == 0;                       // lane 0 drives the copies
    const uint32_t row_bytes = (uint32_t)p.H * 2u;
    const int64_t n = p.T > blockIdx.x ? (p.T - 1 - blockIdx.x) / gridDim.x + 1 : 0;   // this CTA's tokens
    const uint8_t *x = static_cast<const uint8_t *>(p.x);
    uint8_t *recv = static_cast<uint8_t *>(p.recv);
    const uint32_t base = smem_u32(stage_mem);
    auto token = [&](int64_t i) { return (int64_t)blockIdx.x + i * gridDim.x; };

    int64_t loaded = n < kBulkStages ? n : kBulkStages;  // loads issued so far
    if (leader) {
        for (int s = 0; s < kBulkStages; ++s)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[s])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        for (int64_t i = 0; i < loaded; ++i)
            bulk_load(base + (uint32_t)i * row_bytes, x + token(i) * row_bytes, row_bytes, smem_u32(&bars[i]));
    }
    int64_t waited = 0;                                  // loads whose completion was observed
    bool ok = true;
    for (int64_t i = 0; i < n; ++i) {
        const int s = (int)(i % kBulkStages);
        const int64_t t = token(i);
        const int my_row = lane < p.k ? __ldg(p.src_pool_row + t * p.k + lane) : -1;
        int got = 1;
        if (leader)
            got = mbar_wait_bounded(smem_u32(&bars[s]), (uint32_t)((i / kBulkStages) & 1), 100000000ull);
        if (!__shfl_sync(kFullMask, got, 0)) {
            ok = false;
            break;
        }
        waited = i + 1;
        for (int j = 0; j < p.k; ++j) {
            const int row = __shfl_sync(kFullMask, my_row, j);
            if (leader && row >= 0)
                bulk_store(recv + (int64_t)row * row_bytes, base + (uint32_t)s * row_bytes, row_bytes);
        }
        if (leader) {
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // refill the previous stage once the stores of token i-1 have read it
            if (i >= 1 && loaded < n) {
                asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                const int ps = (int)((i - 1) % kBulkStages);
                bulk_load(base + (uint32_t)ps * row_bytes, x + token(loaded) * row_bytes, row_bytes,
                          smem_u32(&bars[ps]));
            }
        }
        if (i >= 1 && loaded < n)
            ++loaded;                                    // every lane keeps the same count
    }
    if (leader) {
        if (!ok) {
            atomicMax(p.error_epoch, p.epoch);
            // let the loads already issued land before the CTA's shared memory goes away
            for (int64_t i = waited; i < loaded; ++i)
                mbar_wait_bounded(smem_u32(&bars[i % kBulkStages]), (uint32_t)((i / kBulkStages) & 1),
                                  100000000ull);
        }
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }
}

// Smallest E with 448 * 2^E >= amax (0 for amax == 0), clamped to [-127, 127].
// amax = m * 2^x with m in [1, 2): 448 = 1.75 * 2^8, so E = x - 8 when
// m <= 1.75 (mantissa field <= 0x600000) and x - 7 otherwise.  Every subnormal
// amax is below 448 * 2^-134 and clamps to -127.
__device__ __forceinline__ int ue8m0_exponent(float amax)
{
    const uint32_t u = __float_as_uint(amax);
    if (u == 0u)
        return 0;
    const int ex = (int)(u >> 23);
    if (ex == 0)
        return -127;
    const int e = ex - 127 - 8 + ((u & 0x7fffffu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^e as fp32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// fp8: a work item is (token, segment of seg_len 512-channel iterations).
template <int SCALE, bool PUBLISH>
__global__ void __launch_bounds__(kWarps * 32) dispatch_fp8_kernel(DispatchParams p)
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
            float amax = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q)
                amax = fmaxf(amax, fabsf(f[q]));
            amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 4));

            float scale_f = 1.f, inv = 1.f;
            int expo = 0;
            if (SCALE == SEP_SCALE_F32) {
                scale_f = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
            } else {
                expo = ue8m0_exponent(amax);
                scale_f = exp2_int(expo);
                inv = exp2_int(-expo);                    // exact: x * 2^-E == x / 2^E
            }
            uint32_t packed[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float a[4];
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    a[r] = SCALE == SEP_SCALE_F32 ? __fdiv_rn(f[4 * q + r], scale_f)
                                                  : __fmul_rn(f[4 * q + r], inv);
                const __nv_fp8x2_storage_t lo =
                    __nv_cvt_float2_to_fp8x2(make_float2(a[0], a[1]), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi =
                    __nv_cvt_float2_to_fp8x2(make_float2(a[2], a[3]), __NV_SATFINITE, __NV_E4M3);
                packed[q] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            const uint4 codes = make_uint4(packed[0], packed[1], packed[2], packed[3]);
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

// One warp per work item and no cap at the resident CTA count: CTAs that
// finish early make room for the rest, which balances the tail across SMs.
template <typename K>
int blocks_for(K, int64_t items, int)
{
    return (int)((items + kWarps - 1) / kWarps);
}

template <bool PUBLISH>
cudaError_t launch_fp8(const DispatchParams &p, cudaStream_t s, int num_sms)
{
    const dim3 grid(blocks_for(0, p.T * p.segs, num_sms)), block(kWarps * 32);
    switch (p.scale) {
    case SEP_SCALE_F32:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_F32, PUBLISH>, grid, block, 0, s, p);
    case SEP_SCALE_UE8M0:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_UE8M0, PUBLISH>, grid, block, 0, s, p);
    default:
        return launch_kernel(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, PUBLISH>, grid, block, 0, s, p);
    }
}

}  // namespace

// Row splitting.  A bf16 step is 128 vectors of 16 bytes (one pass of the
// kernel's 4-deep unroll); without tile publication every step is its own work
// item, so the items divide finely over the waves of CTAs (measured faster
// than whole rows per warp).  With tile publication a row stays on one warp
// where possible, since every item pays a fence and one arrival per row.  FP8
// steps are 512 channels, and a row splits over up to 7 warps.
constexpr int64_t kStepVecs = 128;
constexpr int64_t kMinSegs = 1 << 20;
constexpr int64_t kPublishMinSegs = 1;
constexpr int64_t kFp8MinSegs = 7;

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
    if (payload == SEP_PAYLOAD_BF16) {
        const int64_t smem = (int64_t)kBulkStages * p.H * 2;
        if (kBulkDispatch && p.tile_ready == nullptr && smem <= kBulkMaxSmem) {
            static int attr_set = 0;
            if (!attr_set) {
                cudaError_t e = cudaFuncSetAttribute(dispatch_bf16_bulk_kernel,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kBulkMaxSmem);
                if (e != cudaSuccess)
                    return e;
                attr_set = 1;
            }
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_bf16_bulk_kernel, 32, (size_t)smem) !=
                    cudaSuccess || per_sm < 1)
                per_sm = 1;
            const int64_t want = p.T;
            const int64_t cap = (int64_t)num_sms * per_sm;
            return launch_kernel(dispatch_bf16_bulk_kernel, dim3((int)(want < cap ? want : cap)), dim3(32),
                                 (size_t)smem, s, p);
        }
        if (p.tile_ready != nullptr)
            return launch_kernel(dispatch_bf16_kernel<4, true>, dim3(blocks_for(0, items, num_sms)),
                                 dim3(kWarps * 32), 0, s, p);
        return launch_kernel(dispatch_bf16_kernel<4, false>, dim3(blocks_for(0, items, num_sms)),
                             dim3(kWarps * 32), 0, s, p);
    }
    return p.tile_ready != nullptr ? launch_fp8<true>(p, s, num_sms) : launch_fp8<false>(p, s, num_sms);
}

cudaError_t preload_dispatch_kernels()
{
    const void *k[] = {
        reinterpret_cast<const void *>(dispatch_bf16_bulk_kernel),
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, false>),
        reinterpret_cast<const void *>(dispatch_bf16_kernel<4, true>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32, true>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_UE8M0, true>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, false>),
        reinterpret_cast<const void *>(dispatch_fp8_kernel<SEP_SCALE_F32_POW2, true>)};
    cudaFuncAttributes a;
    for (const void *f : k) {
        const cudaError_t e = cudaFuncGetAttributes(&a, f);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace sep
