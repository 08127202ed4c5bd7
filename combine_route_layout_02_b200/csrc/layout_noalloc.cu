// sep_layout_noalloc: the routing layout without any allocation.
//
// For callers that cannot allocate device memory on this path (a runtime that
// has handed HBM to its own pool, code where an allocation would synchronise
// the device, fixed-footprint deployments).  It computes what sep_layout
// computes, into caller-owned arrays, using as working memory one file-scope
// __device__ array instead of a handle's allocation.  Not an operation of the
// pages; see include/sep.h for the contract.
//
// The kernel is the single-launch layout (count -> per-expert scan -> offsets
// and stable assignment, split by two bounded grid barriers) restated for
// caller-owned outputs; it writes no arrival counters, owner token counts or
// token-owner flags (those belong to a handle).
#include <atomic>
#include <cstring>

#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kPrefetch = 8;
constexpr int kMaxExperts = 256;
constexpr int kMaxChunks = 128;
constexpr int64_t kMaxAssignments = 64LL * kWarps * 32 * kMaxChunks;   // 2^21
constexpr int kTableInts = kMaxExperts * kMaxChunks;                   // one [E][chunk] table
constexpr int kScratchInts = 2 * kTableInts + 64;                      // two tables + barrier word

// The working memory: [0, T) chunk histograms, [T, 2T) chunk bases, then the
// barrier counter.  256 KB + 256 B, held by every GPU that loads the library.
__device__ __align__(256) int32_t g_noalloc_scratch[kScratchInts];

struct NoAllocParams {
    const void *topk_idx;
    int64_t T, Na;
    int k, E, R, B, rounds, chunks;
    int32_t *hist, *base;
    unsigned *barrier;
    sep_layout_arrays out;
};

template <typename IdxT>
__device__ __forceinline__ int expert_at(const IdxT *idx, int64_t a, int64_t Na, int E, bool &bad)
{
    if (a >= Na)
        return -1;
    const long long v = (long long)__ldg(idx + a);
    if (v < 0)
        return -1;
    if (v >= E) {
        bad = true;
        return -1;
    }
    return (int)v;
}

__device__ __forceinline__ int inclusive_scan32(int v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o)
            v += n;
    }
    return v;
}

__device__ __forceinline__ bool barrier_wait(const NoAllocParams &p, unsigned target, int *s_flag)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(p.barrier, 1u);
        bool ok = false;
        uint64_t t0, t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
        for (uint32_t it = 0; it < (1u << 22); ++it) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.barrier) : "memory");
            if ((int)(v - target) >= 0) {
                ok = true;
                break;
            }
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > 200000000ull)
                break;
            __nanosleep(64);
        }
        __threadfence();
        if (!ok)
            atomicExch(p.out.status + 1, 1u);
        *s_flag = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

template <typename IdxT>
__device__ __forceinline__ void walk(const NoAllocParams &p, const IdxT *idx, int64_t a0, int32_t *cnt, int lane,
                                     bool assign, bool &bad)
{
    const unsigned lower = (1u << lane) - 1u;
    for (int r = 0; r < p.rounds; r += kPrefetch) {
        int ev[kPrefetch];
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u)
            ev[u] = (r + u < p.rounds) ? expert_at(idx, a0 + (int64_t)(r + u) * 32 + lane, p.Na, p.E, bad) : -1;
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) {
            if (r + u >= p.rounds)
                break;                                   // warp-uniform
            const int64_t a = a0 + (int64_t)(r + u) * 32 + lane;
            const int e = ev[u];
            const unsigned peers = __match_any_sync(kFullMask, e);
            const int row = (assign && e >= 0) ? cnt[e] + __popc(peers & lower) : -1;
            __syncwarp();
            if (e >= 0 && lane == __ffs(peers) - 1)
                cnt[e] += __popc(peers);
            __syncwarp();
            if (assign && a < p.Na) {
                p.out.src_pool_row[a] = row;
                if (row >= 0) {
                    const unsigned t = (unsigned)a / (unsigned)p.k;
                    p.out.pool_recv_token[row] = (int32_t)t;
                    p.out.pool_recv_slot[row] = (int32_t)((unsigned)a - t * (unsigned)p.k);
                }
            }
        }
    }
}

template <typename IdxT>
__global__ void __launch_bounds__(kWarps * 32) layout_noalloc_kernel(NoAllocParams p)
{
    __shared__ int32_t s_cnt[kWarps * kMaxExperts];
    __shared__ int32_t s_off[kMaxExperts + 1];
    __shared__ int s_part[kWarps];
    __shared__ int s_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, G = gridDim.x, E = p.E, nc = p.chunks;
    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);

    // count this CTA's chunk
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x)
        s_cnt[i] = 0;
    __syncthreads();
    const int64_t a0 = ((int64_t)c * kWarps + warp) * 32 * p.rounds;
    bool bad = false;
    walk(p, idx, a0, s_cnt + warp * E, lane, false, bad);
    if (__any_sync(kFullMask, bad) && lane == 0)
        atomicExch(p.out.status, 1u);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int sum = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            sum += s_cnt[w * E + e];
        p.hist[e * nc + c] = sum;
    }
    if (!barrier_wait(p, (unsigned)G, &s_flag))
        return;

    // per-expert exclusive scan over chunks, one warp per expert
    for (int e = c * kWarps + warp; e < E; e += G * kWarps) {
        int running = 0;
        for (int c0 = 0; c0 < nc; c0 += 32) {
            const int cc = c0 + lane;
            const int x = cc < nc ? __ldcg(p.hist + e * nc + cc) : 0;
            const int incl = inclusive_scan32(x, lane);
            if (cc < nc)
                p.base[e * nc + cc] = running + incl - x;
            running += __shfl_sync(kFullMask, incl, 31);
        }
        if (lane == 0)
            p.out.expert_counts[e] = running;
    }
    if (!barrier_wait(p, 2u * (unsigned)G, &s_flag))
        return;

    // tile offsets over experts (E <= 256: one expert per thread)
    const int e = threadIdx.x;
    const int tiles = e < E ? (__ldcg(p.out.expert_counts + e) + p.B - 1) / p.B : 0;
    const int incl = inclusive_scan32(tiles, lane);
    if (lane == 31)
        s_part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < kWarps ? s_part[lane] : 0;
        const int i2 = inclusive_scan32(v, lane);
        if (lane < kWarps)
            s_part[lane] = i2 - v;
    }
    __syncthreads();
    if (e < E)
        s_off[e] = s_part[warp] + incl - tiles;
    if (e == E - 1)
        s_off[E] = s_part[warp] + incl;
    __syncthreads();
    if (c == 0) {
        for (int q = threadIdx.x; q <= E; q += blockDim.x)
            p.out.expert_pool_block_offset[q] = s_off[q];
        if (threadIdx.x == 0) {
            p.out.sizes[0] = (int64_t)s_off[E] * p.B;
            p.out.sizes[1] = s_off[E];
        }
        const int E_loc = E / p.R;
        for (int r = threadIdx.x; r <= p.R; r += blockDim.x) {
            p.out.owner_pool_row_offset[r] = s_off[r * E_loc] * p.B;
            if (r < p.R) {
                int sum = 0;
                for (int q = r * E_loc; q < (r + 1) * E_loc; ++q)
                    sum += __ldcg(p.out.expert_counts + q);
                p.out.owner_counts[r] = sum;
            }
        }
    }
    // warp counts -> cursors, then the stable assignment walk
    for (int q = threadIdx.x; q < E; q += blockDim.x) {
        int cur = s_off[q] * p.B + __ldcg(p.base + q * nc + c);
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int n = s_cnt[w * E + q];
            s_cnt[w * E + q] = cur;
            cur += n;
        }
    }
    __syncthreads();
    walk(p, idx, a0, s_cnt + warp * E, lane, true, bad);
    // tile tables and padding rows, experts spread over CTAs
    for (int q = c; q < E; q += G) {
        const int t0 = s_off[q], t1 = s_off[q + 1];
        const int n = __ldcg(p.out.expert_counts + q);
        for (int i = threadIdx.x; i < t1 - t0; i += blockDim.x) {
            p.out.tile_expert[t0 + i] = q;
            p.out.pool_arrival_target[t0 + i] = min(p.B, n - i * p.B);
        }
        for (int64_t row = (int64_t)t0 * p.B + n + threadIdx.x; row < (int64_t)t1 * p.B; row += blockDim.x) {
            p.out.pool_recv_token[row] = -1;
            p.out.pool_recv_slot[row] = -1;
        }
    }
}

// Device address of the scratch array, looked up once per device.  Threads
// that make their first call at the same time may both look it up; they store
// the same value, and the atomics make that well defined.
std::atomic<int32_t *> g_scratch_addr[64] = {};

bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace
}  // namespace sep

extern "C" sep_status sep_layout_noalloc(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                                         int num_experts, int num_owners, int block_m,
                                         const sep_layout_arrays *out, void *stream)
{
    using namespace sep;
    const int64_t T = num_tokens;
    const int k = top_k, E = num_experts, R = num_owners, B = block_m;
    if (out == nullptr)
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: out is NULL");
    if (idx_bytes != 4 && idx_bytes != 8)
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: idx_bytes must be 4 or 8");
    if (T < 0 || k < 1 || k > 32 || B < 1 || B > 1024 || R < 1 || E < 1 || R > E || E % R != 0)
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: need T >= 0, 1 <= top_k <= 32, "
                                              "1 <= block_m <= 1024, num_owners dividing num_experts");
    if (E > kMaxExperts)
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: num_experts exceeds its limit of 256");
    if (T * k > kMaxAssignments)
        return set_error(SEP_ERR_INVALID_ARG,
                         "sep_layout_noalloc: num_tokens * top_k exceeds its limit of 2097152");
    if (T > 0 && topk_idx == nullptr)
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: topk_idx is NULL");
    if (!aligned(topk_idx, (uintptr_t)idx_bytes))
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: topk_idx is misaligned");
    const sep_layout_arrays &o = *out;
    const void *int_arrays[] = {o.expert_counts, o.owner_counts, o.expert_pool_block_offset,
                                o.owner_pool_row_offset, o.tile_expert, o.pool_arrival_target, o.src_pool_row,
                                o.pool_recv_token, o.pool_recv_slot, o.status};
    for (const void *a : int_arrays)
        if (a == nullptr || !aligned(a, 4))
            return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: an output array is NULL or misaligned");
    if (o.sizes == nullptr || !aligned(o.sizes, 8))
        return set_error(SEP_ERR_INVALID_ARG, "sep_layout_noalloc: sizes is NULL or misaligned");
    const int64_t Na = T * k;
    const int64_t used = Na < E ? Na : E;
    const int64_t worst_rows = (Na + used * (B - 1) + B - 1) / B * B;
    if (o.max_pool_rows < worst_rows || o.max_tiles < worst_rows / B)
        return set_error(SEP_ERR_CAPACITY, "sep_layout_noalloc: max_pool_rows / max_tiles below the worst "
                                           "case for this num_tokens");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64)
        return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: cudaGetDevice failed");
    int32_t *scratch = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (scratch == nullptr) {
        // set-up, once per device with that device current: the array's device
        // address (host code only sees a host-side stand-in for it) and the
        // kernels loaded now rather than lazily at a later launch
        void *addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
        if (e != cudaSuccess || addr == nullptr)
            return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: cudaGetSymbolAddress of the scratch array failed");
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(layout_noalloc_kernel<int>)) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(layout_noalloc_kernel<long long>)) != cudaSuccess)
            return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: loading its kernels failed");
        scratch = static_cast<int32_t *>(addr);
        g_scratch_addr[dev].store(scratch, std::memory_order_release);
    }

    NoAllocParams p{};
    p.topk_idx = topk_idx;
    p.T = T;
    p.Na = Na;
    p.k = k;
    p.E = E;
    p.R = R;
    p.B = B;
    int64_t rounds = (Na + 32LL * kWarps * kMaxChunks - 1) / (32LL * kWarps * kMaxChunks);
    rounds = rounds < 1 ? 1 : rounds;
    p.rounds = (int)rounds;
    const int64_t chunks = (Na + 32LL * kWarps * rounds - 1) / (32LL * kWarps * rounds);
    p.chunks = (int)(chunks > 0 ? chunks : 1);
    p.hist = scratch;
    p.base = scratch + kTableInts;
    p.barrier = reinterpret_cast<unsigned *>(scratch + 2 * kTableInts);
    p.out = o;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((e = cudaMemsetAsync(p.barrier, 0, sizeof(unsigned), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(o.status, 0, 2 * sizeof(uint32_t), s)) != cudaSuccess)
        return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: clearing the barrier/status words failed");
    const void *kernel = idx_bytes == 8 ? reinterpret_cast<const void *>(layout_noalloc_kernel<long long>)
                                        : reinterpret_cast<const void *>(layout_noalloc_kernel<int>);
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kWarps * 32, 0) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || p.chunks > per_sm * sms)
        return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: the layout grid cannot be co-resident");
    void *args[] = {&p};
    count_launch();
    e = cudaLaunchCooperativeKernel(kernel, dim3(p.chunks), dim3(kWarps * 32), args, 0, s);
    if (e != cudaSuccess)
        return set_error(SEP_ERR_CUDA, "sep_layout_noalloc: launch failed");
    return SEP_OK;
}
