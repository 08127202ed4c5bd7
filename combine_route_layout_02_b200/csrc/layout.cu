// Routing layout: per-expert histogram, pool-layout scan, stable slot
// assignment and inverse maps.
//
// What it computes (StreamEP README, "Streaming dispatch in one paragraph";
// "DeepEP MoE dispatch/combine" blog, "一轮 DeepEP 数据流": count assignments by
// destination/expert, then calculate layout and offsets):
//   n_e                        valid assignments of expert e
//   expert_pool_block_offset   exclusive prefix of ceil(n_e / BLOCK_M), in tiles
//   tile_expert / target       expert and valid-row count of every tile
//   src_pool_row[a]            offset[e]*BLOCK_M + (number of earlier valid a'
//                              with the same expert): a stable counting sort
//   pool_recv_token / _slot    the inverse map; -1 on padding rows
//   owner_counts               L_r = sum of n_e over owner r's experts (blog,
//                              "Imbalance 决定 buffer 与尾延迟")
//
// Three launches on one stream:
//   count   one warp per chunk of 32*rounds assignments; __match_any_sync
//           groups lanes holding the same expert so each distinct expert costs
//           one shared-memory update per round; writes a per-chunk histogram.
//   scan    one 1024-thread CTA: per-expert exclusive prefix over chunks (all
//           loads issued before any use), then a block scan of tiles over experts.
//   assign  the same chunk walk as count; a lane's row is its expert's cursor
//           plus the number of lower lanes holding that expert.  Also writes the
//           tile tables and marks padding rows, experts spread over CTAs.
// The chunk order and the in-warp lane order both follow ascending a, so the
// result is the unique stable order and needs no atomics on the data path.
#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;            // warps per CTA in count / assign
constexpr int kScanThreads = 1024;
constexpr int kScanMaxEPW = 8;       // experts per warp held in registers (E <= 256)
constexpr int kScanMaxGPE = 4;       // 32-chunk groups per expert in registers (<= 128 chunks)
constexpr int kPrefetch = 8;         // rounds whose ids are loaded before use

template <typename IdxT>
__device__ __forceinline__ int expert_of(const IdxT *__restrict__ idx, int64_t a, int64_t Na,
                                         int E, bool &bad)
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

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFullMask, v, o);
        if (lane >= o)
            v += n;
    }
    return v;
}

template <typename IdxT>
__global__ void __launch_bounds__(kWarps * 32) layout_count_kernel(LayoutParams p)
{
    extern __shared__ int32_t s_cnt[];                   // [kWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wc = (int64_t)blockIdx.x * kWarps + warp;
    if (wc >= p.num_wchunks)
        return;                                          // whole warp; no block barrier follows
    int32_t *cnt = s_cnt + warp * p.E;
    for (int e = lane; e < p.E; e += 32)
        cnt[e] = 0;
    __syncwarp();

    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);
    const int64_t a0 = wc * 32 * p.rounds;
    bool bad = false;
    for (int r = 0; r < p.rounds; r += kPrefetch) {
        int ev[kPrefetch];
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u)
            ev[u] = (r + u < p.rounds) ? expert_of(idx, a0 + (int64_t)(r + u) * 32 + lane, p.Na, p.E, bad)
                                       : -1;
#pragma unroll
        for (int u = 0; u < kPrefetch; ++u) {
            if (r + u >= p.rounds)
                break;                                   // warp-uniform
            const int e = ev[u];
            const unsigned peers = __match_any_sync(kFullMask, e);
            if (e >= 0 && lane == __ffs(peers) - 1)
                cnt[e] += __popc(peers);
            __syncwarp();
        }
    }
    for (int e = lane; e < p.E; e += 32)
        p.wchunk_hist[(int64_t)e * p.num_wchunks + wc] = cnt[e];
    if (__any_sync(kFullMask, bad) && lane == 0)
        atomicMax(p.bad_epoch, p.epoch);
}

__global__ void __launch_bounds__(kScanThreads) layout_scan_kernel(LayoutParams p)
{
    __shared__ int32_t s_cnt[1024];
    __shared__ int32_t s_off[1025];
    __shared__ int32_t s_wsum[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E, nw = p.num_wchunks;

    // 1. per expert: exclusive prefix of its chunk counts, and n_e
    if (E <= 32 * kScanMaxEPW && nw <= 32 * kScanMaxGPE) {
        int v[kScanMaxEPW][kScanMaxGPE];
#pragma unroll
        for (int i = 0; i < kScanMaxEPW; ++i) {
            const int e = warp + 32 * i;
#pragma unroll
            for (int g = 0; g < kScanMaxGPE; ++g) {
                const int c = g * 32 + lane;
                v[i][g] = (e < E && c < nw) ? p.wchunk_hist[(int64_t)e * nw + c] : 0;
            }
        }
#pragma unroll
        for (int i = 0; i < kScanMaxEPW; ++i) {
            const int e = warp + 32 * i;
            if (e >= E)
                break;                                   // warp-uniform
            int running = 0;
#pragma unroll
            for (int g = 0; g < kScanMaxGPE; ++g) {
                const int c = g * 32 + lane;
                const int incl = warp_inclusive_scan(v[i][g], lane);
                if (c < nw)
                    p.wchunk_base[(int64_t)e * nw + c] = running + incl - v[i][g];
                running += __shfl_sync(kFullMask, incl, 31);
            }
            if (lane == 0)
                s_cnt[e] = running;
        }
    } else {
        for (int e = warp; e < E; e += 32) {
            int running = 0;
            for (int c0 = 0; c0 < nw; c0 += 32) {
                const int c = c0 + lane;
                const int x = c < nw ? p.wchunk_hist[(int64_t)e * nw + c] : 0;
                const int incl = warp_inclusive_scan(x, lane);
                if (c < nw)
                    p.wchunk_base[(int64_t)e * nw + c] = running + incl - x;
                running += __shfl_sync(kFullMask, incl, 31);
            }
            if (lane == 0)
                s_cnt[e] = running;
        }
    }
    __syncthreads();

    // 2. tiles per expert, exclusive scan over experts (one expert per thread)
    const int e = threadIdx.x;
    const int tiles = e < E ? (s_cnt[e] + p.B - 1) / p.B : 0;
    const int incl = warp_inclusive_scan(tiles, lane);
    if (lane == 31)
        s_wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int ws = s_wsum[lane];
        s_wsum[lane] = warp_inclusive_scan(ws, lane) - ws;
    }
    __syncthreads();
    const int excl = s_wsum[warp] + incl - tiles;
    if (e < E) {
        s_off[e] = excl;
        p.expert_pool_block_offset[e] = excl;
        p.expert_counts[e] = s_cnt[e];
    }
    if (e == E - 1) {
        const int nt = excl + tiles;
        s_off[E] = nt;
        p.expert_pool_block_offset[E] = nt;
        p.sizes[0] = (int64_t)nt * p.B;
        p.sizes[1] = nt;
    }
    __syncthreads();

    // 3. owners: contiguous expert ranges
    const int E_loc = E / p.R;
    for (int r = threadIdx.x; r <= p.R; r += blockDim.x) {
        p.owner_pool_row_offset[r] = s_off[r * E_loc] * p.B;
        if (r < p.R) {
            int sum = 0;
            for (int q = r * E_loc; q < (r + 1) * E_loc; ++q)
                sum += s_cnt[q];
            p.owner_counts[r] = sum;
            p.owner_token_counts[r] = 0;
        }
    }
}

template <typename IdxT>
__global__ void __launch_bounds__(kWarps * 32) layout_assign_kernel(LayoutParams p)
{
    extern __shared__ int32_t s_cur[];                   // [kWarps][E] cursors, then [R]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t wc = (int64_t)blockIdx.x * kWarps + warp;
    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);

    if (wc < p.num_wchunks) {
        int32_t *cur = s_cur + warp * p.E;
        for (int e = lane; e < p.E; e += 32)
            cur[e] = p.expert_pool_block_offset[e] * p.B + p.wchunk_base[(int64_t)e * p.num_wchunks + wc];
        __syncwarp();
        const int64_t a0 = wc * 32 * p.rounds;
        const unsigned lower = (1u << lane) - 1u;
        bool bad = false;
        for (int r = 0; r < p.rounds; r += kPrefetch) {
            int ev[kPrefetch];
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u)
                ev[u] = (r + u < p.rounds)
                            ? expert_of(idx, a0 + (int64_t)(r + u) * 32 + lane, p.Na, p.E, bad)
                            : -1;
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u) {
                if (r + u >= p.rounds)
                    break;                               // warp-uniform
                const int64_t a = a0 + (int64_t)(r + u) * 32 + lane;
                const int e = ev[u];
                const unsigned peers = __match_any_sync(kFullMask, e);
                const int row = e >= 0 ? cur[e] + __popc(peers & lower) : -1;
                __syncwarp();
                if (e >= 0 && lane == __ffs(peers) - 1)
                    cur[e] += __popc(peers);
                __syncwarp();
                if (a < p.Na) {
                    p.src_pool_row[a] = row;
                    if (row >= 0) {
                        const unsigned t = (unsigned)a / (unsigned)p.k;
                        p.pool_recv_token[row] = (int32_t)t;
                        p.pool_recv_slot[row] = (int32_t)((unsigned)a - t * (unsigned)p.k);
                    }
                }
            }
        }
    }

    // tile tables and padding rows; experts spread over CTAs
    for (int e = blockIdx.x; e < p.E; e += gridDim.x) {
        const int t0 = p.expert_pool_block_offset[e];
        const int t1 = p.expert_pool_block_offset[e + 1];
        const int n = p.expert_counts[e];
        for (int i = threadIdx.x; i < t1 - t0; i += blockDim.x) {
            p.tile_expert[t0 + i] = e;
            p.pool_arrival_target[t0 + i] = min(p.B, n - i * p.B);
            p.pool_arrival_count[t0 + i] = 0u;
        }
        const int64_t r1 = (int64_t)t1 * p.B;
        for (int64_t row = (int64_t)t0 * p.B + n + threadIdx.x; row < r1; row += blockDim.x) {
            p.pool_recv_token[row] = -1;
            p.pool_recv_slot[row] = -1;
        }
    }

    // optional: which owners each token reaches, and per-owner token counts
    if (p.is_token_in_rank != nullptr) {
        int32_t *s_own = s_cur + kWarps * p.E;
        for (int r = threadIdx.x; r < p.R; r += blockDim.x)
            s_own[r] = 0;
        __syncthreads();
        const int E_loc = p.E / p.R;
        bool bad = false;
        for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < p.T;
             t += (int64_t)gridDim.x * blockDim.x) {
            uint8_t *dst = p.is_token_in_rank + t * p.R;
            if (p.R <= 64) {
                unsigned long long mask = 0ull;
                for (int j = 0; j < p.k; ++j) {
                    const int e = expert_of(idx, t * p.k + j, p.Na, p.E, bad);
                    if (e >= 0)
                        mask |= 1ull << (e / E_loc);
                }
                for (int r = 0; r < p.R; ++r) {
                    const int in = (int)((mask >> r) & 1ull);
                    dst[r] = (uint8_t)in;
                    if (in)
                        atomicAdd(&s_own[r], 1);
                }
            } else {
                for (int r = 0; r < p.R; ++r) {
                    int in = 0;
                    for (int j = 0; j < p.k; ++j) {
                        const int e = expert_of(idx, t * p.k + j, p.Na, p.E, bad);
                        in |= (e >= 0 && e / E_loc == r);
                    }
                    dst[r] = (uint8_t)in;
                    if (in)
                        atomicAdd(&s_own[r], 1);
                }
            }
        }
        __syncthreads();
        for (int r = threadIdx.x; r < p.R; r += blockDim.x)
            if (s_own[r])
                atomicAdd(&p.owner_token_counts[r], s_own[r]);
    }
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p, cudaStream_t s)
{
    const int blocks = (p.num_wchunks + kWarps - 1) / kWarps;
    const size_t smem_count = (size_t)kWarps * p.E * sizeof(int32_t);
    const size_t smem_assign = smem_count + (size_t)p.R * sizeof(int32_t);
    if (blocks > 0)
        layout_count_kernel<IdxT><<<blocks, kWarps * 32, smem_count, s>>>(p);
    layout_scan_kernel<<<1, kScanThreads, 0, s>>>(p);
    const int ablocks = max(blocks, min(p.E, 64));
    layout_assign_kernel<IdxT><<<ablocks, kWarps * 32, smem_assign, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int layout_rounds_for(int64_t Na)
{
    // about 128 chunks, 1..64 rounds of 32 assignments per chunk
    int64_t r = (Na + 32 * 128 - 1) / (32 * 128);
    if (r < 1)
        r = 1;
    if (r > 64)
        r = 64;
    return (int)r;
}

int64_t layout_wchunks_for(int64_t Na, int rounds)
{
    return (Na + 32LL * rounds - 1) / (32LL * rounds);
}

int64_t layout_wchunk_capacity(int64_t Na_cap)
{
    // rounds < 64 keeps the count at or below 128; at 64 rounds it grows with Na
    const int64_t big = (Na_cap + 32LL * 64 - 1) / (32LL * 64);
    return big > 128 ? big : 128;
}

cudaError_t launch_layout(const LayoutParams &p, int idx_bytes, cudaStream_t s)
{
    return idx_bytes == 8 ? launch_layout_t<long long>(p, s) : launch_layout_t<int>(p, s);
}

cudaError_t preload_layout_kernels()
{
    const void *k[] = {reinterpret_cast<const void *>(layout_count_kernel<int>),
                       reinterpret_cast<const void *>(layout_count_kernel<long long>),
                       reinterpret_cast<const void *>(layout_scan_kernel),
                       reinterpret_cast<const void *>(layout_assign_kernel<int>),
                       reinterpret_cast<const void *>(layout_assign_kernel<long long>)};
    cudaFuncAttributes a;
    for (const void *f : k) {
        const cudaError_t e = cudaFuncGetAttributes(&a, f);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace sep
