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
// Three launches on one stream.  The assignment stream is cut into at most
// 128 CTA chunks of 8 warps x 32 lanes x `rounds` entries; warp w of chunk c
// owns a contiguous run of 32*rounds entries, so chunk order, warp order and
// lane order all follow ascending a.
//   count   per warp, __match_any_sync groups lanes holding the same expert so
//           each distinct expert costs one shared-memory add per round; the
//           CTA sums its warps and writes one histogram column [E][chunk].
//   scan    one 1024-thread CTA: per-expert exclusive prefix over chunks (all
//           loads issued before any use), then a block scan of tiles over experts.
//   assign  recounts its chunk per warp, turns the warp counts into cursors
//           (expert's pool start + chunk prefix + earlier warps of the chunk),
//           then walks the chunk again: a lane's row is its expert's cursor
//           plus the number of lower lanes holding that expert.  Also writes
//           the tile tables and marks padding rows, experts spread over CTAs.
// The result is the unique stable order and needs no atomics on the data path.
#include <atomic>
#include <mutex>

#include "fp8_quant.cuh"
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

// Per-warp expert counts of the warp's run of the chunk into cnt[E] (shared).
template <typename IdxT>
__device__ __forceinline__ void count_warp_run(const LayoutParams &p, const IdxT *idx, int64_t a0,
                                               int32_t *cnt, int lane, bool &bad)
{
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
}

template <typename IdxT>
__global__ void __launch_bounds__(kWarps * 32) layout_count_kernel(LayoutParams p)
{
    extern __shared__ int32_t s_cnt[];                   // [kWarps][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    for (int i = threadIdx.x; i < kWarps * p.E; i += blockDim.x)
        s_cnt[i] = 0;
    __syncthreads();
    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);
    const int64_t a0 = ((int64_t)c * kWarps + warp) * 32 * p.rounds;
    bool bad = false;
    count_warp_run(p, idx, a0, s_cnt + warp * p.E, lane, bad);
    if (__any_sync(kFullMask, bad) && lane == 0)
        atomicMax(p.bad_epoch, p.epoch);
    __syncthreads();
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
        int sum = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w)
            sum += s_cnt[w * p.E + e];
        p.wchunk_hist[(int64_t)e * p.num_wchunks + c] = sum;
    }
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
    allow_dependents();
    extern __shared__ int32_t s_cur[];                   // [kWarps][E] cursors, then [R]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);

    if (c < p.num_wchunks) {                             // block-uniform
        for (int i = threadIdx.x; i < kWarps * p.E; i += blockDim.x)
            s_cur[i] = 0;
        __syncthreads();
        const int64_t a0 = ((int64_t)c * kWarps + warp) * 32 * p.rounds;
        bool bad = false;
        count_warp_run(p, idx, a0, s_cur + warp * p.E, lane, bad);
        __syncthreads();
        // warp counts -> cursors: pool start of e + earlier chunks + earlier warps
        for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
            int run = p.expert_pool_block_offset[e] * p.B + p.wchunk_base[(int64_t)e * p.num_wchunks + c];
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const int n = s_cur[w * p.E + e];
                s_cur[w * p.E + e] = run;
                run += n;
            }
        }
        __syncthreads();
        int32_t *cur = s_cur + warp * p.E;
        const unsigned lower = (1u << lane) - 1u;
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
        __syncthreads();                                 // s_cur is reused below
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

// ------------------------------------------------------- single launch
//
// The same computation in one cooperative launch (every CTA resident) with a
// single grid barrier:
//   A  count this CTA's chunk per warp (shared memory); write the CTA's row
//      hist[c][0..E) of a chunk-major table whose row stride is E rounded up
//      to 4 (the padding is written as zeros)
//   -- grid barrier --
//   B  every CTA reads the whole table with 16-byte loads (one L2 round trip
//      at 128 chunks x 128 experts) and reduces it to n_e over all chunks and
//      to its own prefix over the chunks before it; the scan of
//      ceil(n_e / BLOCK_M) over experts follows in shared memory; CTA 0
//      writes the counts, offsets, sizes and owner arrays
//   C  the warp counts of A become cursors and the chunk is walked again
//   D  tile tables and padding rows, one warp per expert
// A routing small enough for one CTA chunk skips the table and the barrier.
// The barrier arrives with atom.release and waits with ld.acquire, bounded; a
// barrier that gives up records the epoch in the handle's timeout word and the
// kernel returns (sep_handle_sync reports it).  The counter is never reset:
// each launch advances it by one fixed window (see grid_barrier).

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *ptr)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// A launch moves the barrier counter by exactly kBarrierWindow, whatever its
// grid size G (< kBarrierWindow): CTA 0 adds kBarrierWindow - (G - 1), every other CTA
// adds 1.  So every arrival of one launch returns an old value inside the same
// window [base, base + kBarrierWindow), the window is found from the old value
// alone, and the counter never needs a reset: the barrier depends on no host
// state and stays correct when the launch is replayed from a CUDA graph.
// 2^32 is a multiple of the window, so the counter may wrap.
constexpr unsigned kBarrierWindow = 4096;

// CTAs 0..G-1 arrive on *counter; false (in every thread of the CTA) if the
// window did not fill within the limit.
__device__ __forceinline__ bool grid_barrier(const LayoutParams &p, unsigned *counter, int *s_flag, int c, int G)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned add = c == 0 ? kBarrierWindow - (unsigned)(G - 1) : 1u;
        unsigned old;
        asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(counter), "r"(add) : "memory");
        const unsigned target = (old & ~(kBarrierWindow - 1)) + kBarrierWindow;
        bool ok = false;
        const uint64_t t0 = global_ns();
        for (uint32_t it = 0; it < (1u << 22); ++it) {
            if ((int)(ld_acquire_u32(counter) - target) >= 0) {
                ok = true;
                break;
            }
            if (global_ns() - t0 > 200000000ull)
                break;
            __nanosleep(32);
        }
        if (!ok)
            atomicMax(p.timeout_epoch, p.epoch);
        *s_flag = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

constexpr int64_t kSingleCtaMaxNa = 1024;     // routings this small run as one CTA chunk

constexpr int kFusedThreads = kWarps * 32;
constexpr int kRedInts = 2048;               // per reduction table: row groups x padded experts
// chunk table of 16-bit counts for the 8-warp chunks (a chunk holds at most
// 16 384 assignments): train8k step 152.1 against 152.6 us, prefill_skew 573.0
// against 573.9; the 4-warp chunks of a decode step keep 32-bit entries (their
// table is 16 rows; 27.3 against 27.6 us)
constexpr bool kTable16 = true;

// Chunk c of the G = p.num_wchunks chunks of the layout, run by one CTA
// (phases A to D above).  sm: the dynamic shared memory of
// layout_smem_bytes(); false if its grid barrier gave up.
template <typename IdxT, int WARPS = kWarps>
__device__ bool layout_chunk(const LayoutParams &p, const int c, const int G, int32_t *sm, int &s_flag,
                             int *s_part)
{
    const int E = p.E, nc = p.num_wchunks;
    const int hs = (E + 3) & ~3;                         // padded row stride of the chunk table
    int32_t *s_red = sm;                                 // [2][kRedInts], read and written as int4: first
    int32_t *s_cnt = s_red + 2 * kRedInts;               // [WARPS][E]
    int32_t *s_off = s_cnt + WARPS * E;                 // [E+1]
    int32_t *s_tot = s_off + E + 1;                      // [E]
    int32_t *s_pre = s_tot + E;                          // [E]
    int32_t *s_own = s_pre + E;                          // [R]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const IdxT *idx = static_cast<const IdxT *>(p.topk_idx);
    unsigned *counter = p.barrier_words;
    if (c == 0)
        for (int r = tid; r < p.R; r += blockDim.x)
            p.owner_token_counts[r] = 0;

    // A. count
    for (int i = tid; i < WARPS * E; i += blockDim.x)
        s_cnt[i] = 0;
    __syncthreads();
    const int64_t a0 = ((int64_t)c * WARPS + warp) * 32 * p.rounds;
    bool bad = false;
    count_warp_run(p, idx, a0, s_cnt + warp * E, lane, bad);
    if (__any_sync(kFullMask, bad) && lane == 0)
        atomicMax(p.bad_epoch, p.epoch);
    __syncthreads();
    if (G == 1) {
        // one chunk: the totals are this CTA's own counts; no table, no grid barrier
        for (int e = tid; e < E; e += blockDim.x) {
            int sum = 0;
#pragma unroll
            for (int w = 0; w < WARPS; ++w)
                sum += s_cnt[w * E + e];
            s_tot[e] = sum;
            s_pre[e] = 0;
        }
        __syncthreads();
    } else {
    if (kTable16 && WARPS >= 8) {
        // 16-bit entries (a chunk holds at most 16 384 assignments): half the bytes
        // to write here and for every CTA to read after the barrier
        const int hs16 = (E + 7) & ~7;
        uint16_t *hist16 = reinterpret_cast<uint16_t *>(p.wchunk_hist);
        for (int e = tid; e < hs16; e += blockDim.x) {
            int sum = 0;
            if (e < E) {
#pragma unroll
                for (int w = 0; w < WARPS; ++w)
                    sum += s_cnt[w * E + e];
            }
            hist16[(int64_t)c * hs16 + e] = (uint16_t)sum;
        }
    } else {
    for (int e = tid; e < hs; e += blockDim.x) {
        int sum = 0;
        if (e < E) {
#pragma unroll
            for (int w = 0; w < WARPS; ++w)
                sum += s_cnt[w * E + e];
        }
        p.wchunk_hist[(int64_t)c * hs + e] = sum;
    }
    }
    if (!grid_barrier(p, counter, &s_flag, c, G))
        return false;

    // B. totals and this chunk's prefix, from the whole table
    if (kTable16 && WARPS >= 8) {
        constexpr int TH = WARPS * 32;
        const int cols = ((E + 7) & ~7) / 8;             // 16-byte columns of eight 16-bit counts per row
        const int span = min(cols, TH);
        const int groups = TH / cols > 0 ? TH / cols : 1;
        for (int q0 = 0; q0 < cols; q0 += TH) {
            const int q = q0 + tid % span;
            const int g = tid / span;
            int tot[8], pre[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                tot[i] = pre[i] = 0;
            if (g < groups && q < cols) {
                const uint4 *col = reinterpret_cast<const uint4 *>(p.wchunk_hist) + q;
                int r = g;
                for (; r + 3 * groups < nc; r += 4 * groups) {
                    uint4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = __ldcg(col + (int64_t)(r + u * groups) * cols);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                        const bool before = r + u * groups < c;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int lo = (int)(w4[i] & 0xffffu), hi = (int)(w4[i] >> 16);
                            tot[2 * i] += lo;
                            tot[2 * i + 1] += hi;
                            if (before) {
                                pre[2 * i] += lo;
                                pre[2 * i + 1] += hi;
                            }
                        }
                    }
                }
                for (; r < nc; r += groups) {
                    const uint4 v = __ldcg(col + (int64_t)r * cols);
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int lo = (int)(w4[i] & 0xffffu), hi = (int)(w4[i] >> 16);
                        tot[2 * i] += lo;
                        tot[2 * i + 1] += hi;
                        if (r < c) {
                            pre[2 * i] += lo;
                            pre[2 * i + 1] += hi;
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    s_red[(g * span + q - q0) * 8 + i] = tot[i];
                    s_red[kRedInts + (g * span + q - q0) * 8 + i] = pre[i];
                }
            }
            __syncthreads();
            for (int e = tid; e < min(8 * (cols - q0), 8 * TH); e += blockDim.x) {
                const int ee = 8 * q0 + e;
                if (ee < E) {
                    int t = 0, b = 0;
                    for (int gg = 0; gg < groups; ++gg) {
                        t += s_red[gg * 8 * span + e];
                        b += s_red[kRedInts + gg * 8 * span + e];
                    }
                    s_tot[ee] = t;
                    s_pre[ee] = b;
                }
            }
            __syncthreads();
        }
    } else {
        const int cols = hs / 4;                         // int4 columns per row
        const int groups = (WARPS * 32) / cols > 0 ? (WARPS * 32) / cols : 1;
        for (int q0 = 0; q0 < cols; q0 += (WARPS * 32)) {   // more than 1024 experts never happens
            const int q = q0 + tid % min(cols, (WARPS * 32));
            const int g = tid / min(cols, (WARPS * 32));
            int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
            if (g < groups && q < cols) {
                const int4 *col = reinterpret_cast<const int4 *>(p.wchunk_hist) + q;
                int r = g;
                for (; r + 3 * groups < nc; r += 4 * groups) {
                    int4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        v[u] = __ldcg(col + (int64_t)(r + u * groups) * cols);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        tot.x += v[u].x; tot.y += v[u].y; tot.z += v[u].z; tot.w += v[u].w;
                        if (r + u * groups < c) {
                            pre.x += v[u].x; pre.y += v[u].y; pre.z += v[u].z; pre.w += v[u].w;
                        }
                    }
                }
                for (; r < nc; r += groups) {
                    const int4 v = __ldcg(col + (int64_t)r * cols);
                    tot.x += v.x; tot.y += v.y; tot.z += v.z; tot.w += v.w;
                    if (r < c) {
                        pre.x += v.x; pre.y += v.y; pre.z += v.z; pre.w += v.w;
                    }
                }
                reinterpret_cast<int4 *>(s_red)[g * cols + q - q0] = tot;
                reinterpret_cast<int4 *>(s_red + kRedInts)[g * cols + q - q0] = pre;
            }
            __syncthreads();
            for (int e = tid; e < min(4 * (cols - q0), 4 * (WARPS * 32)); e += blockDim.x) {
                const int ee = 4 * q0 + e;
                if (ee < E) {
                    int t = 0, b = 0;
                    for (int gg = 0; gg < groups; ++gg) {
                        t += s_red[gg * 4 * min(cols, (WARPS * 32)) + e];
                        b += s_red[kRedInts + gg * 4 * min(cols, (WARPS * 32)) + e];
                    }
                    s_tot[ee] = t;
                    s_pre[ee] = b;
                }
            }
            __syncthreads();
        }
    }
    }

    // tile offsets over experts (each thread a run of experts), in shared memory
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = tid * per;
    int local = 0;
    for (int e = e0; e < min(E, e0 + per); ++e)
        local += (s_tot[e] + p.B - 1) / p.B;
    const int incl = warp_inclusive_scan(local, lane);
    if (lane == 31)
        s_part[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < WARPS ? s_part[lane] : 0;
        const int inc2 = warp_inclusive_scan(v, lane);
        if (lane < WARPS)
            s_part[lane] = inc2 - v;
    }
    __syncthreads();
    int run = s_part[warp] + incl - local;
    for (int e = e0; e < min(E, e0 + per); ++e) {
        s_off[e] = run;
        run += (s_tot[e] + p.B - 1) / p.B;
    }
    if (tid == blockDim.x - 1)
        s_off[E] = s_part[warp] + incl;                  // the last thread holds the grand total
    __syncthreads();
    if (c == 0) {
        for (int e = tid; e <= E; e += blockDim.x) {
            p.expert_pool_block_offset[e] = s_off[e];
            if (e < E)
                p.expert_counts[e] = s_tot[e];
        }
        if (tid == 0) {
            p.sizes[0] = (int64_t)s_off[E] * p.B;
            p.sizes[1] = s_off[E];
        }
        const int E_loc = E / p.R;
        for (int r = tid; r <= p.R; r += blockDim.x) {
            p.owner_pool_row_offset[r] = s_off[r * E_loc] * p.B;
            if (r < p.R) {
                int sum = 0;
                for (int q = r * E_loc; q < (r + 1) * E_loc; ++q)
                    sum += s_tot[q];
                p.owner_counts[r] = sum;
            }
        }
    }

    // C. warp counts -> cursors, then the assignment walk
    for (int e = tid; e < E; e += blockDim.x) {
        int cur = s_off[e] * p.B + s_pre[e];
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const int n = s_cnt[w * E + e];
            s_cnt[w * E + e] = cur;
            cur += n;
        }
    }
    __syncthreads();
    {
        int32_t *cur = s_cnt + warp * E;
        const unsigned lower = (1u << lane) - 1u;
        for (int r = 0; r < p.rounds; r += kPrefetch) {
            int ev[kPrefetch];
#pragma unroll
            for (int u = 0; u < kPrefetch; ++u)
                ev[u] = (r + u < p.rounds)
                            ? expert_of(idx, a0 + (int64_t)(r + u) * 32 + lane, p.Na, E, bad)
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

    // D. tile tables and padding rows; one warp per expert, experts spread over
    // the warps of all CTAs
    for (int e = c * WARPS + warp; e < E; e += G * WARPS) {
        const int t0 = s_off[e], t1 = s_off[e + 1];
        const int n = s_tot[e];
        for (int i = lane; i < t1 - t0; i += 32) {
            p.tile_expert[t0 + i] = e;
            p.pool_arrival_target[t0 + i] = min(p.B, n - i * p.B);
            p.pool_arrival_count[t0 + i] = 0u;
        }
        const int64_t r1 = (int64_t)t1 * p.B;
        for (int64_t row = (int64_t)t0 * p.B + n + lane; row < r1; row += 32) {
            p.pool_recv_token[row] = -1;
            p.pool_recv_slot[row] = -1;
        }
    }
    // optional: which owners each token reaches, and per-owner token counts
    if (p.is_token_in_rank != nullptr) {
        for (int r = tid; r < p.R; r += blockDim.x)
            s_own[r] = 0;
        __syncthreads();
        const int E_loc = E / p.R;
        for (int64_t t = (int64_t)c * blockDim.x + tid; t < p.T; t += (int64_t)G * blockDim.x) {
            uint8_t *dst = p.is_token_in_rank + t * p.R;
            for (int r = 0; r < p.R; ++r) {
                int in = 0;
                for (int j = 0; j < p.k; ++j) {
                    const int e = expert_of(idx, t * p.k + j, p.Na, E, bad);
                    in |= (e >= 0 && e / E_loc == r);
                }
                dst[r] = (uint8_t)in;
                if (in)
                    atomicAdd(&s_own[r], 1);
            }
        }
        __syncthreads();
        for (int r = tid; r < p.R; r += blockDim.x)
            if (s_own[r])
                atomicAdd(&p.owner_token_counts[r], s_own[r]);
    }
    return true;
}

size_t layout_smem_bytes(const LayoutParams &p, int warps = kWarps)
{
    return (size_t)(warps * p.E + 3 * p.E + 1 + 2 * kRedInts + p.R) * sizeof(int32_t);
}

template <typename IdxT, int WARPS = kWarps>
__global__ void __launch_bounds__(WARPS * 32) layout_fused_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t sm[];
    __shared__ int s_flag;
    __shared__ int s_part[WARPS];
    grid_dependency_wait();                              // launched dependent (one CTA): the previous kernel's
    allow_dependents();                                  // writes first; a no-op for a cooperative launch
    layout_chunk<IdxT, WARPS>(p, blockIdx.x, gridDim.x, sm, s_flag, s_part);
}

// Routings of 1025 to 4096 assignments (a decode step) in narrower chunks:
// kNarrowWarps warps per CTA, one 32-entry round per warp, so more CTAs (and
// SMs) share the layout's latency-bound phases (decode: 16 CTAs of 4 warps,
// 26.9 against 27.6 us per step, graph replay 28.1 against 28.6).  Smaller
// routings keep one CTA of 8 warps, which needs no grid barrier.
constexpr int kNarrowWarps = 4;
constexpr int64_t kNarrowMinNa = 1025;
constexpr int64_t kNarrowMaxNa = 4096;

// ------------------------------------------- layout and dispatch, one launch
//
// For small routings (a decode step): one cooperative launch runs the layout
// in its first nc = num_wchunks CTAs (exactly as above, its grid barrier among
// those CTAs) and the dispatch in the other CTAs.  A dispatch warp loads its
// items of x, and for FP8 quantises them, into registers while the layout is
// still running; it then waits for the layout and stores the items to the
// token's pool rows.  Items: one 16-byte vector per lane of a 32-vector step
// of a bf16 row, or 16 channels per lane of a 512-channel step of an FP8 row
// (the quantisation of the separate FP8 dispatch kernel, shared through
// fp8_quant.cuh), at most kLdMaxItems per warp.
//
// The wait is on barrier_words[kDoneWord], a counter that is never reset.  Every CTA
// arrives once on entry and every layout CTA once more when its chunk is
// written; CTA 0's entry adds kBarrierWindow - (G - 1) - nc, so one launch
// moves the counter by exactly one window, every entry arrival learns the
// launch's window from the old value it returns, and the layout is complete
// when the counter reaches the window's end.  As with the layout's own
// barrier, nothing depends on host state, so a CUDA graph may replay the
// launch.  The waits are bounded (%globaltimer and a poll budget); one that
// gives up records the epoch in the handle's timeout word and its CTA stores
// nothing.  Every arrival is unconditional, so the counter stays on its
// window grid whatever happens.

constexpr int kLdMaxItems = 4;
constexpr int kLdItemsPerWarp = 2;   // preferred items per warp when the grid fits
constexpr unsigned kDonePollNs = 256;

__device__ __forceinline__ unsigned atom_add_release_u32(unsigned *ptr, unsigned v)
{
    unsigned old;
    asm volatile("atom.release.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

// SCALE: SEP_SCALE_NONE for the bf16 payload, else the FP8 scale format.
template <typename IdxT, int SCALE>
__global__ void __launch_bounds__(kFusedThreads) layout_dispatch_kernel(LayoutParams p, DispatchParams d)
{
    extern __shared__ __align__(16) int32_t sm[];
    __shared__ int s_flag;
    __shared__ int s_part[kWarps];
    __shared__ unsigned s_base;
    // no early griddepcontrol.launch_dependents: the next kernel starts when this
    // one ends (measured: an early trigger cost the decode step 2 us)
    const int c = blockIdx.x, G = gridDim.x, nc = p.num_wchunks;
    unsigned *done = p.barrier_words + kDoneWord;
    if (threadIdx.x == 0) {
        const unsigned add = c == 0 ? kBarrierWindow - (unsigned)(G - 1) - (unsigned)nc : 1u;
        s_base = atom_add_release_u32(done, add) & ~(kBarrierWindow - 1);
    }
    if (c < nc) {
        layout_chunk<IdxT>(p, c, nc, sm, s_flag, s_part);
        __syncthreads();                                 // every thread's layout writes precede the arrival
        if (threadIdx.x == 0) {
            __threadfence();
            atom_add_release_u32(done, 1u);
        }
        return;
    }

    constexpr bool FP8 = SCALE != SEP_SCALE_NONE;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = d.H, V = H / 8, G8 = H / 128;
    const int per_row = FP8 ? (H + 511) / 512 : (V + 31) / 32;
    const int64_t items = d.T * per_row;
    const int64_t nw = (int64_t)(G - nc) * kWarps;
    const int64_t gw = (int64_t)(c - nc) * kWarps + warp;
    uint4 val[kLdMaxItems];
    float sf[kLdMaxItems];
    int ex[kLdMaxItems];
#pragma unroll
    for (int m = 0; m < kLdMaxItems; ++m) {
        const int64_t it = gw + m * nw;
        val[m] = make_uint4(0u, 0u, 0u, 0u);
        sf[m] = 1.f;
        ex[m] = 0;
        if (it < items) {                                // warp-uniform
            const int64_t t = it / per_row;
            const int st = (int)(it - t * per_row);
            if (!FP8) {
                const int v = st * 32 + lane;
                if (v < V)
                    val[m] = ld_nc_v4(static_cast<const uint4 *>(d.x) + t * V + v);
            } else {
                const int c0 = st * 512 + lane * 16;
                float f[16];
                if (c0 < H) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(d.x) +
                                                                       t * H + c0);
                    bf16x8_to_f32(ld_nc_v4(src), f);
                    bf16x8_to_f32(ld_nc_v4(src + 1), f + 8);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        f[q] = 0.f;
                }
                val[m] = quantize_lane16<FP8 ? SCALE : SEP_SCALE_F32>(f, sf[m], ex[m]);
            }
        }
    }

    // wait for every layout CTA (bounded)
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned target = s_base + kBarrierWindow;
        bool ok = false;
        const uint64_t t0 = global_ns();
        for (uint32_t n = 0; n < (1u << 22); ++n) {
            if ((int)(ld_acquire_u32(done) - target) >= 0) {
                ok = true;
                break;
            }
            if (global_ns() - t0 > 200000000ull)
                break;
            __nanosleep(kDonePollNs);
        }
        if (!ok)
            atomicMax(p.timeout_epoch, p.epoch);
        s_flag = ok ? 1 : 0;
    }
    __syncthreads();
    if (!s_flag)
        return;

#pragma unroll
    for (int m = 0; m < kLdMaxItems; ++m) {
        const int64_t it = gw + m * nw;
        if (it >= items)
            break;                                       // warp-uniform
        const int64_t t = it / per_row;
        const int st = (int)(it - t * per_row);
        const int my_row = lane < d.k ? __ldcg(d.src_pool_row + t * d.k + lane) : -1;
        for (int j = 0; j < d.k; ++j) {
            const int row = __shfl_sync(kFullMask, my_row, j);
            if (row < 0)
                continue;                                // warp-uniform
            if (!FP8) {
                const int v = st * 32 + lane;
                if (v < V)
                    static_cast<uint4 *>(d.recv)[(int64_t)row * V + v] = val[m];
            } else {
                const int c0 = st * 512 + lane * 16;
                if (c0 < H) {
                    *reinterpret_cast<uint4 *>(static_cast<uint8_t *>(d.recv) + (int64_t)row * H + c0) = val[m];
                    if ((lane & 7) == 0) {
                        if (SCALE == SEP_SCALE_UE8M0)
                            static_cast<uint8_t *>(d.recv_scales)[(int64_t)row * G8 + c0 / 128] =
                                (uint8_t)(ex[m] + 127);
                        else
                            static_cast<float *>(d.recv_scales)[(int64_t)row * G8 + c0 / 128] = sf[m];
                    }
                }
            }
        }
    }
}

// Resident CTAs per SM of a layout kernel at a dynamic shared-memory size,
// queried once per (device, kernel, threads, size): the launch decisions below
// are taken on every layout, and the query otherwise costs host time on each.
// 0 when the query fails (the caller then takes the launch that needs no
// residency).
int layout_blocks_per_sm(int dev, const void *kernel, int threads, size_t smem)
{
    struct Entry {
        int dev;
        const void *kernel;
        int threads;
        size_t smem;
        int blocks;
    };
    static Entry cache[64];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].kernel == kernel && cache[i].threads == threads && cache[i].smem == smem)
            return cache[i].blocks;
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, smem) != cudaSuccess) {
        (void)cudaGetLastError();
        b = 0;
    }
    if (used < 64)
        cache[used++] = Entry{dev, kernel, threads, smem, b};
    return b;
}

template <typename IdxT, int SCALE>
cudaError_t try_layout_dispatch_t(const LayoutParams &p, const DispatchParams &d, cudaStream_t s, bool *launched)
{
    using K = void (*)(LayoutParams, DispatchParams);
    const K kernel = layout_dispatch_kernel<IdxT, SCALE>;
    static std::atomic<bool> attr_set[64] = {};
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
        if (e != cudaSuccess)
            return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const size_t smem = layout_smem_bytes(p);
    sms = device_sm_count();
    per_sm = layout_blocks_per_sm(dev, reinterpret_cast<const void *>(kernel), kFusedThreads, smem);
    if (per_sm < 1)
        return cudaSuccess;                              // not fused: the caller launches the two kernels
    const int per_row = SCALE != SEP_SCALE_NONE ? (d.H + 511) / 512 : (d.H / 8 + 31) / 32;
    const int64_t items = d.T * per_row;
    const int64_t resident = (int64_t)per_sm * sms;
    const int nc = p.num_wchunks;
    // two items per warp when that fits, so more warps have stores in flight
    int64_t ctas = (items + kLdItemsPerWarp * kWarps - 1) / (kLdItemsPerWarp * kWarps);
    if (nc + ctas > resident)
        ctas = (items + kLdMaxItems * kWarps - 1) / (kLdMaxItems * kWarps);
    if (ctas < 1 || nc + ctas > resident || 2 * nc + ctas >= (int64_t)kBarrierWindow)
        return cudaSuccess;
    LayoutParams lp = p;
    DispatchParams dp = d;
    void *args[] = {&lp, &dp};
    count_launch();
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kernel), dim3((unsigned)(nc + ctas)),
                                                      dim3(kFusedThreads), args, smem, s);
    if (e == cudaSuccess)
        *launched = true;
    return e;
}

template <typename IdxT>
cudaError_t try_layout_dispatch_idx(const LayoutParams &p, const DispatchParams &d, int payload, cudaStream_t s,
                                    bool *launched)
{
    if (payload == SEP_PAYLOAD_BF16)
        return try_layout_dispatch_t<IdxT, SEP_SCALE_NONE>(p, d, s, launched);
    switch (d.scale) {
    case SEP_SCALE_F32:
        return try_layout_dispatch_t<IdxT, SEP_SCALE_F32>(p, d, s, launched);
    case SEP_SCALE_UE8M0:
        return try_layout_dispatch_t<IdxT, SEP_SCALE_UE8M0>(p, d, s, launched);
    default:
        return try_layout_dispatch_t<IdxT, SEP_SCALE_F32_POW2>(p, d, s, launched);
    }
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p, cudaStream_t s)
{
    if (p.Na >= kNarrowMinNa && p.Na <= kNarrowMaxNa && p.E <= 1024) {
        // one chunk per 32 * kNarrowWarps assignments, one cooperative launch, one grid barrier
        LayoutParams q = p;
        q.rounds = 1;
        q.num_wchunks = (int)((p.Na + 32LL * kNarrowWarps - 1) / (32LL * kNarrowWarps));
        const size_t smem = layout_smem_bytes(q, kNarrowWarps);
        static std::atomic<bool> narrow_attr[64] = {};
        int dev = 0, sms = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return cudaErrorInvalidDevice;
        if (!narrow_attr[dev].load(std::memory_order_acquire)) {
            const cudaError_t e = cudaFuncSetAttribute(layout_fused_kernel<IdxT, kNarrowWarps>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
            if (e != cudaSuccess)
                return e;
            narrow_attr[dev].store(true, std::memory_order_release);
        }
        sms = device_sm_count();
        per_sm = layout_blocks_per_sm(dev, reinterpret_cast<const void *>(layout_fused_kernel<IdxT, kNarrowWarps>),
                                      kNarrowWarps * 32, smem);
        if (q.num_wchunks <= p.num_wchunks * 64 && q.num_wchunks < (int)kBarrierWindow &&
            q.num_wchunks <= per_sm * sms) {
            void *args[] = {&q};
            count_launch();
            return cudaLaunchCooperativeKernel(
                reinterpret_cast<const void *>(layout_fused_kernel<IdxT, kNarrowWarps>), dim3(q.num_wchunks),
                dim3(kNarrowWarps * 32), args, smem, s);
        }
    }
    const int chunks = p.num_wchunks;
    const size_t smem_count = (size_t)kWarps * p.E * sizeof(int32_t);
    const size_t smem_fused = layout_smem_bytes(p);
    if (chunks > 0) {
        // single launch when every CTA can be resident at once
        // function attributes are per device; setting one twice (two threads) is harmless
        static std::atomic<bool> attr_set[64] = {};
        int dev = 0, sms = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return cudaErrorInvalidDevice;
        if (!attr_set[dev].load(std::memory_order_acquire)) {
            const cudaError_t e = cudaFuncSetAttribute(layout_fused_kernel<IdxT>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, 128 * 1024);
            if (e != cudaSuccess)
                return e;
            attr_set[dev].store(true, std::memory_order_release);
        }
        if (chunks == 1)                                 // one CTA: no grid barrier, so an ordinary dependent launch
            return launch_kernel(layout_fused_kernel<IdxT>, dim3(1), dim3(kFusedThreads), smem_fused, s, p);
        sms = device_sm_count();
        per_sm = layout_blocks_per_sm(dev, reinterpret_cast<const void *>(layout_fused_kernel<IdxT>), kFusedThreads,
                                      smem_fused);
        if (chunks <= per_sm * sms && chunks < (int)kBarrierWindow) {
            LayoutParams q = p;
            void *args[] = {&q};
            count_launch();
            return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(layout_fused_kernel<IdxT>),
                                               dim3(chunks), dim3(kFusedThreads), args, smem_fused, s);
        }
        count_launch();
        layout_count_kernel<IdxT><<<chunks, kWarps * 32, smem_count, s>>>(p);
    }
    const size_t smem_assign = smem_count + (size_t)p.R * sizeof(int32_t);
    count_launch();
    layout_scan_kernel<<<1, kScanThreads, 0, s>>>(p);
    const int ablocks = max(chunks, min(p.E, 64));
    count_launch();
    layout_assign_kernel<IdxT><<<ablocks, kWarps * 32, smem_assign, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int layout_rounds_for(int64_t Na)
{
    // small routings: one CTA chunk, which needs neither the chunk table nor the
    // grid barrier (measured: 256 assignments, 17.6 -> 15.4 us per step; at
    // 2048 assignments and 256 experts one CTA is slower than eight)
    if (Na <= kSingleCtaMaxNa)
        return (int)(Na > 0 ? (Na + 32LL * kWarps - 1) / (32LL * kWarps) : 1);
    // at most 128 CTA chunks of 8 warps; 1..64 rounds of 32 assignments per warp
    const int64_t per_round = 32LL * kWarps * 128;
    int64_t r = (Na + per_round - 1) / per_round;
    if (r < 1)
        r = 1;
    if (r > 64)
        r = 64;
    return (int)r;
}

int64_t layout_wchunks_for(int64_t Na, int rounds)
{
    const int64_t per_chunk = 32LL * kWarps * rounds;
    return (Na + per_chunk - 1) / per_chunk;
}

int64_t layout_wchunk_capacity(int64_t Na_cap)
{
    // below 64 rounds the chunk count stays at or below 128; at 64 it grows with Na
    const int64_t big = (Na_cap + 32LL * kWarps * 64 - 1) / (32LL * kWarps * 64);
    return big > 128 ? big : 128;
}

cudaError_t launch_layout(const LayoutParams &p, int idx_bytes, cudaStream_t s)
{
    return idx_bytes == 8 ? launch_layout_t<long long>(p, s) : launch_layout_t<int>(p, s);
}

cudaError_t try_layout_dispatch(const LayoutParams &p, int idx_bytes, const DispatchParams &d, int payload,
                                cudaStream_t s, bool *launched)
{
    *launched = false;
    if (p.T <= 0 || p.num_wchunks < 1 || d.tile_ready != nullptr)
        return cudaSuccess;
    return idx_bytes == 8 ? try_layout_dispatch_idx<long long>(p, d, payload, s, launched)
                          : try_layout_dispatch_idx<int>(p, d, payload, s, launched);
}

cudaError_t preload_layout_kernels()
{
    const void *k[] = {reinterpret_cast<const void *>(layout_dispatch_kernel<int, SEP_SCALE_NONE>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<int, SEP_SCALE_F32>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<int, SEP_SCALE_UE8M0>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<int, SEP_SCALE_F32_POW2>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<long long, SEP_SCALE_NONE>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<long long, SEP_SCALE_F32>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<long long, SEP_SCALE_UE8M0>),
                       reinterpret_cast<const void *>(layout_dispatch_kernel<long long, SEP_SCALE_F32_POW2>),
                       reinterpret_cast<const void *>(layout_fused_kernel<int>),
                       reinterpret_cast<const void *>(layout_fused_kernel<long long>),
                       reinterpret_cast<const void *>(layout_fused_kernel<int, kNarrowWarps>),
                       reinterpret_cast<const void *>(layout_fused_kernel<long long, kNarrowWarps>),
                       reinterpret_cast<const void *>(layout_count_kernel<int>),
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
