// Expert parallelism across ranks over peer memory (StreamEP README, "What's
// in the box": intranode dispatch / combine on NVLink; the "DeepEP MoE
// dispatch/combine" blog, "一轮 DeepEP 数据流": each rank sends its tokens to
// the ranks that own their experts, the receiver lays them out by local expert,
// and combine brings the expert outputs back to the source token).
//
// Rank r (of R) holds its own tokens and routing; owner o = rank o holds
// experts [o*E/R, (o+1)*E/R).  Owner o's pool is expert-major and
// BLOCK_M-padded over its own experts; inside expert e the rows are ordered by
// (source rank, token, slot), the stable order the single-GPU layout gives to
// the concatenation of all ranks' tokens in rank order.  So with counts[r][e]
// the valid assignments of rank r to expert e (exchanged between ranks):
//   N_e        = sum_r counts[r][e],  tau_e = ceil(N_e / B)
//   gboff[e]   = sum of tau over owner(e)'s experts before e   (tiles)
//   row(r,t,j) = gboff[e]*B + sum_{r' < r} counts[r'][e] + s
// where s is the assignment's stable index among rank r's assignments to e,
// which the rank's own layout already holds: its local row is
// loff_r[e]*B + s.  The plan is therefore one shift per (rank, expert),
//   delta_r[e] = gboff[e]*B + sum_{r' < r} counts[r'][e] - loff_r[e]*B,
// computed on the host from the exchanged counts (sep_ep_plan).
//
// The dispatch writes each token row straight into the owner's pool through
// the owner's pointer (a peer pointer on another GPU: stores over NVLink;
// bf16 rows without publication go as untiled bulk stores from shared
// memory, everything else from registers; no tensor map, no multicast)
// together with the owner's receive map (token, rank, slot); the owner marks
// its own padding rows.
//
// The plan can also be computed on the GPU from the exchanged counts
// (ep_plan_kernel), so a step needs no copy to the host.  With publication
// (StreamEP README, "Streaming dispatch in one paragraph": the receiver counts
// arrivals per tile and release-stores dispatch_seq at system scope once the
// tile is complete, so the owner starts on a tile as soon as it is whole) a
// warp owns whole rows; after its stores it fences at system scope, and lane j
// adds one arrival to its row's tile in the owner's memory (atom.add.acq_rel
// .sys); the arrival that reaches the tile's valid-row count (from N_e and the
// expert's first tile, both from the plan) release-stores seq into the
// owner's tile_ready (st.release.sys).  A warp owns whole rows, so a tile is
// complete after one arrival per valid row.  The owner's consumer acquires at
// system scope and zeroes each tile's counter after copying it.  The combine
// gathers each token's k rows from the owners' expert-output pools the same
// way (peer loads) and reduces them exactly as the single-GPU combine does.
#include <cuda_bf16.h>

#include "fp8_quant.cuh"
#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 4;
constexpr int kRowBatch = 4;
constexpr int kKMax = 8;             // combine: row pointers and weights held in registers

__device__ __forceinline__ uint4 ld_stream(const uint4 *ptr)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr));
    return v;
}

// Global row of assignment (t, j) of this rank in its owner's pool, and the
// owner; -1 for a masked assignment or (with *err set) a row outside the
// owner's pool or an owner outside the group.
template <typename P>
__device__ __forceinline__ int64_t owner_row(const P &p, int64_t a, int *owner)
{
    const int local = __ldg(p.src_pool_row + a);
    if (local < 0)
        return -1;
    const int e = __ldg(p.tile_expert + local / p.B);
    const int o = e / p.E_loc;
    const int64_t row = (int64_t)local + __ldg(p.delta + e);
    if (o >= p.R || row < 0 || row >= p.pool_rows[o]) {
        atomicExch(p.error, 1u);
        return -1;
    }
    *owner = o;
    return row;
}

__device__ __forceinline__ unsigned atom_add_acq_rel_sys(unsigned *ptr, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.sys.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(ptr), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void st_release_sys(unsigned *ptr, unsigned v)
{
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}

// After the warp's stores of token t's rows (whole rows: one warp per token):
// one arrival per row on its owner tile; the arrival that completes the tile
// publishes it.  (Rows cut into several warps' segments would need one
// system-scope fence per segment: measured slower, 24.4 against 19.2 us for a
// 1024-token rank at H = 3072.)
__device__ __forceinline__ void ep_publish_rows(const EpDispatchParams &p, int64_t a, int64_t my_row, int my_owner,
                                                int lane)
{
    __threadfence_system();
    __syncwarp();
    if (lane < p.k && my_row >= 0) {
        const int local = __ldg(p.src_pool_row + a);
        const int e = __ldg(p.tile_expert + local / p.B);
        const int tile = (int)(my_row / p.B);
        const int left = __ldg(p.expert_rows + e) - (tile - __ldg(p.expert_tile_offset + e)) * p.B;
        const unsigned need = (unsigned)(left < p.B ? left : p.B);
        if (atom_add_acq_rel_sys(p.arrival_count[my_owner] + tile, 1u) + 1u == need)
            st_release_sys(p.tile_ready[my_owner] + tile, p.seq);
    }
}

// bf16 dispatch into the owners' pools: a work item is (token, segment).
// STAGED (no publication): each 2 KB step of x[t] goes through one of two
// shared-memory stages of the warp and lane 0 issues one bulk store
// (cp.async.bulk, no multicast) of the stage per destination row, as the
// single-GPU dispatch does; a stage is rewritten once the bulk group that read
// it two steps earlier has finished reading.  Otherwise the lanes store from
// registers.
constexpr int kStageVecs = 32 * kUnroll;         // one 2 KB step

template <bool STAGED>
__global__ void __launch_bounds__(kWarps * 32) ep_dispatch_kernel(EpDispatchParams p)
{
    __shared__ __align__(128) uint4 s_stage[STAGED ? kWarps : 1][2][STAGED ? kStageVecs : 1];
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int stage = 0;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t t = it / p.segs;
        const int s = (int)(it - t * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        int my_owner = 0;
        const int64_t my_row = lane < p.k ? owner_row(p, t * p.k + lane, &my_owner) : -1;
        uint4 *my_dst = my_row >= 0 ? static_cast<uint4 *>(p.pools[my_owner]) + my_row * V : nullptr;
        if (s == 0 && my_row >= 0) {                     // the owner's receive map, once per assignment
            if (p.recv_token[my_owner])
                p.recv_token[my_owner][my_row] = (int32_t)t;
            if (p.recv_rank[my_owner])
                p.recv_rank[my_owner][my_row] = p.rank;
            if (p.recv_slot[my_owner])
                p.recv_slot[my_owner][my_row] = lane;
        }
        const uint4 *src = static_cast<const uint4 *>(p.x) + t * V;
        for (int v0 = v_begin; v0 < v_end; v0 += 32 * kUnroll) {
            uint4 buf[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * 32 + lane;
                buf[u] = v < v_end ? ld_stream(src + v) : make_uint4(0, 0, 0, 0);
            }
            if constexpr (STAGED) {
                const int n = min(kStageVecs, v_end - v0);
                if (lane == 0)                               // the stage's previous bulk reads are done
                    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                __syncwarp();
                uint4 *st = s_stage[warp][stage];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u)
                    st[u * 32 + lane] = buf[u];
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                const uint32_t saddr = static_cast<uint32_t>(__cvta_generic_to_shared(st));
                for (int j = 0; j < p.k; ++j) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_dst), j));
                    if (dst != nullptr && lane == 0)
                        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                                     ::"l"(dst + v0), "r"(saddr), "r"(n * 16) : "memory");
                }
                if (lane == 0)
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                stage ^= 1;
            } else {
                for (int j = 0; j < p.k; ++j) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_dst), j));
                    if (dst == nullptr)
                        continue;                        // warp-uniform
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < v_end)
                            dst[v] = buf[u];
                    }
                }
            }
        }
        if (!STAGED && p.tile_ready[0] != nullptr)       // publication
            ep_publish_rows(p, t * p.k + lane, my_row, my_owner, lane);
    }
    if (STAGED && lane == 0)
        asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// FP8 dispatch into the owners' pools: a work item is (token, segment of
// 512-channel iterations); each token is quantised once (the single-GPU
// kernel's arithmetic) and its codes and scales stored to the k owners' rows.
// Rows split over up to 7 warps: unlike the single-GPU kernel, every item
// resolves its rows' owners through three dependent loads, and splitting
// over up to 14 warps with 6 CTAs per SM measured slower here (8 emulated
// prefill_skew ranks on their own streams: dispatches 221.6 against 212.0 us).
template <int SCALE>
__global__ void __launch_bounds__(kWarps * 32) ep_dispatch_fp8_kernel(EpDispatchParams p)
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
        int my_owner = 0;
        const int64_t my_row = lane < p.k ? owner_row(p, t * p.k + lane, &my_owner) : -1;
        uint8_t *my_codes = my_row >= 0 ? static_cast<uint8_t *>(p.pools[my_owner]) + my_row * H : nullptr;
        uint8_t *my_scales = my_row >= 0 ? static_cast<uint8_t *>(p.scales[my_owner]) +
                                               my_row * G * (SCALE == SEP_SCALE_UE8M0 ? 1 : 4)
                                         : nullptr;
        if (s == 0 && my_row >= 0) {                     // the owner's receive map, once per assignment
            if (p.recv_token[my_owner])
                p.recv_token[my_owner][my_row] = (int32_t)t;
            if (p.recv_rank[my_owner])
                p.recv_rank[my_owner][my_row] = p.rank;
            if (p.recv_slot[my_owner])
                p.recv_slot[my_owner][my_row] = lane;
        }
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
                uint8_t *dst = reinterpret_cast<uint8_t *>(
                    __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_codes), j));
                uint8_t *sc = reinterpret_cast<uint8_t *>(
                    __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_scales), j));
                if (dst == nullptr)
                    continue;                            // warp-uniform
                if (active) {
                    *reinterpret_cast<uint4 *>(dst + c0) = codes;
                    if ((lane & 7) == 0) {
                        if (SCALE == SEP_SCALE_UE8M0)
                            sc[g] = (uint8_t)(expo + 127);
                        else
                            reinterpret_cast<float *>(sc)[g] = scale_f;
                    }
                }
            }
        }
        if (p.tile_ready[0] != nullptr)                  // publication
            ep_publish_rows(p, t * p.k + lane, my_row, my_owner, lane);
    }
}

// The plan on the GPU: one CTA, thread e computes expert e's totals (as the
// host sep_ep_plan does: N_e, the rows of earlier ranks, this rank's own
// local block offset and the owner-local global block offset), with two
// block scans over experts (tiles of N_e, tiles of this rank's own counts).
constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long *s_warp, long long *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(kFullMask, incl, o);
        if (lane >= o)
            incl += n;
    }
    if (lane == 31)
        s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const long long w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0;
        long long wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long n = __shfl_up_sync(kFullMask, wi, o);
            if (lane >= o)
                wi += n;
        }
        s_warp[lane] = wi - w;
        if (lane == 31)
            s_warp[32] = wi;
    }
    __syncthreads();
    const long long ex = s_warp[warp] + incl - v;
    *total = s_warp[32];
    __syncthreads();                                     // s_warp is reused by the next scan
    return ex;
}

__global__ void __launch_bounds__(kPlanThreads) ep_plan_kernel(EpPlanParams p)
{
    __shared__ long long s_warp[33];
    __shared__ long long s_gtile[kPlanThreads + 1];      // exclusive scan of tau over all experts
    const int e = threadIdx.x;
    const int E = p.E, R = p.R, B = p.B, El = E / R;
    long long N = 0, before = 0, own = 0;
    bool bad = false;
    if (e < E) {
        for (int r = 0; r < R; ++r) {
            const long long c = p.all_counts[(int64_t)r * E + e];
            bad |= c < 0;
            if (r < p.rank)
                before += c;
            N += c;
        }
        own = p.all_counts[(int64_t)p.rank * E + e];
    }
    const long long tau = e < E && N > 0 ? (N + B - 1) / B : 0;
    const long long own_tau = e < E && own > 0 ? (own + B - 1) / B : 0;
    long long total;
    const long long gex = block_exclusive_scan(tau, s_warp, &total);
    s_gtile[e] = gex;
    if (e == 0)
        s_gtile[kPlanThreads] = total;
    const long long loff = block_exclusive_scan(own_tau, s_warp, &total);
    __syncthreads();
    if (e < E) {
        const int o = e / El;
        const long long gboff = gex - s_gtile[o * El];  // tiles before e inside its owner's pool
        const long long d = gboff * B + before - loff * B;
        if (bad || N > INT32_MAX || d > INT32_MAX || d < INT32_MIN || (gboff + tau) * B > INT32_MAX)
            atomicExch(p.error, 1u);
        p.delta[e] = (int32_t)d;
        if (p.expert_rows)
            p.expert_rows[e] = (int32_t)N;
        if (p.expert_tile_offset)
            p.expert_tile_offset[e] = (int32_t)gboff;
        if (o == p.rank) {
            if (p.owner_block_offset) {
                p.owner_block_offset[e % El] = (int32_t)gboff;
                if (e % El == El - 1)
                    p.owner_block_offset[El] = (int32_t)(gboff + tau);
            }
            if (p.owner_expert_counts)
                p.owner_expert_counts[e % El] = (int32_t)N;
        }
    }
    if (p.owner_rows && e < R) {
        const long long end = (e + 1) * El < E ? s_gtile[(e + 1) * El] : s_gtile[kPlanThreads];
        p.owner_rows[e] = (end - s_gtile[e * El]) * B;
    }
}

// Owner side: -1 in the receive map on the padding rows of its pool.
__global__ void __launch_bounds__(256) ep_mark_padding_kernel(EpPaddingParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int64_t n = p.pool_rows;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < n; r += (int64_t)gridDim.x * blockDim.x) {
        const int tile = (int)(r / p.B);
        int lo = 0, hi = p.E_loc;                        // expert e with block_offset[e] <= tile < block_offset[e+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(p.block_offset + mid) <= tile)
                lo = mid;
            else
                hi = mid;
        }
        const int64_t slot = r - (int64_t)__ldg(p.block_offset + lo) * p.B;
        if (slot >= __ldg(p.expert_counts + lo)) {
            if (p.recv_token)
                p.recv_token[r] = -1;
            if (p.recv_rank)
                p.recv_rank[r] = -1;
            if (p.recv_slot)
                p.recv_slot[r] = -1;
        }
    }
}

__device__ __forceinline__ void accumulate_word(float &lo, float &hi, uint32_t word, float w)
{
    lo = __fadd_rn(lo, __fmul_rn(w, __uint_as_float(word << 16)));
    hi = __fadd_rn(hi, __fmul_rn(w, __uint_as_float(word & 0xffff0000u)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

// Combine from the owners' expert outputs: a warp owns (token, segment); the
// k row pointers and weights are broadcast into registers once (k <= 8) or
// per batch of rows; fp32 sums in ascending j, as the single-GPU combine.
// Tokens are visited in descending order, as there: a dispatch that ran just
// before wrote the highest tokens' rows last.
__global__ void __launch_bounds__(kWarps * 32) ep_combine_kernel(EpCombineParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int V = p.H / 8;
    const int64_t items = p.T * p.segs;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t it = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; it < items; it += nwarps) {
        const int64_t q = it / p.segs;
        const int64_t t = p.T - 1 - q;
        const int s = (int)(it - q * p.segs);
        const int v_begin = s * p.seg_len;
        const int v_end = min(V, v_begin + p.seg_len);
        int my_owner = 0;
        const int64_t my_row = lane < p.k ? owner_row(p, t * p.k + lane, &my_owner) : -1;
        const uint4 *my_src = my_row >= 0 ? static_cast<const uint4 *>(p.y_pools[my_owner]) + my_row * V : nullptr;
        const float my_w = lane < p.k ? __ldg(p.w + t * p.k + lane) : 0.f;
        uint4 *out = static_cast<uint4 *>(p.out) + t * V;
        if (p.k <= kKMax) {
            const uint4 *srcs[kKMax];
            float ws[kKMax];
#pragma unroll
            for (int j = 0; j < kKMax; ++j) {
                srcs[j] = reinterpret_cast<const uint4 *>(
                    __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_src), j));
                ws[j] = __shfl_sync(kFullMask, my_w, j);
            }
            for (int v = v_begin + lane; v < v_end; v += 32) {
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j0 = 0; j0 < kKMax; j0 += kRowBatch) {
                    uint4 buf[kRowBatch];
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u)
                        buf[u] = srcs[j0 + u] != nullptr ? ld_stream(srcs[j0 + u] + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int u = 0; u < kRowBatch; ++u)
                        if (srcs[j0 + u] != nullptr) {
                            accumulate_word(acc[0], acc[1], buf[u].x, ws[j0 + u]);
                            accumulate_word(acc[2], acc[3], buf[u].y, ws[j0 + u]);
                            accumulate_word(acc[4], acc[5], buf[u].z, ws[j0 + u]);
                            accumulate_word(acc[6], acc[7], buf[u].w, ws[j0 + u]);
                        }
                }
                out[v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
            }
            continue;
        }
        for (int v0 = v_begin; v0 < v_end; v0 += 32) {
            const int v = v0 + lane;
            const bool act = v < v_end;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < p.k; j0 += kRowBatch) {
                uint4 buf[kRowBatch];
                const uint4 *src[kRowBatch];
#pragma unroll
                for (int u = 0; u < kRowBatch; ++u) {
                    const int j = j0 + u;
                    src[u] = reinterpret_cast<const uint4 *>(
                        __shfl_sync(kFullMask, reinterpret_cast<unsigned long long>(my_src), j & 31));
                    if (j >= p.k)
                        src[u] = nullptr;
                    buf[u] = (src[u] != nullptr && act) ? ld_stream(src[u] + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kRowBatch; ++u) {
                    const float w = __shfl_sync(kFullMask, my_w, (j0 + u) & 31);
                    if (src[u] != nullptr) {
                        accumulate_word(acc[0], acc[1], buf[u].x, w);
                        accumulate_word(acc[2], acc[3], buf[u].y, w);
                        accumulate_word(acc[4], acc[5], buf[u].z, w);
                        accumulate_word(acc[6], acc[7], buf[u].w, w);
                    }
                }
            }
            if (act)
                out[v] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        }
    }
}

}  // namespace

cudaError_t launch_ep_plan(const EpPlanParams &p, cudaStream_t s)
{
    return launch_kernel(ep_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, p);
}

cudaError_t launch_ep_dispatch(EpDispatchParams p, cudaStream_t s, int num_sms)
{
    if (p.T == 0)
        return cudaSuccess;
    int64_t steps = 1;                                   // 128-vector steps, as the single-GPU dispatch
    split_rows(p.T, ((p.H / 8) + 127) / 128, (int64_t)num_sms * 32, 1 << 20, &p.segs, &steps);
    p.seg_len = (int)(steps * 128);
    if (p.tile_ready[0] != nullptr) {                    // publication counts whole rows: one warp a row
        p.segs = 1;
        p.seg_len = p.H / 8;
    }
    const int64_t items = p.T * p.segs;
    const dim3 grid((int)((items + kWarps - 1) / kWarps)), block(kWarps * 32);
    if (p.tile_ready[0] == nullptr && p.seg_len % kStageVecs == 0)
        return launch_kernel(ep_dispatch_kernel<true>, grid, block, 0, s, p);
    return launch_kernel(ep_dispatch_kernel<false>, grid, block, 0, s, p);
}

cudaError_t launch_ep_dispatch_fp8(EpDispatchParams p, cudaStream_t s, int num_sms)
{
    if (p.T == 0)
        return cudaSuccess;
    int64_t steps = 1;                                   // 512-channel steps, up to 7 warps a row
    split_rows(p.T, (p.H + 511) / 512, (int64_t)num_sms * 32, 7, &p.segs, &steps);
    p.seg_len = (int)steps;
    if (p.tile_ready[0] != nullptr) {                    // publication counts whole rows: one warp a row
        p.segs = 1;
        p.seg_len = (p.H + 511) / 512;
    }
    const dim3 grid((int)((p.T * p.segs + kWarps - 1) / kWarps)), block(kWarps * 32);
    switch (p.scale) {
    case SEP_SCALE_F32:
        return launch_kernel(ep_dispatch_fp8_kernel<SEP_SCALE_F32>, grid, block, 0, s, p);
    case SEP_SCALE_UE8M0:
        return launch_kernel(ep_dispatch_fp8_kernel<SEP_SCALE_UE8M0>, grid, block, 0, s, p);
    default:
        return launch_kernel(ep_dispatch_fp8_kernel<SEP_SCALE_F32_POW2>, grid, block, 0, s, p);
    }
}

cudaError_t launch_ep_mark_padding(const EpPaddingParams &p, cudaStream_t s, int num_sms)
{
    if (p.pool_rows == 0)
        return cudaSuccess;
    int64_t blocks = (p.pool_rows + 255) / 256;
    if (blocks > (int64_t)num_sms * 8)
        blocks = (int64_t)num_sms * 8;
    return launch_kernel(ep_mark_padding_kernel, dim3((int)blocks), dim3(256), 0, s, p);
}

cudaError_t launch_ep_combine(EpCombineParams p, cudaStream_t s, int num_sms)
{
    if (p.T == 0)
        return cudaSuccess;
    int64_t steps = 1;                                   // 32-vector steps, as the single-GPU combine
    split_rows(p.T, ((p.H / 8) + 31) / 32, (int64_t)num_sms * 32, 1, &p.segs, &steps);
    p.seg_len = (int)(steps * 32);
    const int64_t items = p.T * p.segs;
    return launch_kernel(ep_combine_kernel, dim3((int)((items + kWarps - 1) / kWarps)), dim3(kWarps * 32), 0, s, p);
}

cudaError_t preload_ep_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_dispatch_kernel<false>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_dispatch_kernel<true>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_plan_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_mark_padding_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_combine_kernel));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_dispatch_fp8_kernel<SEP_SCALE_F32>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_dispatch_fp8_kernel<SEP_SCALE_UE8M0>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(ep_dispatch_fp8_kernel<SEP_SCALE_F32_POW2>));
    return e;
}

}  // namespace sep
