// Internal declarations of the sep library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sep.h"

namespace sep {

constexpr unsigned kFullMask = 0xffffffffu;

// Work items of the row kernels are (row, segment of the row).  A row of
// `units` warp-steps is split so that there are at least `want_warps` items
// and at least `min_segs` segments per row (never more segments than steps);
// returns the segment count and the steps per segment.
inline void split_rows(int64_t rows, int64_t units, int64_t want_warps, int64_t min_segs, int *segs, int64_t *steps)
{
    int64_t n = rows > 0 ? (want_warps + rows - 1) / rows : 1;
    if (n < min_segs)
        n = min_segs;
    if (n > units)
        n = units;
    if (n < 1)
        n = 1;
    *steps = (units + n - 1) / n;
    *segs = (int)((units + *steps - 1) / *steps);
}

// ----------------------------------------------------------------- layout

// CTA chunks of the assignment stream: CTA c of the count / assign kernels
// owns assignments [c * 256 * rounds, (c + 1) * 256 * rounds), and its warp w
// the contiguous run of 32 * rounds entries starting at w * 32 * rounds.
// Index of the one-launch layout + dispatch's completion counter in
// barrier_words: 128 bytes from the grid barrier's, so that the dispatch CTAs
// polling it do not contend for the barrier's cache line.
constexpr int kDoneWord = 32;

struct LayoutParams {
    const void *topk_idx;
    int64_t T;
    int k, E, R, B;
    int64_t Na;                      // T * k
    int rounds;                      // 32-entry rounds per warp
    int num_wchunks;                 // CTA chunks
    int32_t *wchunk_hist;            // [E][num_wchunks] counts per (expert, chunk)
    int32_t *wchunk_base;            // [E][num_wchunks] exclusive prefix over chunks
    int32_t *expert_counts;          // [E]
    int32_t *owner_counts;           // [R]
    int32_t *owner_token_counts;     // [R]
    uint8_t *is_token_in_rank;       // [T][R] or nullptr
    int32_t *expert_pool_block_offset;  // [E+1]
    int32_t *owner_pool_row_offset;  // [R+1]
    int32_t *tile_expert;            // [NT_cap]
    int32_t *pool_arrival_target;    // [NT_cap]
    uint32_t *pool_arrival_count;    // [NT_cap]
    int32_t *src_pool_row;           // [Na]
    int32_t *pool_recv_token;        // [P_cap]
    int32_t *pool_recv_slot;         // [P_cap]
    int64_t *sizes;                  // [2] = {P, NT}
    uint32_t *bad_epoch;             // last epoch that met an id >= E
    uint32_t *timeout_epoch;         // last epoch whose grid barrier gave up
    uint32_t *barrier_words;         // [64]: [0] the grid barrier's arrival counter, [kDoneWord] the
                                     // one-launch layout + dispatch's completion counter (never reset)
    uint32_t epoch;
};

int layout_rounds_for(int64_t Na);
int64_t layout_wchunks_for(int64_t Na, int rounds);
int64_t layout_wchunk_capacity(int64_t Na_cap);
cudaError_t launch_layout(const LayoutParams &p, int idx_bytes, cudaStream_t s);

// --------------------------------------------------------------- dispatch

// Warps per CTA of a dispatch or combine launched under a CTA budget below
// its default grid: a whole SM's worth, so max_ctas CTAs cover about as many SMs.
constexpr int kBudgetWarps = 32;

struct DispatchParams {
    const void *x;                   // bf16 [T][H]
    int64_t T;
    int H, k, B;
    const int32_t *src_pool_row;     // [T][k]
    void *recv;                      // [rows][H] bf16 or e4m3
    void *recv_scales;               // [rows][H/128] f32 or u8
    int scale;                       // sep_scale
    int segs;                        // warps sharing one token row (set by launch_dispatch)
    int seg_len;                     // per warp: 16-byte vectors (bf16) or 512-channel steps (fp8)
    int max_ctas;                    // > 0: at most this many CTAs (the grid walks the items)
    // streaming publication (tile_ready != nullptr)
    uint32_t *tile_ready;
    uint32_t *pool_arrival_count;
    const int32_t *pool_arrival_target;
    uint32_t seq;
    // a bounded wait that gave up records the layout epoch here
    uint32_t *error_epoch;
    uint32_t epoch;
};

cudaError_t launch_dispatch(DispatchParams p, int payload, cudaStream_t s, int num_sms);

// Layout and dispatch in one cooperative launch when the routing is small
// enough for every dispatch item to sit in registers while the layout runs;
// *launched = false (and nothing enqueued) when it is not.
cudaError_t try_layout_dispatch(const LayoutParams &p, int idx_bytes, const DispatchParams &d, int payload,
                                cudaStream_t s, bool *launched);

// -------------------------------------------------------- backward pair

struct DispatchGradsParams {
    const void *g;                   // bf16 [T][H]: gradient of the combine output
    const float *w;                  // [T][k]
    const void *y;                   // bf16 [rows][H]: expert outputs (grad_w only)
    void *grad_y;                    // bf16 [rows][H]
    float *grad_w;                   // [T][k] or nullptr
    int64_t T;
    int H, k;
    const int32_t *src_pool_row;     // [T][k]
    int segs;                        // warps sharing one token row (no grad_w)
    int seg_len;                     // 16-byte vectors per warp
};

cudaError_t launch_dispatch_grads(DispatchGradsParams p, cudaStream_t s, int num_sms);
cudaError_t preload_backward_kernels();

// ---------------------------------------------------------------- combine

struct CombineParams {
    const void *y;                   // bf16 [rows][H]
    int64_t T;
    int H, k;
    const int32_t *src_pool_row;     // [T][k]
    const float *w;                  // [T][k]
    void *out;                       // bf16 [T][H]
    int segs;                        // warps sharing one token row
    int seg_len;                     // 16-byte vectors per warp
    int max_ctas;                    // > 0: at most this many CTAs (ungated; the grid walks the items)
    uint32_t *error_epoch;           // a bounded wait that gave up records the epoch
    uint32_t epoch;
    // per-token gate (y_done != nullptr): token t is reduced once y_done[t] >= done_seq
    const uint32_t *y_done;          // [T]
    uint32_t done_seq;
    uint64_t timeout_ns;
    uint32_t max_polls;
    uint32_t *status;                // [2]: code, tokens not reduced
};

// num_ctas bounds the persistent grid of the gated variant (y_done != nullptr)
cudaError_t launch_combine(CombineParams p, cudaStream_t s, int num_sms, int num_ctas);

// ---------------------------------------------------- atomic-scatter combine

struct ScatterParams {
    const void *y;                   // bf16 [rows][H]
    int H, k;
    const int32_t *pool_recv_token;  // [rows]
    const int32_t *pool_recv_slot;   // [rows]
    const float *w;                  // [T][k]
    void *out;                       // bf16 [T][H], zero at launch
    const int64_t *num_pool_rows;    // device word: P of the current layout
    int64_t rows_cap;                // rows the grid covers (>= P)
    int segs;                        // warps sharing one pool row
    int seg_len;                     // 16-byte vectors per warp
};

cudaError_t launch_combine_scatter(ScatterParams p, cudaStream_t s, int num_sms);
cudaError_t preload_scatter_kernels();

// ------------------------------------------------- expert parallelism (ranks)

// Ranks of one expert-parallel group (the per-rank pointers travel in the
// kernel parameters, so the host can check them).
constexpr int kEpMaxRanks = 64;

struct EpDispatchParams {
    const void *x;                   // bf16 [T][H], this rank's tokens
    int64_t T;
    int H, k, B, E_loc, R;
    const int32_t *src_pool_row;     // this rank's layout: local row of (t, j)
    const int32_t *tile_expert;      // this rank's layout: expert of each local tile
    const int32_t *delta;            // [E] global-row shift of this rank's rows of expert e
    int rank;
    uint32_t *error;                 // set to 1 when a row falls outside its owner's pool
    int segs, seg_len;               // set by launch_ep_dispatch
    int64_t pool_rows[kEpMaxRanks];  // rows of each owner's pool
    void *pools[kEpMaxRanks];        // owners' pools (bf16 rows; peer pointers on other GPUs)
    int32_t *recv_token[kEpMaxRanks];   // owners' receive maps (entries may be nullptr)
    int32_t *recv_rank[kEpMaxRanks];
    int32_t *recv_slot[kEpMaxRanks];
    // FP8 payload (pools hold e4m3 codes): owners' scale arrays [rows][H/128]
    int scale;                       // sep_scale
    void *scales[kEpMaxRanks];
    // per-tile publication into the owners' memory (tile_ready[0] != nullptr):
    // a row's arrival on its owner tile, and the arrival that completes the
    // tile release-stores seq into the owner's tile_ready (system scope)
    uint32_t *tile_ready[kEpMaxRanks];
    uint32_t *arrival_count[kEpMaxRanks];
    const int32_t *expert_rows;       // [E] N_e over all ranks
    const int32_t *expert_tile_offset;  // [E] first tile of expert e in its owner's pool
    uint32_t seq;
};

// Device-side plan of an expert-parallel step (the host sep_ep_plan, on the GPU).
struct EpPlanParams {
    const int32_t *all_counts;       // [R][E]
    int R, E, B, rank;
    int32_t *delta;                  // [E]
    int64_t *owner_rows;             // [R] or nullptr
    int32_t *owner_block_offset;     // [E/R + 1] or nullptr
    int32_t *owner_expert_counts;    // [E/R] or nullptr
    int32_t *expert_rows;            // [E] or nullptr
    int32_t *expert_tile_offset;     // [E] or nullptr
    uint32_t *error;                 // set to 1 for a negative count or rows beyond 32 bits
};

cudaError_t launch_ep_plan(const EpPlanParams &p, cudaStream_t s);

struct EpPaddingParams {
    int E_loc, B;
    const int32_t *block_offset;     // [E_loc + 1] tiles, this owner's pool
    const int32_t *expert_counts;    // [E_loc] valid rows of each expert
    int64_t pool_rows;
    int32_t *recv_token, *recv_rank, *recv_slot;   // this owner's maps (each may be nullptr)
};

struct EpCombineParams {
    int64_t T;
    int H, k, B, E_loc, R;
    const int32_t *src_pool_row;
    const int32_t *tile_expert;
    const int32_t *delta;
    const float *w;                  // [T][k]
    void *out;                       // bf16 [T][H]
    uint32_t *error;
    int segs, seg_len;               // set by launch_ep_combine
    int64_t pool_rows[kEpMaxRanks];
    const void *y_pools[kEpMaxRanks];   // owners' expert outputs (bf16 rows)
};

cudaError_t launch_ep_dispatch(EpDispatchParams p, cudaStream_t s, int num_sms);
cudaError_t launch_ep_dispatch_fp8(EpDispatchParams p, cudaStream_t s, int num_sms);
cudaError_t launch_ep_mark_padding(const EpPaddingParams &p, cudaStream_t s, int num_sms);
cudaError_t launch_ep_combine(EpCombineParams p, cudaStream_t s, int num_sms);
cudaError_t preload_ep_kernels();

// --------------------------------------------------------------- consumer

struct ConsumeParams {
    const uint8_t *src;
    uint8_t *dst;
    int64_t row_bytes;
    int E, B;
    const int32_t *expert_pool_block_offset;   // [E+1]
    const int32_t *pool_recv_token;
    const uint32_t *tile_ready;
    uint32_t seq;
    uint64_t timeout_ns;
    uint32_t max_polls;
    uint32_t *status;                // [2]: code, tiles not copied
    uint32_t *abort_flag;            // = &status[0]
    // per-token completion stamps (y_done != nullptr)
    uint32_t *y_done;                // [T]
    uint32_t *token_arrivals;        // [T], zero at launch
    const int32_t *src_pool_row;     // [T][k]
    int k;
    uint32_t done_seq;
    // an expert-parallel owner's pool (arrival_count != nullptr): flags are
    // acquired at system scope, the receive map is read through L2, and each
    // consumed tile's arrival counter is zeroed for the next step
    uint32_t *arrival_count;
    int64_t max_tiles;               // tiles the owner's arrays hold; a tile past them is refused
};

cudaError_t launch_consume(const ConsumeParams &p, int num_ctas, cudaStream_t s);

struct GatherParams {
    const uint8_t *slab;
    const int32_t *row_indices;
    uint8_t *dst;
    int64_t rows;
    int64_t row_bytes;
    int indexed;
};

cudaError_t launch_gather(const GatherParams &p, cudaStream_t s, int num_sms);
cudaError_t preload_gather_kernels();

// ------------------------------------------------------------------ utils

// Programmatic dependent launch: dispatch and combine are launched so their
// CTAs may start while the previous kernel of the stream drains, and every
// one of them executes griddepcontrol.wait before its first global memory
// access, which waits for the previous grid to complete and its writes to be
// visible.  Stream-order semantics are unchanged; only launch latency overlaps.
constexpr bool kUsePDL = true;

__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void allow_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Kernels this process has launched through the library (sep_launch_count).
void count_launch();

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args... args)
{
    count_launch();
    if (!kUsePDL) {
        kernel<<<grid, block, smem, s>>>(args...);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Force-load every kernel of a file on the current device.  CUDA loads kernels
// lazily by default, and a load can synchronise the context; a consumer that
// spins on flags written by a later kernel must never meet such a load, so the
// library loads all its kernels up front (on the first handle of a device).
cudaError_t preload_layout_kernels();
cudaError_t preload_dispatch_kernels();
cudaError_t preload_combine_kernels();
cudaError_t preload_consumer_kernels();

int device_sm_count();

// Records msg as the calling thread's last error and returns st.
sep_status set_error(sep_status st, const char *msg);

// Resident CTAs per SM for a kernel at a block size (cached per kernel).
int occupancy_blocks_per_sm(const void *kernel, int threads, size_t smem);

}  // namespace sep

// Library-owned state behind the opaque handle.
struct sep_handle {
    int device;
    int k, E, R, B;
    uint32_t flags_cap;              // flags the storage was sized for
    int64_t T_cap, Na_cap, P_cap, NT_cap, wchunk_cap;
    // current layout
    int64_t T;
    uint32_t flags;
    uint32_t epoch;
    int synced;
    int64_t P, NT;
    // streaming-dispatch guard
    const uint32_t *last_tile_ready;
    uint32_t last_seq;
    int arrivals_used;               // a streaming dispatch ran since the layout reset the counts
    cudaStream_t last_stream;
    // device storage: one block, carved
    void *block;
    int32_t *expert_counts, *owner_counts, *owner_token_counts;
    int32_t *expert_pool_block_offset, *owner_pool_row_offset;
    int32_t *tile_expert, *pool_arrival_target;
    uint32_t *pool_arrival_count;
    int32_t *src_pool_row, *pool_recv_token, *pool_recv_slot;
    int32_t *wchunk_hist, *wchunk_base;
    uint8_t *is_token_in_rank;
    int64_t *sizes;
    uint32_t *bad_epoch;
    uint32_t *timeout_epoch;         // a bounded wait gave up during this epoch
    uint32_t *barrier_words;         // grid-barrier counter of the single-launch layout
    uint32_t *token_arrivals;        // [T_cap] per-token row counters of the stamping consumer
    // CTA budget of the dispatch and combine launches (0: one warp per work item)
    int max_ctas;
    // borrowed-view lease and the consumer events its release recorded
    int leased;
    int n_release;
    cudaEvent_t release_events[8];
    int release_events_made;
    // pinned host mirror of {P, NT, bad_epoch, timeout_epoch}
    int64_t *host_mirror;
};
