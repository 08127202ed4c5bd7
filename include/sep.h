/*
 * sep.h — single-GPU MoE expert-parallel dispatch + combine for B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only; every device pointer is CUDA global
 * memory on the current device, every stream argument is a cudaStream_t passed
 * as void* (NULL = the legacy default stream).  All calls are stream-ordered:
 * they validate their arguments on the host, enqueue kernels and return before
 * the GPU has finished ("DeepEP MoE dispatch/combine" blog, section
 * "EventOverlap": an asynchronous return does not mean the data is ready).
 * Nothing here synchronises the device unless a flag below says so.
 *
 * The operation ("DeepEP MoE dispatch/combine" blog, "一轮 DeepEP 数据流" — one
 * round of data flow):
 *   inputs   x [T, H], topk_idx [T, k], topk_weight [T, k], num_experts E;
 *   dispatch counts assignments per expert, computes the layout and offsets,
 *            and moves the hidden states into recv_x grouped by expert;
 *   combine  restores source token / top-k slot and reduces the
 *            routing-weighted expert outputs back into token order.
 * The receive buffer is the StreamEP pool ("StreamEP" README, "Streaming
 * dispatch in one paragraph"): expert-major and BLOCK_M-padded, expert e's
 * block starting at row expert_pool_block_offset[e] * BLOCK_M; each slot
 * belongs to one expert and one BLOCK_M tile; padding rows have
 * pool_recv_token < 0 and are never read or written.
 *
 * Logical owners ("ranks") are contiguous expert ranges: owner r holds experts
 * [r*E/R, (r+1)*E/R).  The core calls run on one GPU with no communication;
 * the sep_ep_* calls extend dispatch and combine to owners that are separate
 * processes (one per GPU), whose pools are reached through peer pointers.
 *
 * Errors: every entry point returns a sep_status; SEP_OK means the work was
 * enqueued.  On any other status nothing was enqueued (except SEP_ERR_CUDA,
 * where a launch may have failed part way) and sep_last_error() gives a
 * message for the calling thread.  Errors found on the device (an expert id
 * >= E) are reported by sep_handle_sync().  No call aborts, traps or prints.
 */
#ifndef SEP_H
#define SEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SEP_ABI_VERSION 1

/* Exported from the shared library even when it is built with hidden visibility. */
#if defined(__GNUC__) || defined(__clang__)
#define SEP_API __attribute__((visibility("default")))
#else
#define SEP_API
#endif

typedef enum sep_status {
    SEP_OK = 0,
    SEP_ERR_INVALID_ARG = 1,     /* a size, pointer, alignment or mode is not supported */
    SEP_ERR_CAPACITY = 2,        /* an output buffer has fewer rows than the layout needs */
    SEP_ERR_BAD_EXPERT_ID = 3,   /* a topk_idx entry was >= num_experts (device-detected) */
    SEP_ERR_HANDLE_MISMATCH = 4, /* handle used with another routing, shape or epoch */
    SEP_ERR_TIMEOUT = 5,         /* a bounded wait on the device gave up */
    SEP_ERR_CUDA = 6             /* a CUDA runtime call failed */
} sep_status;

/* Payload written into the pool by sep_dispatch. */
typedef enum sep_payload {
    SEP_PAYLOAD_BF16 = 0,        /* rows copied bit for bit, 2 bytes per element */
    SEP_PAYLOAD_FP8_E4M3 = 1     /* rows quantised per 128 channels, 1 byte per element */
} sep_payload;

/* Per-128-channel scale format for SEP_PAYLOAD_FP8_E4M3 ("DeepEP Low-Latency
 * Dispatch and Combine Kernels" article, "FP8 and Quantization Support" and
 * the use_fp8 / round_scale / use_ue8m0 flags of "API Signature and Return
 * Values").  For a group with amax = max |x|:
 *   SEP_SCALE_F32      fp32 s = amax / 448 (IEEE division), s = 1 if amax == 0
 *   SEP_SCALE_UE8M0    byte E* + 127, s = 2^E*, E* the smallest integer with
 *                      448 * 2^E* >= amax (E* = 0 if amax == 0), clamped to [-127, 127]
 *   SEP_SCALE_F32_POW2 the same 2^E* stored as fp32 ("round_scale")
 * and every code is e4m3(x / s), rounded to nearest even, saturated to +-448. */
typedef enum sep_scale {
    SEP_SCALE_NONE = 0,
    SEP_SCALE_F32 = 1,
    SEP_SCALE_UE8M0 = 2,
    SEP_SCALE_F32_POW2 = 3
} sep_scale;

/* sep_layout flags */
#define SEP_LAYOUT_SYNC_COUNTS   0x1u  /* wait for the stream and copy the exact pool size to
                                          the host, so capacity checks use it (the "CPU counts"
                                          of PR #769) instead of the worst case */
#define SEP_LAYOUT_TOKEN_IN_OWNER 0x2u /* also write is_token_in_rank [T, R] and
                                          owner_token_counts [R] */
#define SEP_LAYOUT_ONE_LAUNCH    0x4u  /* sep_layout_dispatch only: run a small routing's
                                          layout and dispatch as one cooperative launch */

/* Opaque routing layout ("EPHandle" in the blog): valid only for the routing
 * that produced it (blog, "EPHandle": the handle is valid only for the routing
 * layout that produced it).  Owns its device metadata. */
typedef struct sep_handle sep_handle;

/* Sizes and device arrays of a handle.  Device pointers belong to the handle
 * and stay valid until the next sep_layout into it or sep_handle_free. */
typedef struct sep_layout_info {
    int64_t num_tokens;          /* T of the current layout */
    int32_t top_k, num_experts, num_owners, block_m;
    int64_t max_tokens;          /* T capacity of the handle */
    int64_t max_pool_rows;       /* worst-case pool rows for max_tokens: any routing fits */
    int64_t max_tiles;           /* max_pool_rows / block_m */
    int64_t num_pool_rows;       /* exact pool rows P (multiple of block_m), -1 unless synced */
    int64_t num_tiles;           /* exact tile count P / block_m, -1 unless synced */
    uint32_t epoch;              /* bumped by every sep_layout into this handle */
    uint32_t flags;              /* flags of the current layout */
    const int32_t *expert_counts;            /* [E]   n_e: valid assignments per expert */
    const int32_t *owner_counts;             /* [R]   L_r = sum of n_e over owner r's experts */
    const int32_t *owner_token_counts;       /* [R]   tokens with >= 1 assignment on owner r
                                                      (SEP_LAYOUT_TOKEN_IN_OWNER, else zeros) */
    const uint8_t *is_token_in_rank;         /* [T, R] or NULL without SEP_LAYOUT_TOKEN_IN_OWNER */
    const int32_t *expert_pool_block_offset; /* [E+1] first tile of expert e; [E] = tiles */
    const int32_t *owner_pool_row_offset;    /* [R+1] first pool row of owner r; [R] = P */
    const int32_t *tile_expert;              /* [max_tiles] expert of each tile (first NT valid) */
    const int32_t *pool_arrival_target;      /* [max_tiles] valid rows in each tile, 1..block_m */
    const uint32_t *pool_arrival_count;      /* [max_tiles] arrivals counted by a streaming dispatch */
    const int32_t *src_pool_row;             /* [T, k] pool row of assignment (t, j), -1 if none */
    const int32_t *pool_recv_token;          /* [max_pool_rows] source token t of a row, -1 = padding */
    const int32_t *pool_recv_slot;           /* [max_pool_rows] source slot j of a row, -1 = padding */
    const int64_t *device_sizes;             /* [2] device copy of {P, NT} for the current layout */
} sep_layout_info;

/*
 * sep_layout — routing layout (the dispatch layout step: count, scan, assign).
 *
 * Counts valid assignments per expert and per owner, scans them into the
 * expert-major BLOCK_M-padded pool (expert_pool_block_offset in tiles,
 * tile_expert, pool_arrival_target = valid rows per tile) and assigns every
 * valid assignment a = t*k + j a pool row.  Rows inside an expert follow
 * ascending a (a stable counting sort), so the result is unique.
 *
 *  topk_idx     device [T, k] row-major, int32 (idx_bytes = 4) or int64 (8).
 *               Entries < 0 mean "no assignment"; entries >= num_experts are
 *               errors: skipped, and reported by sep_handle_sync().
 *  num_tokens   T >= 0 (T = 0 is a valid, empty layout); T * k < 2^31.
 *  top_k        1..32.
 *  num_experts  1..1024; num_owners 1..num_experts dividing it.
 *  block_m      1..1024 rows per tile.
 *  flags        SEP_LAYOUT_* bits.
 *  handle       in/out.  *handle == NULL: a new handle sized for exactly T
 *               tokens is created.  *handle != NULL: it is reused (its epoch
 *               is bumped, its previous layout is invalidated) if top_k,
 *               num_experts, num_owners and block_m match and T fits its
 *               capacity; otherwise SEP_ERR_HANDLE_MISMATCH and nothing changes.
 * The handle's device memory is allocated stream-ordered on `stream` when it is
 * created, and its pinned host words come from a process-wide pool (no
 * cudaMallocHost per handle); later layouts into it allocate nothing.  Creating the first handle
 * on a device also loads all of the library's kernels on it (CUDA otherwise
 * loads kernels lazily, and a load may wait for running kernels, which would
 * stall a dispatch behind a consumer that is waiting for it).
 */
SEP_API sep_status sep_layout(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                      int num_experts, int num_owners, int block_m, uint32_t flags,
                      void *stream, sep_handle **handle);

/* Creates an empty handle with capacity for max_tokens tokens (preallocation,
 * as the blog's "ElasticBuffer" section recommends; flags as for sep_layout:
 * SEP_LAYOUT_TOKEN_IN_OWNER reserves is_token_in_rank). */
SEP_API sep_status sep_handle_create(int64_t max_tokens, int top_k, int num_experts, int num_owners,
                             int block_m, uint32_t flags, void *stream, sep_handle **handle);

/* Fills *info (host struct) for the handle's current layout.  Never blocks. */
SEP_API sep_status sep_handle_info(const sep_handle *handle, sep_layout_info *info);

/* Waits for `stream`, then reads the exact pool size and the device error words
 * of the current layout into the handle (afterwards capacity checks use the
 * exact size).  Returns SEP_ERR_BAD_EXPERT_ID if the layout met an expert id
 * >= num_experts, SEP_ERR_TIMEOUT if the layout's grid barrier or a dispatch
 * or combine of this layout gave up a bounded wait, else SEP_OK. */
SEP_API sep_status sep_handle_sync(sep_handle *handle, void *stream);

/*
 * sep_handle_set_max_ctas — the CTA budget of this handle's dispatch and
 * combine launches (sep_dispatch, bf16 or FP8, with or without tile_ready; the
 * dispatch launch of sep_layout_dispatch; sep_combine; sep_combine_grads).
 * 0 (the default): one 8-warp CTA per eight work items, every SM used.  n > 0
 * below that grid: at most n CTAs of 32 warps (about one per SM), which walk
 * all the work items, so the kernels leave the other SMs to a concurrent
 * kernel (an expert GEMM) at the cost of bandwidth (the DeepEP vibeleaderboard
 * entry, "Why it's ranked here": peak bandwidth with a fraction of the SMs).
 * Results are identical under any budget.  Host-only; takes effect at the next
 * launch; SEP_ERR_INVALID_ARG for n < 0.
 */
SEP_API sep_status sep_handle_set_max_ctas(sep_handle *handle, int max_ctas);

/*
 * sep_dispatch — permute token rows into the pool (optionally FP8-quantised).
 *
 * For every valid assignment (t, j): recv_x[src_pool_row[t, j]] = x[t]
 * (bf16 bits), or the e4m3 codes of x[t] with recv_scales[row] = its per-128
 * channel scales (quantised once per token, written k times).  Weights are not
 * applied (they belong to combine).  Padding rows are not written.
 *
 *  x             device bf16 [T, hidden], 16-byte aligned.
 *  hidden        H: multiple of 8 for bf16, of 128 for FP8; H <= 65536.
 *  payload/scale a sep_payload and a sep_scale (SEP_SCALE_NONE iff bf16).
 *  recv_x        device [recv_capacity_rows, H] of bf16 or e4m3 bytes, 16-byte aligned.
 *  recv_scales   device [recv_capacity_rows, H/128] fp32 (F32, F32_POW2) or
 *                uint8 (UE8M0); NULL for bf16.
 *  recv_capacity_rows  rows of recv_x (and recv_scales); must be >= the exact
 *                pool size after a synced layout, else >= max_pool_rows
 *                (SEP_ERR_CAPACITY otherwise: nothing is silently dropped, as
 *                the blog's "Imbalance" section asks).
 *  tile_ready    NULL, or device uint32 [tile_ready_len].  When given, each tile
 *                is published once all its valid rows are written: the
 *                dispatch counts arrivals in the handle's pool_arrival_count
 *                (reset by sep_layout) and the writer that completes a tile
 *                release-stores dispatch_seq into tile_ready[tile] (StreamEP
 *                README, "Streaming dispatch in one paragraph").  A consumer
 *                on another stream may acquire-load tile_ready[tile] and wait
 *                until it reaches dispatch_seq (see sep_consume_tiles).
 *  tile_ready_len entries of tile_ready; must cover the layout's tiles: the
 *                exact tile count after a synced layout, else the worst case
 *                for the current T (its worst-case pool rows / block_m).
 *                SEP_ERR_CAPACITY otherwise.
 *  dispatch_seq  != 0 when tile_ready is given, and (mod 2^32) greater than the
 *                value used by the previous dispatch of this handle into the
 *                same tile_ready array, so stale flags are never taken as
 *                ready; SEP_ERR_INVALID_ARG otherwise.  tile_ready never needs
 *                a reset.
 */
SEP_API sep_status sep_dispatch(sep_handle *handle, const void *x, int64_t hidden, int payload,
                        int scale, void *recv_x, void *recv_scales,
                        int64_t recv_capacity_rows, uint32_t *tile_ready,
                        int64_t tile_ready_len, uint32_t dispatch_seq, void *stream);

/*
 * sep_layout_dispatch — the layout and the dispatch of one routing in one call.
 *
 * The dispatch of the pages' problem statement takes the router's top-k
 * output and the hidden states together ("DeepEP MoE dispatch/combine" blog,
 * "一轮 DeepEP 数据流": count by destination/expert, compute the layout and
 * offsets, move the hidden states; the low-latency article's
 * low_latency_dispatch takes x and topk_idx in one call).  This call computes
 * exactly what sep_layout followed by sep_dispatch (no tile_ready) computes,
 * into the same handle, with the same arguments and errors, except:
 *  - recv_capacity_rows must cover the worst case for num_tokens (the exact
 *    pool size is known only after the layout), else SEP_ERR_CAPACITY and
 *    nothing changes;
 *  - with SEP_LAYOUT_ONE_LAUNCH, when the routing is small enough (every
 *    dispatch item of x held in registers by the CTAs the GPU can keep
 *    resident beside the layout's), the two run as ONE cooperative launch:
 *    the dispatch CTAs load, and for FP8 quantise, their slices of x while
 *    the layout runs, wait for it (bounded; a wait that gives up is reported
 *    by sep_handle_sync as SEP_ERR_TIMEOUT), then store to the pool rows.
 *    Otherwise, and by default, the layout and dispatch kernels are launched
 *    one after the other, as by the two calls (the dispatch with programmatic
 *    dependent launch, resident while the layout drains).  Measured on one
 *    B200 the one launch is not faster: decode step 27.6 us against 27.0,
 *    graph replay 30.2 against 28.6; tiny 13.5 against 15.3 eager, 16.4
 *    against 15.6 replayed.
 * SEP_LAYOUT_SYNC_COUNTS waits for both, then reads the exact pool size.
 * sep_launch_count tells the two cases apart (one launch or two).
 */
SEP_API sep_status sep_layout_dispatch(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                               int num_experts, int num_owners, int block_m, uint32_t flags,
                               const void *x, int64_t hidden, int payload, int scale, void *recv_x,
                               void *recv_scales, int64_t recv_capacity_rows, void *stream,
                               sep_handle **handle);

/*
 * sep_combine — weighted top-k reduction back into token order.
 *
 * out[t] = bf16( sum over valid j, ascending, of topk_weight[t, j] *
 *                y_pool[src_pool_row[t, j]] ) with fp32 products and sums
 * ("DeepEP MoE dispatch/combine" blog, "Router 权重什么时候应用":
 * y_t = sum_j p_{t,j} o_{t,j}).  Masked assignments contribute nothing; a
 * token with none gets +0.
 *
 *  layout_epoch  the handle's epoch when the caller's routing was laid out;
 *                a different value means the handle now holds another routing
 *                (SEP_ERR_HANDLE_MISMATCH: the blog's "EPHandle" and
 *                integration-contract sections ask to detect this).
 *  y_pool        device bf16 [y_capacity_rows, hidden] in pool layout, 16-byte aligned.
 *  hidden        multiple of 8.
 *  topk_weight   device fp32 [T, k].
 *  out           device bf16 [T, hidden], 16-byte aligned.
 */
SEP_API sep_status sep_combine(const sep_handle *handle, uint32_t layout_epoch, const void *y_pool,
                       int64_t hidden, int64_t y_capacity_rows, const float *topk_weight,
                       void *out, void *stream);

/*
 * sep_consume_tiles — a reference consumer of a streaming dispatch.
 *
 * Stands in for the grouped-GEMM consumer of the StreamEP README ("Streaming
 * dispatch in one paragraph": a consumer spins on the acquire-load of
 * tile_ready[tile] >= dispatch_seq from another stream, then proceeds).
 * Launches num_ctas persistent CTAs (1..1024; keep it well below the SM count
 * so a dispatch launched on another stream can run beside it).  Tiles are
 * visited in the order a token-major dispatch completes them (tile i of every
 * expert before tile i+1).  Each CTA waits for its tile with a bounded spin,
 * then copies the tile's valid rows (pool_recv_token >= 0) from recv_x to the
 * same rows of dst.  A wait gives up after timeout_ns nanoseconds of
 * %globaltimer (or a fixed poll budget); then every CTA stops waiting,
 * status[0] becomes SEP_ERR_TIMEOUT and status[1] counts the tiles not copied.
 *
 *  recv_x, dst   device [capacity_rows, row_bytes]; row_bytes a multiple of 16;
 *                16-byte aligned; capacity_rows as for sep_dispatch's recv_x.
 *  tile_ready    the array given to sep_dispatch, tile_ready_len entries.
 *  status        device uint32 [2]; reset by this call, written by the kernel.
 * Must be stream-ordered after the sep_layout of the handle (e.g. via an event);
 * it is ordered against the dispatch only through tile_ready.  Between this
 * call and the sep_dispatch it waits for, the host must not wait for the
 * device (a device or stream synchronisation, or a copy from pageable host
 * memory): that wait would hold the dispatch back until the consumer's waits
 * time out (SEP_ERR_TIMEOUT; nothing hangs).
 */
SEP_API sep_status sep_consume_tiles(const sep_handle *handle, const void *recv_x, int64_t row_bytes,
                             int64_t capacity_rows, const uint32_t *tile_ready,
                             int64_t tile_ready_len, uint32_t dispatch_seq, void *dst,
                             int num_ctas, uint64_t timeout_ns, uint32_t *status, void *stream);

/*
 * sep_combine_scatter — the combine driven from the pool side with bf16
 * atomic reductions (StreamEP README, "What's in the box": kernel_y's
 * AtomicScatterStore, per-warp coalesced bf16 atomic scatter into the output).
 *
 * Zeroes out, then for every valid pool row r adds bf16(topk_weight[t, j] *
 * y_pool[r]) into out[t] (t = pool_recv_token[r], j = pool_recv_slot[r]) with
 * bf16x2 reductions.  Same arguments and errors as sep_combine; the result is
 * NOT deterministic: the k terms of a token are each rounded to bf16 and added
 * in bf16 in arrival order, so it differs from sep_combine by at most about
 * 2k * 2^-8 * sum_j |w[t, j] * y[row(t, j)]| per element.  Works on an
 * unsynced layout (the pool size is read on the device).
 */
SEP_API sep_status sep_combine_scatter(const sep_handle *handle, uint32_t layout_epoch, const void *y_pool,
                                       int64_t hidden, int64_t y_capacity_rows, const float *topk_weight,
                                       void *out, void *stream);

/*
 * Per-token combine gate (StreamEP README, opening section: y_done_per_token
 * lets the combine start on a token as soon as that token's compute has
 * drained, instead of after the whole compute kernel).  On one GPU the gate is
 * an array y_done [T] in token order: the producer of y_pool release-stores a
 * sequence number into y_done[t] once every valid row of token t is written;
 * the gated combine waits (acquire, bounded) for y_done[t] >= done_seq before
 * it reads token t's rows.  Sequence numbers compare modulo 2^32 (as
 * int32(y_done[t] - done_seq) >= 0); start y_done at 0 and use a new nonzero
 * done_seq for each pass.
 */

/*
 * sep_consume_tiles_stamp — sep_consume_tiles plus per-token completion stamps.
 *
 * The same reference consumer; after a CTA has copied a tile it adds one
 * arrival per valid row to the row's token counter, and the arrival that
 * completes token t (its count of valid assignments) release-stores done_seq
 * into y_done[t].  With dst used as y_pool this stands in for the expert
 * compute that feeds a gated combine (identity experts).  The token counters
 * belong to the handle and are reset on `stream` by this call, so two stamping
 * consumers of one handle must not overlap on the GPU.
 *
 *  y_done      device uint32 [y_done_len >= T], 4-byte aligned.
 *  done_seq    nonzero.
 * Other arguments, ordering rules and errors as sep_consume_tiles.
 */
SEP_API sep_status sep_consume_tiles_stamp(const sep_handle *handle, const void *recv_x, int64_t row_bytes,
                                           int64_t capacity_rows, const uint32_t *tile_ready,
                                           int64_t tile_ready_len, uint32_t dispatch_seq, void *dst,
                                           int num_ctas, uint64_t timeout_ns, uint32_t *status,
                                           uint32_t *y_done, int64_t y_done_len, uint32_t done_seq,
                                           void *stream);

/*
 * sep_combine_gated — sep_combine that waits per token on the gate.
 *
 * Same result as sep_combine for every token whose wait succeeds (a token
 * with no valid assignment is not waited for: it gets +0).  Launches at
 * most num_ctas (1..1024) persistent CTAs, so keep it below the SM count left
 * over by the producer; tokens are visited in ascending order.  A wait gives
 * up after timeout_ns nanoseconds of %globaltimer (0: one second) or a fixed
 * poll budget; then every warp stops waiting, status[0] becomes
 * SEP_ERR_TIMEOUT, status[1] counts the tokens not reduced, and their out rows
 * are left unwritten.
 *
 *  y_done      device uint32 [y_done_len >= T], written by the producer.
 *  status      device uint32 [2]; reset by this call, written by the kernel.
 * Other arguments as sep_combine.  Like sep_consume_tiles, the host must not
 * wait for the device between this call and the work that sets the gate.
 */
SEP_API sep_status sep_combine_gated(const sep_handle *handle, uint32_t layout_epoch, const void *y_pool,
                                     int64_t hidden, int64_t y_capacity_rows, const float *topk_weight,
                                     void *out, const uint32_t *y_done, int64_t y_done_len, uint32_t done_seq,
                                     int num_ctas, uint64_t timeout_ns, uint32_t *status, void *stream);

/*
 * Backward pair (StreamEP README, "What's in the box": dispatch_grads and
 * combine_grads give the backward symmetry of dispatch and combine).
 *
 * sep_dispatch_grads — the backward of sep_combine.  With
 * out[t] = sum_j w[t, j] * y[row(t, j)]:
 *   grad_y[row(t, j)] = bf16( w[t, j] * grad_out[t] )   fp32 product, rounded
 *                                                       to nearest even
 *   grad_w[t, j]      = sum_h grad_out[t, h] * y[row(t, j), h]
 *                       fp32 sums in a fixed order (reproducible run to run);
 *                       0 for a masked assignment.
 *  grad_out     device bf16 [T, hidden], 16-byte aligned.
 *  topk_weight  device fp32 [T, k] (the forward weights).
 *  y_pool       device bf16 [y_capacity_rows, hidden], the forward expert
 *               outputs in pool layout; read only when grad_w != NULL.
 *  grad_y       device bf16 [grad_y_capacity_rows, hidden] in pool layout;
 *               padding rows are not written.
 *  grad_w       device fp32 [T, k], or NULL to skip the weight gradient.
 * Errors as sep_combine.
 */
SEP_API sep_status sep_dispatch_grads(const sep_handle *handle, uint32_t layout_epoch, const void *grad_out,
                                      int64_t hidden, const float *topk_weight, const void *y_pool,
                                      int64_t y_capacity_rows, void *grad_y, int64_t grad_y_capacity_rows,
                                      float *grad_w, void *stream);

/*
 * sep_combine_grads — the backward of sep_dispatch (bf16 payload).
 *   grad_x[t] = bf16( sum over valid j, ascending, of grad_recv[row(t, j)] )
 * in fp32 (sep_combine with every weight 1; exact up to the final rounding
 * order of the definition).  A token with no valid assignment gets +0.
 *  grad_recv  device bf16 [capacity_rows, hidden] in pool layout, 16-byte aligned.
 *  grad_x     device bf16 [T, hidden], 16-byte aligned.
 * Errors as sep_combine.
 */
SEP_API sep_status sep_combine_grads(const sep_handle *handle, uint32_t layout_epoch, const void *grad_recv,
                                     int64_t hidden, int64_t capacity_rows, void *grad_x, void *stream);

/*
 * Borrowed receive (PR #769 "Add opt-in borrowed receive storage for compact
 * BF16 dispatch", "Description"): instead of copying every assigned token row
 * into the pool, the dispatch hands out a view (slab, row_indices) that an
 * indexed consumer reads directly.  On one GPU the slab is x itself and
 * row_indices is the layout's pool_recv_token: pool row r holds
 * slab[row_indices[r]] (row_indices[r] < 0: padding, never read).
 */
typedef struct sep_recv_view {
    const void *slab;              /* device rows the view reads from */
    const int32_t *row_indices;    /* device [num_rows]: slab row of each pool row, -1 = padding */
    int64_t num_rows;              /* pool rows P */
    int64_t row_bytes;             /* bytes per row (multiple of 16) */
    int32_t indexed;               /* 1: pool row r is slab[row_indices[r]]; 0: pool row r is slab[r]
                                      (a pool that was copied; row_indices only marks validity) */
    uint32_t epoch;                /* layout epoch of the handle the view came from */
} sep_recv_view;

/*
 * sep_dispatch_borrow — a dispatch that copies nothing.
 *
 * Fills *view = {x, pool_recv_token, P, 2*hidden, indexed=1, epoch} and puts an
 * exclusive lease on the handle: until sep_view_release, sep_layout,
 * sep_dispatch, sep_dispatch_borrow and sep_combine on this handle are refused
 * (SEP_ERR_HANDLE_MISMATCH) and sep_handle_free leaves it allocated, because
 * they would change or free the row map the consumers are reading.  x must stay
 * valid and unchanged until the release.  Supported, as in the PR, only for a
 * bf16 payload after a synced layout (SEP_LAYOUT_SYNC_COUNTS or
 * sep_handle_sync: the "CPU counts" that give P); everything else is rejected
 * up front with SEP_ERR_INVALID_ARG.  Launches nothing.
 */
SEP_API sep_status sep_dispatch_borrow(sep_handle *handle, const void *x, int64_t hidden, int payload,
                                       sep_recv_view *view);

/*
 * sep_view_release — ends the lease of sep_dispatch_borrow.
 *
 * Records an event on each of the num_streams consumer streams; the handle's
 * next layout, dispatch or combine waits for all of them on its own stream
 * before it touches the row map (the PR's release(*streams): the next
 * communication is ordered after the consumers).  SEP_ERR_INVALID_ARG if the
 * handle has no active view or num_streams is not in 0..8.
 */
SEP_API sep_status sep_view_release(sep_handle *handle, void *const *streams, int num_streams);

/*
 * sep_gather_rows — a reference indexed consumer of a view.
 *
 * dst[r] = (view->indexed ? slab[row_indices[r]] : slab[r]) for every pool row
 * r < num_rows with row_indices[r] >= 0; padding rows of dst are not written.
 * dst: device [dst_rows, row_bytes], 16-byte aligned, dst_rows >= num_rows.
 * It stands in for the gathered-GEMM consumer of the PR; with indexed = 0 it
 * reads a copied pool in place, which gives the copy path's consumer.
 */
SEP_API sep_status sep_gather_rows(const sep_recv_view *view, void *dst, int64_t dst_rows, void *stream);

/*
 * Expert parallelism across ranks over peer memory (StreamEP README, "What's
 * in the box": intranode dispatch / combine over NVLink; "DeepEP MoE
 * dispatch/combine" blog, "一轮 DeepEP 数据流": tokens go to the ranks that
 * own their experts, the receiver groups them by local expert, combine brings
 * the expert outputs back).
 *
 * R ranks (at most 64); rank o owns experts [o*E/R, (o+1)*E/R).  Each rank lays
 * out its own routing with sep_layout(num_owners = R).  Owner o's pool is
 * expert-major and BLOCK_M-padded over its own experts, and inside an expert
 * the rows are ordered by (source rank, token, slot): exactly owner o's segment
 * of the single-GPU layout of all ranks' tokens concatenated in rank order.
 * A pool is any device memory of this or a peer GPU (a peer pointer from CUDA
 * IPC or symmetric memory); rows are written by stores from registers, or
 * (sep_ep_dispatch, which publishes nothing) by untiled bulk stores from
 * shared memory, and read with plain loads: no tensor map, no multicast.
 * Only the one-GPU emulation has run here: bulk stores to a peer's pool are
 * not tested across GPUs.  Between the dispatches of all ranks and the
 * owners' expert compute, and between that and the combines, the caller
 * synchronises the ranks (a barrier or a collective).
 */

/*
 * sep_ep_plan — host-only: the per-rank row shift from every rank's expert
 * counts.  Calls no CUDA function.
 *
 *  all_counts           host int32 [num_ranks, num_experts]: row r is rank r's
 *                       expert_counts (exchanged between ranks, e.g. by an all-gather).
 *  delta                host int32 [num_experts], out: a row of this rank's layout
 *                       at local row L (expert e) goes to row L + delta[e] of its
 *                       owner's pool.
 *  owner_rows           host int64 [num_ranks] or NULL, out: pool rows of each owner.
 *  owner_block_offset   host int32 [E/R + 1] or NULL, out: this rank's pool, tile
 *                       offset of each local expert (for its grouped GEMM).
 *  owner_expert_counts  host int32 [E/R] or NULL, out: valid rows of each local expert.
 * SEP_ERR_INVALID_ARG for a size out of range, a negative count or a pool
 * that would not fit 32-bit rows.
 */
SEP_API sep_status sep_ep_plan(const int32_t *all_counts, int num_ranks, int num_experts, int block_m, int rank,
                               int32_t *delta, int64_t *owner_rows, int32_t *owner_block_offset,
                               int32_t *owner_expert_counts);

/*
 * sep_ep_dispatch — copies this rank's token rows into their owners' pools
 * (bf16), and writes each owner's receive map entry: recv_token = source
 * token, recv_rank = this rank, recv_slot = top-k slot.
 *
 *  handle, layout_epoch  this rank's layout (num_owners = R) and its epoch.
 *  rank                  this rank (0..R-1).
 *  delta                 device int32 [E]: sep_ep_plan's delta for this rank.
 *  pools, pool_rows      host arrays [R]: each owner's pool (device bf16
 *                        [pool_rows[o], hidden], 16-byte aligned) and its rows.
 *  recv_token, recv_rank, recv_slot
 *                        host arrays [R] of device int32 [pool_rows[o]] maps, or
 *                        NULL (an entry may be NULL too).
 *  error                 device uint32: set to 1 when a row falls outside its
 *                        owner's pool (the write is skipped; a wrong delta or a
 *                        short pool is never written past).
 */
SEP_API sep_status sep_ep_dispatch(const sep_handle *handle, uint32_t layout_epoch, const void *x, int64_t hidden,
                                   int rank, const int32_t *delta, void *const *pools, const int64_t *pool_rows,
                                   int32_t *const *recv_token, int32_t *const *recv_rank, int32_t *const *recv_slot,
                                   uint32_t *error, void *stream);

/*
 * sep_ep_dispatch_fp8 — sep_ep_dispatch with the FP8 e4m3 payload: each token
 * is quantised once per 128-channel group exactly as sep_dispatch does
 * (scale = SEP_SCALE_F32, SEP_SCALE_UE8M0 or SEP_SCALE_F32_POW2), and its
 * codes and scales are stored to the owners' rows.
 *
 *  pools    host array [R] of device e4m3 [pool_rows[o], hidden] (16-byte aligned).
 *  scales   host array [R] of device [pool_rows[o], hidden / 128] fp32 or u8.
 *  hidden   a multiple of 128.
 * Other arguments and errors as sep_ep_dispatch.
 */
SEP_API sep_status sep_ep_dispatch_fp8(const sep_handle *handle, uint32_t layout_epoch, const void *x,
                                       int64_t hidden, int rank, int scale, const int32_t *delta,
                                       void *const *pools, void *const *scales, const int64_t *pool_rows,
                                       int32_t *const *recv_token, int32_t *const *recv_rank,
                                       int32_t *const *recv_slot, uint32_t *error, void *stream);

/*
 * sep_ep_mark_padding — owner side: -1 in the receive maps (each may be NULL)
 * on the padding rows of this owner's pool, from sep_ep_plan's
 * owner_block_offset and owner_expert_counts (device copies).  Touches no
 * valid row, so it may run while other ranks dispatch.
 */
SEP_API sep_status sep_ep_mark_padding(int num_local_experts, int block_m, const int32_t *owner_block_offset,
                                       const int32_t *owner_expert_counts, int64_t pool_rows, int32_t *recv_token,
                                       int32_t *recv_rank, int32_t *recv_slot, void *stream);

/*
 * sep_ep_plan_device — sep_ep_plan on the GPU: the same outputs from the same
 * exchanged counts, computed by one kernel on `stream`, so a step needs no
 * copy to the host (the counts can be all-gathered device to device).
 *
 *  all_counts           device int32 [num_ranks, num_experts], as for sep_ep_plan.
 *  delta, owner_rows (int64 [num_ranks]), owner_block_offset, owner_expert_counts:
 *                       device outputs as for sep_ep_plan (the last three may be NULL).
 *  expert_rows          device int32 [num_experts] or NULL, out: N_e, every rank's
 *                       assignments of expert e (the owner's valid rows of e).
 *  expert_tile_offset   device int32 [num_experts] or NULL, out: the first tile of
 *                       expert e in its owner's pool.  With expert_rows, what a
 *                       publishing dispatch needs to know when a tile is complete.
 *  error                device uint32, set to 1 (never cleared) for a negative
 *                       count or a pool beyond 32-bit rows; the outputs are then
 *                       not to be used.
 * num_ranks <= 64 (the expert-parallel kernels' limit), num_experts <= 1024.
 */
SEP_API sep_status sep_ep_plan_device(const int32_t *all_counts, int num_ranks, int num_experts, int block_m,
                                      int rank, int32_t *delta, int64_t *owner_rows, int32_t *owner_block_offset,
                                      int32_t *owner_expert_counts, int32_t *expert_rows,
                                      int32_t *expert_tile_offset, uint32_t *error, void *stream);

/*
 * sep_ep_dispatch_publish — sep_ep_dispatch (payload SEP_PAYLOAD_BF16, scale
 * SEP_SCALE_NONE, scales NULL) or sep_ep_dispatch_fp8 (SEP_PAYLOAD_FP8_E4M3),
 * that also publishes every owner tile as soon as it is complete (StreamEP
 * README, "Streaming dispatch in one paragraph": arrivals counted per tile on
 * the receiver, dispatch_seq release-stored at system scope by the arrival
 * that completes the tile).  A warp writes whole rows; after its stores it
 * fences at system scope and adds one arrival per row to
 * arrival_count[owner][tile] (atom.add.acq_rel.sys); the arrival that reaches
 * the tile's valid rows (from expert_rows and expert_tile_offset of
 * sep_ep_plan_device) stores dispatch_seq into tile_ready[owner][tile]
 * (st.release.sys).  No load with multicast, no TMA: plain peer stores and
 * atomics.
 *
 *  tile_ready, arrival_count  host arrays [R] of device uint32 arrays in the
 *                       owners' memory (peer pointers), each of at least
 *                       ceil(pool_rows[o] / block_m) entries.  Every counter
 *                       must be zero when the group's dispatches start:
 *                       allocate them zeroed; sep_ep_consume_tiles zeroes each
 *                       tile it consumes.
 *  dispatch_seq         nonzero, advancing (mod 2^32) per step of the group.
 * Other arguments and errors as sep_ep_dispatch / sep_ep_dispatch_fp8.
 */
SEP_API sep_status sep_ep_dispatch_publish(const sep_handle *handle, uint32_t layout_epoch, const void *x,
                                           int64_t hidden, int rank, int payload, int scale, const int32_t *delta,
                                           void *const *pools, void *const *scales, const int64_t *pool_rows,
                                           int32_t *const *recv_token, int32_t *const *recv_rank,
                                           int32_t *const *recv_slot, uint32_t *const *tile_ready,
                                           uint32_t *const *arrival_count, const int32_t *expert_rows,
                                           const int32_t *expert_tile_offset, uint32_t dispatch_seq,
                                           uint32_t *error, void *stream);

/*
 * sep_ep_consume_tiles — owner side: the reference consumer of a publishing
 * dispatch (a stand-in for the owner's expert compute).  Persistent CTAs walk
 * the owner's tiles (from owner_block_offset of sep_ep_plan_device, device
 * [E_loc + 1]); thread 0 acquire-loads tile_ready[tile] at system scope
 * until it reaches dispatch_seq, bounded by timeout_ns (0: 1 s) and a poll
 * budget; the CTA then copies the tile's valid rows (recv_token >= 0, read
 * through L2) from pool to dst and zeroes arrival_count[tile] for the next
 * step.  status (device uint32 [2]) = {SEP_OK or SEP_ERR_TIMEOUT, tiles not
 * copied}; a tile beyond pool_rows / block_m (a plan larger than the owner's
 * arrays) is not touched and gives SEP_ERR_CAPACITY.  After a timeout the
 * group must zero the arrival counters before its next step.  Launch it after
 * the dispatches it waits for are enqueued on their GPUs, or before them on
 * another GPU; never wait on a dispatch that another process launches on the
 * same GPU (nothing guarantees the two kernels run at the same time).
 */
SEP_API sep_status sep_ep_consume_tiles(int num_local_experts, int block_m, const int32_t *owner_block_offset,
                                        const void *pool, const int32_t *recv_token, int64_t row_bytes,
                                        int64_t pool_rows, const uint32_t *tile_ready, uint32_t *arrival_count,
                                        uint32_t dispatch_seq, void *dst, int num_ctas, uint64_t timeout_ns,
                                        uint32_t *status, void *stream);

/*
 * sep_ep_combine — out[t] = bf16( sum over valid j, ascending, of
 * topk_weight[t, j] * y_pools[owner][row(t, j)] ) with fp32 products and sums:
 * sep_combine over the owners' expert-output pools (host array [R] of device
 * bf16 [pool_rows[o], hidden], 16-byte aligned).  Other arguments as
 * sep_ep_dispatch.
 */
SEP_API sep_status sep_ep_combine(const sep_handle *handle, uint32_t layout_epoch, const void *const *y_pools,
                                  const int64_t *pool_rows, int64_t hidden, const int32_t *delta,
                                  const float *topk_weight, void *out, uint32_t *error, void *stream);

/*
 * Buffers shared across the processes of an expert-parallel group (CUDA IPC;
 * plain device memory mapped into the peers, no multicast object).  No
 * counterpart on the pages: they are the plumbing a multi-process group needs
 * to hand each other pool pointers.
 *
 * sep_ep_buffer_alloc   cudaMalloc of `bytes` on the current device; writes the
 *                       SEP_IPC_HANDLE_BYTES-byte handle other processes open.
 * sep_ep_buffer_open    maps a handle from another process (on this device or a
 *                       peer) and returns its device pointer.  A process cannot
 *                       open its own handle: it uses its own pointer.
 * sep_ep_buffer_close   opened = 1: unmaps a buffer from sep_ep_buffer_open;
 *                       opened = 0: frees one from sep_ep_buffer_alloc (after
 *                       every peer has closed it).  Both synchronise the device.
 */
#define SEP_IPC_HANDLE_BYTES 64
SEP_API sep_status sep_ep_buffer_alloc(int64_t bytes, void **ptr, void *ipc_handle);
SEP_API sep_status sep_ep_buffer_open(const void *ipc_handle, void **ptr);
SEP_API sep_status sep_ep_buffer_close(void *ptr, int opened);

/* Frees the handle.  Its device memory is released stream-ordered on the
 * stream of the last call that used it, after the streams the last
 * sep_view_release named; the caller must have ordered every other stream
 * that used the handle before that point.  The call does not wait for the
 * device: its pinned host words go back to a process-wide pool (no
 * cudaFreeHost), so a free between a consumer's launch and the dispatch it
 * waits for does not stall.  If the wait on the view's consumers cannot be
 * enqueued, the host waits for them instead and sep_last_error says so.
 * NULL is a no-op; a handle with an active borrowed view is not freed
 * (release the view first).  Handles may be created and freed from several
 * host threads at once. */
SEP_API void sep_handle_free(sep_handle *handle);

/* Message for the calling thread's last failed call ("" if none). */
SEP_API const char *sep_last_error(void);

/* Name of a status code. */
SEP_API const char *sep_status_string(sep_status status);

/* SEP_ABI_VERSION of the library. */
SEP_API int sep_abi_version(void);

/* Number of CUDA kernels this process has launched through the library so far
 * (all devices, all threads); memsets and copies are not counted. */
SEP_API uint64_t sep_launch_count(void);

/*
 * sep_layout_noalloc — the routing layout for callers that cannot allocate.
 *
 * Not an operation of the pages: it computes exactly what sep_layout computes
 * (counts, pool offsets, tile tables, stable slot maps), into arrays the caller
 * owns, and allocates nothing: no cudaMalloc/cudaMallocAsync/cudaFree, no
 * host allocation, no handle.  It exists for callers that must not allocate
 * device memory on this path: a serving runtime that has already handed all
 * of HBM to its own pool (KV cache and expert workspaces) and forbids further
 * cudaMalloc, code that runs where an allocation would synchronise the device
 * or fragment a caching allocator, and callers that need a fixed memory
 * footprint known at start-up.
 *
 * Its working memory (per-chunk expert histograms and prefix sums, and a
 * grid-barrier counter) is one file-scope __device__ array of 256 KB + 256 B
 * that every GPU which loads the library holds until the process exits.  Hence
 * the limits: num_experts <= 256 and num_tokens * top_k <= 2^21 (2 097 152);
 * larger sizes are rejected with SEP_ERR_INVALID_ARG.  All calls share that
 * array: calls that overlap on the GPU (two streams, or two threads) race and
 * give wrong results; order them.  The call clears the barrier counter and
 * the status words before its kernel; everything else in the array is
 * overwritten before it is read.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current);
 * make that first call before any stream capture.  No dispatch or combine
 * goes with it (those take a handle); the maps it writes are the ones
 * sep_layout would put in a handle.
 *
 *  topk_idx, idx_bytes, num_tokens, top_k, num_experts, num_owners, block_m:
 *      as for sep_layout.
 *  out      host struct of caller-owned device arrays (below).
 *  stream   the stream the work is enqueued on; nothing is synchronised.
 * Errors: SEP_ERR_INVALID_ARG (sizes, limits, pointers, alignment),
 * SEP_ERR_CAPACITY (an output array shorter than the worst case for T),
 * SEP_ERR_CUDA.  Device-side findings go to out->status: status[0] = 1 if an
 * expert id >= num_experts was met (the entry is skipped, as in sep_layout),
 * status[1] = 1 if the kernel's grid barrier gave up its bounded wait.
 */
typedef struct sep_layout_arrays {
    int32_t *expert_counts;            /* [E] */
    int32_t *owner_counts;             /* [R] */
    int32_t *expert_pool_block_offset; /* [E+1] */
    int32_t *owner_pool_row_offset;    /* [R+1] */
    int32_t *tile_expert;              /* [max_tiles] */
    int32_t *pool_arrival_target;      /* [max_tiles] */
    int32_t *src_pool_row;             /* [T, k] */
    int32_t *pool_recv_token;          /* [max_pool_rows] */
    int32_t *pool_recv_slot;           /* [max_pool_rows] */
    int64_t *sizes;                    /* [2] {P, NT} */
    uint32_t *status;                  /* [2] see above */
    int64_t max_pool_rows;             /* rows of the pool_recv_* arrays: >= the worst case
                                          N_a + min(E, N_a) * (block_m - 1), rounded up to block_m */
    int64_t max_tiles;                 /* entries of the tile arrays: >= max_pool_rows / block_m */
} sep_layout_arrays;

SEP_API sep_status sep_layout_noalloc(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                                      int num_experts, int num_owners, int block_m,
                                      const sep_layout_arrays *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SEP_H */
