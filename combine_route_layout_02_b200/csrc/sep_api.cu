// Host side of the sep C ABI: argument validation, handle storage, launches.
//
// Every check happens on the host before anything is enqueued (PR #769,
// "Description": unsupported modes are rejected up front), capacity is checked
// against the worst case or the synced exact size so rows are never silently
// dropped ("DeepEP MoE dispatch/combine" blog, "Imbalance 决定 buffer 与尾延迟"),
// and a handle carries the epoch of its routing so a combine against a
// re-laid-out handle is refused (blog, "EPHandle" and "集成时的数据契约").
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "sep_internal.cuh"

namespace {

thread_local char g_err[512] = "";

sep_status fail(sep_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

sep_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(SEP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int64_t kMaxRows = (1LL << 31) - 1;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Worst-case pool rows for Na assignments: every used expert pads < B rows.
int64_t worst_pool_rows(int64_t Na, int E, int B)
{
    const int64_t used = Na < E ? Na : E;
    const int64_t rows = Na + used * (B - 1);
    return (rows + B - 1) / B * B;
}

sep_status check_dims(int64_t T, int k, int E, int R, int B)
{
    if (T < 0)
        return fail(SEP_ERR_INVALID_ARG, "num_tokens must be >= 0 (got %lld)", (long long)T);
    if (k < 1 || k > 32)
        return fail(SEP_ERR_INVALID_ARG, "top_k must be in 1..32 (got %d)", k);
    if (E < 1 || E > 1024)
        return fail(SEP_ERR_INVALID_ARG, "num_experts must be in 1..1024 (got %d)", E);
    if (R < 1 || R > E || E % R != 0)
        return fail(SEP_ERR_INVALID_ARG, "num_owners must divide num_experts (got %d, %d)", R, E);
    if (B < 1 || B > 1024)
        return fail(SEP_ERR_INVALID_ARG, "block_m must be in 1..1024 (got %d)", B);
    if (T * k > kMaxRows || worst_pool_rows(T * k, E, B) > kMaxRows)
        return fail(SEP_ERR_INVALID_ARG, "num_tokens * top_k too large for 32-bit pool rows");
    return SEP_OK;
}

sep_status current_device(int *dev)
{
    const cudaError_t e = cudaGetDevice(dev);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "cudaGetDevice");
}

sep_status check_device(const sep_handle *h)
{
    int dev = -1;
    sep_status st = current_device(&dev);
    if (st != SEP_OK)
        return st;
    if (dev != h->device)
        return fail(SEP_ERR_INVALID_ARG, "handle lives on device %d, current device is %d", h->device, dev);
    return SEP_OK;
}

size_t carve(size_t *off, size_t bytes)
{
    const size_t at = *off;
    *off = (at + bytes + 255) / 256 * 256;
    return at;
}

// Pinned host words a handle reads its layout sizes and error words into.
// One pinned slab serves many handles, so creating a handle calls no
// cudaMallocHost and freeing one no cudaFreeHost (which synchronises the
// device: a free between a consumer's launch and the dispatch it waits for
// would then stall until the consumer's wait gave up).  Slabs stay until the
// process exits.  A slot is handed back only by sep_handle_free; the one copy
// into it (sep_handle_sync) has completed by then, since that call waits for
// its stream.
class MirrorPool {
  public:
    int64_t *take(cudaError_t *err)
    {
        std::lock_guard<std::mutex> lock(mu_);
        if (free_.empty()) {
            void *slab = nullptr;
            *err = cudaHostAlloc(&slab, kSlots * kSlotBytes, cudaHostAllocPortable);
            if (*err != cudaSuccess)
                return nullptr;
            char *b = static_cast<char *>(slab);
            for (int i = kSlots - 1; i >= 0; --i)
                free_.push_back(reinterpret_cast<int64_t *>(b + (size_t)i * kSlotBytes));
        }
        int64_t *slot = free_.back();
        free_.pop_back();
        *err = cudaSuccess;
        return slot;
    }
    void give(int64_t *slot)
    {
        std::lock_guard<std::mutex> lock(mu_);
        free_.push_back(slot);
    }

  private:
    static constexpr int kSlots = 2048;
    static constexpr size_t kSlotBytes = 32;
    std::mutex mu_;
    std::vector<int64_t *> free_;
};

MirrorPool &mirror_pool()
{
    static MirrorPool pool;
    return pool;
}

// Load all kernels on this device once (see preload_* in sep_internal.cuh).
// Threads that create their first handles at the same time serialise here.
sep_status preload_once(int dev)
{
    static std::atomic<bool> done[64] = {};
    static std::mutex mu;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire))
        return SEP_OK;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_relaxed))
        return SEP_OK;
    cudaError_t e = sep::preload_layout_kernels();
    if (e == cudaSuccess)
        e = sep::preload_dispatch_kernels();
    if (e == cudaSuccess)
        e = sep::preload_combine_kernels();
    if (e == cudaSuccess)
        e = sep::preload_consumer_kernels();
    if (e == cudaSuccess)
        e = sep::preload_gather_kernels();
    if (e == cudaSuccess)
        e = sep::preload_backward_kernels();
    if (e == cudaSuccess)
        e = sep::preload_scatter_kernels();
    if (e == cudaSuccess)
        e = sep::preload_ep_kernels();
    if (e != cudaSuccess)
        return cuda_fail(e, "loading the library's kernels");
    if (dev >= 0 && dev < 64)
        done[dev].store(true, std::memory_order_release);
    return SEP_OK;
}

sep_status create(int64_t T_cap, int k, int E, int R, int B, uint32_t flags, cudaStream_t s,
                  sep_handle **out)
{
    sep_status st = check_dims(T_cap, k, E, R, B);
    if (st != SEP_OK)
        return st;
    int dev = -1;
    if ((st = current_device(&dev)) != SEP_OK)
        return st;
    if ((st = preload_once(dev)) != SEP_OK)
        return st;
    sep_handle *h = new (std::nothrow) sep_handle();
    if (h == nullptr)
        return fail(SEP_ERR_CUDA, "out of host memory");
    h->device = dev;
    h->k = k;
    h->E = E;
    h->R = R;
    h->B = B;
    h->flags_cap = flags;
    h->T_cap = T_cap;
    h->Na_cap = T_cap * k;
    h->P_cap = worst_pool_rows(h->Na_cap, E, B);
    h->NT_cap = h->P_cap / B;
    h->wchunk_cap = sep::layout_wchunk_capacity(h->Na_cap);
    h->last_stream = s;

    const int64_t P1 = h->P_cap > 0 ? h->P_cap : 1;
    const int64_t NT1 = h->NT_cap > 0 ? h->NT_cap : 1;
    const int64_t Na1 = h->Na_cap > 0 ? h->Na_cap : 1;
    size_t off = 0;
    const size_t o_sizes = carve(&off, 32);              // {P, NT}, bad_epoch, timeout_epoch: one copy to the host
    const size_t o_bar = carve(&off, 256);             // two counters, 128 bytes apart (own cache lines)
    const size_t o_ec = carve(&off, (size_t)E * 4);
    const size_t o_oc = carve(&off, (size_t)R * 4);
    const size_t o_otc = carve(&off, (size_t)R * 4);
    const size_t o_off = carve(&off, (size_t)(E + 1) * 4);
    const size_t o_roff = carve(&off, (size_t)(R + 1) * 4);
    const size_t o_te = carve(&off, (size_t)NT1 * 4);
    const size_t o_tg = carve(&off, (size_t)NT1 * 4);
    const size_t o_ac = carve(&off, (size_t)NT1 * 4);
    const size_t o_spr = carve(&off, (size_t)Na1 * 4);
    const size_t o_tok = carve(&off, (size_t)P1 * 4);
    const size_t o_slot = carve(&off, (size_t)P1 * 4);
    const size_t o_hist = carve(&off, (size_t)h->wchunk_cap * ((E + 3) / 4 * 4) * 4);   // rows padded to 4
    const size_t o_base = carve(&off, (size_t)h->wchunk_cap * E * 4);
    const size_t o_in = (flags & SEP_LAYOUT_TOKEN_IN_OWNER) ? carve(&off, (size_t)(T_cap > 0 ? T_cap : 1) * R) : 0;
    const size_t o_arr = carve(&off, (size_t)(T_cap > 0 ? T_cap : 1) * 4);

    cudaError_t e = cudaMallocAsync(&h->block, off, s);
    if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "cudaMallocAsync (handle storage)");
    }
    h->host_mirror = mirror_pool().take(&e);
    if (h->host_mirror == nullptr) {
        cudaFreeAsync(h->block, s);
        delete h;
        return cuda_fail(e, "cudaHostAlloc (pinned mirror slab)");
    }
    char *b = static_cast<char *>(h->block);
    h->sizes = reinterpret_cast<int64_t *>(b + o_sizes);
    h->bad_epoch = reinterpret_cast<uint32_t *>(b + o_sizes + 16);
    h->timeout_epoch = reinterpret_cast<uint32_t *>(b + o_sizes + 20);
    h->barrier_words = reinterpret_cast<uint32_t *>(b + o_bar);
    h->expert_counts = reinterpret_cast<int32_t *>(b + o_ec);
    h->owner_counts = reinterpret_cast<int32_t *>(b + o_oc);
    h->owner_token_counts = reinterpret_cast<int32_t *>(b + o_otc);
    h->expert_pool_block_offset = reinterpret_cast<int32_t *>(b + o_off);
    h->owner_pool_row_offset = reinterpret_cast<int32_t *>(b + o_roff);
    h->tile_expert = reinterpret_cast<int32_t *>(b + o_te);
    h->pool_arrival_target = reinterpret_cast<int32_t *>(b + o_tg);
    h->pool_arrival_count = reinterpret_cast<uint32_t *>(b + o_ac);
    h->src_pool_row = reinterpret_cast<int32_t *>(b + o_spr);
    h->pool_recv_token = reinterpret_cast<int32_t *>(b + o_tok);
    h->pool_recv_slot = reinterpret_cast<int32_t *>(b + o_slot);
    h->wchunk_hist = reinterpret_cast<int32_t *>(b + o_hist);
    h->wchunk_base = reinterpret_cast<int32_t *>(b + o_base);
    h->is_token_in_rank = (flags & SEP_LAYOUT_TOKEN_IN_OWNER) ? reinterpret_cast<uint8_t *>(b + o_in) : nullptr;
    h->token_arrivals = reinterpret_cast<uint32_t *>(b + o_arr);
    e = cudaMemsetAsync(h->sizes, 0, o_bar + 256 - o_sizes, s);   // sizes, error words, barrier counters
    if (e != cudaSuccess) {
        cudaFreeAsync(h->block, s);
        mirror_pool().give(h->host_mirror);
        delete h;
        return cuda_fail(e, "cudaMemsetAsync (handle)");
    }
    h->T = 0;
    h->epoch = 0;
    h->synced = 0;
    h->P = h->NT = -1;
    *out = h;
    return SEP_OK;
}

// A borrowed view leases the handle's row map to its consumers.
sep_status check_not_leased(const sep_handle *h)
{
    if (h->leased)
        return fail(SEP_ERR_HANDLE_MISMATCH, "a borrowed view of this handle is active: call sep_view_release first");
    return SEP_OK;
}

// Order work on stream s after the consumers a view release recorded.
sep_status wait_for_release(sep_handle *h, cudaStream_t s, bool clear)
{
    for (int i = 0; i < h->n_release; ++i) {
        const cudaError_t e = cudaStreamWaitEvent(s, h->release_events[i], 0);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaStreamWaitEvent (view release)");
    }
    if (clear)
        h->n_release = 0;
    return SEP_OK;
}

// Rows a buffer must hold for the handle's current layout.
int64_t needed_rows(const sep_handle *h)
{
    return h->synced ? h->P : worst_pool_rows(h->T * h->k, h->E, h->B);
}

}  // namespace

namespace sep {

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

sep_status set_error(sep_status st, const char *msg)
{
    return fail(st, "%s", msg);
}

int device_sm_count()
{
    static std::atomic<int> cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

int occupancy_blocks_per_sm(const void *kernel, int threads, size_t smem)
{
    struct Entry {
        const void *kernel;
        int threads;
        int blocks;
    };
    static Entry cache[32];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].kernel == kernel && cache[i].threads == threads)
            return cache[i].blocks;
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, smem) != cudaSuccess || b < 1)
        b = 1;
    if (used < 32)
        cache[used++] = Entry{kernel, threads, b};
    return b;
}

}  // namespace sep

extern "C" {

int sep_abi_version(void) { return SEP_ABI_VERSION; }

uint64_t sep_launch_count(void) { return sep::g_launches.load(std::memory_order_relaxed); }

const char *sep_last_error(void) { return g_err; }

const char *sep_status_string(sep_status st)
{
    switch (st) {
    case SEP_OK: return "SEP_OK";
    case SEP_ERR_INVALID_ARG: return "SEP_ERR_INVALID_ARG";
    case SEP_ERR_CAPACITY: return "SEP_ERR_CAPACITY";
    case SEP_ERR_BAD_EXPERT_ID: return "SEP_ERR_BAD_EXPERT_ID";
    case SEP_ERR_HANDLE_MISMATCH: return "SEP_ERR_HANDLE_MISMATCH";
    case SEP_ERR_TIMEOUT: return "SEP_ERR_TIMEOUT";
    case SEP_ERR_CUDA: return "SEP_ERR_CUDA";
    }
    return "SEP_ERR_UNKNOWN";
}

sep_status sep_handle_create(int64_t max_tokens, int top_k, int num_experts, int num_owners,
                             int block_m, uint32_t flags, void *stream, sep_handle **handle)
{
    if (handle == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "handle out-pointer is NULL");
    if (flags & ~(SEP_LAYOUT_SYNC_COUNTS | SEP_LAYOUT_TOKEN_IN_OWNER))
        return fail(SEP_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    return create(max_tokens, top_k, num_experts, num_owners, block_m, flags,
                  static_cast<cudaStream_t>(stream), handle);
}

}  // extern "C"

namespace {

// Everything sep_layout does before its launch: argument checks, the handle
// (created, or reused and re-armed for a new routing) and the kernel
// parameters.  Nothing is enqueued except a new handle's allocation.
sep_status layout_begin(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k, int num_experts,
                        int num_owners, int block_m, uint32_t flags, cudaStream_t s, sep_handle **handle,
                        sep::LayoutParams *out)
{
    if (handle == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "handle in/out pointer is NULL");
    if (flags & ~(SEP_LAYOUT_SYNC_COUNTS | SEP_LAYOUT_TOKEN_IN_OWNER))
        return fail(SEP_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if (idx_bytes != 4 && idx_bytes != 8)
        return fail(SEP_ERR_INVALID_ARG, "idx_bytes must be 4 or 8 (got %d)", idx_bytes);
    sep_status st = check_dims(num_tokens, top_k, num_experts, num_owners, block_m);
    if (st != SEP_OK)
        return st;
    if (num_tokens > 0 && topk_idx == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "topk_idx is NULL");
    if (topk_idx != nullptr && (reinterpret_cast<uintptr_t>(topk_idx) % idx_bytes) != 0)
        return fail(SEP_ERR_INVALID_ARG, "topk_idx is not %d-byte aligned", idx_bytes);

    sep_handle *h = *handle;
    if (h != nullptr) {
        if ((st = check_device(h)) != SEP_OK)
            return st;
        if (h->k != top_k || h->E != num_experts || h->R != num_owners || h->B != block_m)
            return fail(SEP_ERR_HANDLE_MISMATCH, "handle was made for k=%d E=%d R=%d B=%d", h->k, h->E, h->R, h->B);
        if (num_tokens > h->T_cap)
            return fail(SEP_ERR_HANDLE_MISMATCH, "handle holds at most %lld tokens (got %lld)",
                        (long long)h->T_cap, (long long)num_tokens);
        if ((flags & SEP_LAYOUT_TOKEN_IN_OWNER) && h->is_token_in_rank == nullptr)
            return fail(SEP_ERR_HANDLE_MISMATCH, "handle was made without SEP_LAYOUT_TOKEN_IN_OWNER");
        if ((st = check_not_leased(h)) != SEP_OK)
            return st;
        if ((st = wait_for_release(h, s, true)) != SEP_OK)   // consumers of the old row map finish first
            return st;
    } else {
        if ((st = create(num_tokens, top_k, num_experts, num_owners, block_m, flags, s, &h)) != SEP_OK)
            return st;
    }

    h->T = num_tokens;
    h->flags = flags;
    h->arrivals_used = 0;                                // the assign kernel zeroes the counts
    h->epoch += 1;
    h->synced = 0;
    h->P = h->NT = -1;
    h->last_stream = s;

    sep::LayoutParams p{};
    p.topk_idx = topk_idx;
    p.T = num_tokens;
    p.k = top_k;
    p.E = num_experts;
    p.R = num_owners;
    p.B = block_m;
    p.Na = num_tokens * top_k;
    p.rounds = sep::layout_rounds_for(p.Na);
    p.num_wchunks = (int)sep::layout_wchunks_for(p.Na, p.rounds);
    p.wchunk_hist = h->wchunk_hist;
    p.wchunk_base = h->wchunk_base;
    p.expert_counts = h->expert_counts;
    p.owner_counts = h->owner_counts;
    p.owner_token_counts = h->owner_token_counts;
    p.is_token_in_rank = (flags & SEP_LAYOUT_TOKEN_IN_OWNER) ? h->is_token_in_rank : nullptr;
    p.expert_pool_block_offset = h->expert_pool_block_offset;
    p.owner_pool_row_offset = h->owner_pool_row_offset;
    p.tile_expert = h->tile_expert;
    p.pool_arrival_target = h->pool_arrival_target;
    p.pool_arrival_count = h->pool_arrival_count;
    p.src_pool_row = h->src_pool_row;
    p.pool_recv_token = h->pool_recv_token;
    p.pool_recv_slot = h->pool_recv_slot;
    p.sizes = h->sizes;
    p.bad_epoch = h->bad_epoch;
    p.timeout_epoch = h->timeout_epoch;
    p.barrier_words = h->barrier_words;
    p.epoch = h->epoch;
    *handle = h;
    if (p.num_wchunks > h->wchunk_cap)
        return fail(SEP_ERR_CUDA, "internal: chunk table too small");
    *out = p;
    return SEP_OK;
}

}  // namespace

extern "C" {

sep_status sep_layout(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                      int num_experts, int num_owners, int block_m, uint32_t flags, void *stream,
                      sep_handle **handle)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sep::LayoutParams p{};
    sep_status st = layout_begin(topk_idx, idx_bytes, num_tokens, top_k, num_experts, num_owners, block_m, flags, s,
                                 handle, &p);
    if (st != SEP_OK)
        return st;
    cudaError_t e = sep::launch_layout(p, idx_bytes, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "layout launch");
    if (flags & SEP_LAYOUT_SYNC_COUNTS)
        return sep_handle_sync(*handle, stream);
    return SEP_OK;
}

sep_status sep_handle_info(const sep_handle *h, sep_layout_info *info)
{
    if (h == nullptr || info == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle or info");
    std::memset(info, 0, sizeof *info);
    info->num_tokens = h->T;
    info->top_k = h->k;
    info->num_experts = h->E;
    info->num_owners = h->R;
    info->block_m = h->B;
    info->max_tokens = h->T_cap;
    info->max_pool_rows = h->P_cap;
    info->max_tiles = h->NT_cap;
    info->num_pool_rows = h->synced ? h->P : -1;
    info->num_tiles = h->synced ? h->NT : -1;
    info->epoch = h->epoch;
    info->flags = h->flags;
    info->expert_counts = h->expert_counts;
    info->owner_counts = h->owner_counts;
    info->owner_token_counts = h->owner_token_counts;
    info->is_token_in_rank = (h->flags & SEP_LAYOUT_TOKEN_IN_OWNER) ? h->is_token_in_rank : nullptr;
    info->expert_pool_block_offset = h->expert_pool_block_offset;
    info->owner_pool_row_offset = h->owner_pool_row_offset;
    info->tile_expert = h->tile_expert;
    info->pool_arrival_target = h->pool_arrival_target;
    info->pool_arrival_count = h->pool_arrival_count;
    info->src_pool_row = h->src_pool_row;
    info->pool_recv_token = h->pool_recv_token;
    info->pool_recv_slot = h->pool_recv_slot;
    info->device_sizes = h->sizes;
    return SEP_OK;
}

sep_status sep_handle_set_max_ctas(sep_handle *h, int max_ctas)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    if (max_ctas < 0)
        return fail(SEP_ERR_INVALID_ARG, "max_ctas must be >= 0 (got %d)", max_ctas);
    h->max_ctas = max_ctas;
    return SEP_OK;
}

sep_status sep_handle_sync(sep_handle *h, void *stream)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(h->host_mirror, h->sizes, 24, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync (sizes)");
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess)
        return cuda_fail(e, "cudaStreamSynchronize");
    h->P = h->host_mirror[0];
    h->NT = h->host_mirror[1];
    h->synced = 1;
    uint32_t words[2] = {0, 0};
    std::memcpy(words, h->host_mirror + 2, sizeof words);
    if (words[0] != 0 && words[0] == h->epoch)
        return fail(SEP_ERR_BAD_EXPERT_ID, "topk_idx holds an expert id >= num_experts (%d)", h->E);
    if (words[1] != 0 && words[1] == h->epoch)
        return fail(SEP_ERR_TIMEOUT, "a layout barrier or dispatch/combine copy did not complete within its wait limit");
    return SEP_OK;
}

}  // extern "C"

namespace {

// Checks of a dispatch's payload arguments against a pool that must hold
// need_rows rows (the handle-independent part of sep_dispatch's checks).
sep_status check_payload_args(int64_t T, const void *x, int64_t hidden, int payload, int scale, const void *recv_x,
                              const void *recv_scales, int64_t recv_capacity_rows, int64_t need_rows, bool synced)
{
    if (payload != SEP_PAYLOAD_BF16 && payload != SEP_PAYLOAD_FP8_E4M3)
        return fail(SEP_ERR_INVALID_ARG, "unknown payload %d", payload);
    const bool fp8 = payload == SEP_PAYLOAD_FP8_E4M3;
    if (!fp8 && scale != SEP_SCALE_NONE)
        return fail(SEP_ERR_INVALID_ARG, "bf16 payload takes SEP_SCALE_NONE");
    if (fp8 && scale != SEP_SCALE_F32 && scale != SEP_SCALE_UE8M0 && scale != SEP_SCALE_F32_POW2)
        return fail(SEP_ERR_INVALID_ARG, "FP8 payload needs a scale format (got %d)", scale);
    if (hidden < 1 || hidden > 65536 || hidden % (fp8 ? 128 : 8) != 0)
        return fail(SEP_ERR_INVALID_ARG, "hidden must be a multiple of %d in 1..65536 (got %lld)",
                    fp8 ? 128 : 8, (long long)hidden);
    if (T > 0 && (x == nullptr || recv_x == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "x or recv_x is NULL");
    if (!aligned16(x) || !aligned16(recv_x))
        return fail(SEP_ERR_INVALID_ARG, "x and recv_x must be 16-byte aligned");
    if (fp8) {
        if (T > 0 && recv_scales == nullptr)
            return fail(SEP_ERR_INVALID_ARG, "recv_scales is NULL");
        if (scale != SEP_SCALE_UE8M0 && (reinterpret_cast<uintptr_t>(recv_scales) & 3u))
            return fail(SEP_ERR_INVALID_ARG, "fp32 recv_scales must be 4-byte aligned");
    }
    if (recv_capacity_rows < need_rows)
        return fail(SEP_ERR_CAPACITY, "recv_x holds %lld rows, the layout needs %lld%s",
                    (long long)recv_capacity_rows, (long long)need_rows,
                    synced ? "" : " (worst case; sync the layout for the exact size)");
    return SEP_OK;
}

sep::DispatchParams dispatch_params(const sep_handle *h, const void *x, int64_t hidden, int scale, void *recv_x,
                                    void *recv_scales)
{
    sep::DispatchParams p{};
    p.x = x;
    p.T = h->T;
    p.H = (int)hidden;
    p.k = h->k;
    p.B = h->B;
    p.src_pool_row = h->src_pool_row;
    p.recv = recv_x;
    p.recv_scales = recv_scales;
    p.scale = scale;
    p.pool_arrival_count = h->pool_arrival_count;
    p.pool_arrival_target = h->pool_arrival_target;
    p.error_epoch = h->timeout_epoch;
    p.epoch = h->epoch;
    p.max_ctas = h->max_ctas;
    return p;
}

}  // namespace

extern "C" {

sep_status sep_dispatch(sep_handle *h, const void *x, int64_t hidden, int payload, int scale,
                        void *recv_x, void *recv_scales, int64_t recv_capacity_rows,
                        uint32_t *tile_ready, int64_t tile_ready_len, uint32_t dispatch_seq, void *stream)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st == SEP_OK)
        st = check_not_leased(h);
    if (st != SEP_OK)
        return st;
    const int64_t need = needed_rows(h);
    if ((st = check_payload_args(h->T, x, hidden, payload, scale, recv_x, recv_scales, recv_capacity_rows, need,
                                 h->synced)) != SEP_OK)
        return st;
    if (tile_ready != nullptr) {
        if (dispatch_seq == 0)
            return fail(SEP_ERR_INVALID_ARG, "dispatch_seq must be nonzero with tile_ready");
        if ((reinterpret_cast<uintptr_t>(tile_ready) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "tile_ready must be 4-byte aligned");
        if (tile_ready_len < need / h->B)
            return fail(SEP_ERR_CAPACITY, "tile_ready holds %lld entries, the layout needs %lld",
                        (long long)tile_ready_len, (long long)(need / h->B));
        if (tile_ready == h->last_tile_ready && (int32_t)(dispatch_seq - h->last_seq) <= 0)
            return fail(SEP_ERR_INVALID_ARG, "dispatch_seq %u does not advance past %u for this tile_ready",
                        dispatch_seq, h->last_seq);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(h, s, false)) != SEP_OK)
        return st;
    h->last_stream = s;
    if (tile_ready != nullptr) {
        h->last_tile_ready = tile_ready;
        h->last_seq = dispatch_seq;
    }
    if (h->T == 0)
        return SEP_OK;
    if (tile_ready != nullptr) {
        if (h->arrivals_used) {                          // a second streaming dispatch of this layout
            cudaError_t e = cudaMemsetAsync(h->pool_arrival_count, 0, (size_t)(h->NT_cap > 0 ? h->NT_cap : 1) * 4, s);
            if (e != cudaSuccess)
                return cuda_fail(e, "cudaMemsetAsync (arrival counts)");
        }
        h->arrivals_used = 1;
    }

    sep::DispatchParams p = dispatch_params(h, x, hidden, scale, recv_x, recv_scales);
    p.tile_ready = tile_ready;
    p.seq = dispatch_seq;
    cudaError_t e = sep::launch_dispatch(p, payload, s, sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "dispatch launch");
}

sep_status sep_layout_dispatch(const void *topk_idx, int idx_bytes, int64_t num_tokens, int top_k,
                               int num_experts, int num_owners, int block_m, uint32_t flags, const void *x,
                               int64_t hidden, int payload, int scale, void *recv_x, void *recv_scales,
                               int64_t recv_capacity_rows, void *stream, sep_handle **handle)
{
    // every check before anything changes: the pool must hold the worst case
    // for num_tokens, since the exact size is known only after the layout
    sep_status st = check_dims(num_tokens, top_k, num_experts, num_owners, block_m);
    if (st != SEP_OK)
        return st;
    if ((st = check_payload_args(num_tokens, x, hidden, payload, scale, recv_x, recv_scales, recv_capacity_rows,
                                 worst_pool_rows(num_tokens * top_k, num_experts, block_m), false)) != SEP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool one_launch = (flags & SEP_LAYOUT_ONE_LAUNCH) != 0;
    flags &= ~(uint32_t)SEP_LAYOUT_ONE_LAUNCH;
    sep::LayoutParams lp{};
    if ((st = layout_begin(topk_idx, idx_bytes, num_tokens, top_k, num_experts, num_owners, block_m,
                           flags & ~(uint32_t)SEP_LAYOUT_SYNC_COUNTS, s, handle, &lp)) != SEP_OK)
        return st;
    sep_handle *h = *handle;
    h->flags = flags;
    const sep::DispatchParams dp = dispatch_params(h, x, hidden, scale, recv_x, recv_scales);
    bool fused = false;
    cudaError_t e = one_launch ? sep::try_layout_dispatch(lp, idx_bytes, dp, payload, s, &fused) : cudaSuccess;
    if (e != cudaSuccess)
        return cuda_fail(e, "layout + dispatch launch");
    if (!fused) {
        if ((e = sep::launch_layout(lp, idx_bytes, s)) != cudaSuccess)
            return cuda_fail(e, "layout launch");
        if (h->T > 0 && (e = sep::launch_dispatch(dp, payload, s, sep::device_sm_count())) != cudaSuccess)
            return cuda_fail(e, "dispatch launch");
    }
    if (flags & SEP_LAYOUT_SYNC_COUNTS)
        return sep_handle_sync(h, stream);
    return SEP_OK;
}

namespace {

// Checks shared by the combine family and the parameters they launch with.
// y is a pool-layout bf16 array of y_rows rows, w the routing weights (NULL:
// unit weights), out the token-order result.  *empty is set when the layout
// has no tokens (nothing to launch).
sep_status prepare_combine(const sep_handle *h, uint32_t layout_epoch, const void *y, int64_t hidden,
                           int64_t y_rows, const float *w, bool weighted, void *out, cudaStream_t s,
                           sep::CombineParams *p, bool *empty)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    if (layout_epoch != h->epoch)
        return fail(SEP_ERR_HANDLE_MISMATCH, "handle epoch is %u, caller's routing has epoch %u",
                    h->epoch, layout_epoch);
    if ((st = check_not_leased(h)) != SEP_OK)
        return st;
    if (hidden < 1 || hidden > 65536 || hidden % 8 != 0)
        return fail(SEP_ERR_INVALID_ARG, "hidden must be a multiple of 8 in 1..65536 (got %lld)",
                    (long long)hidden);
    if (h->T > 0 && (y == nullptr || (weighted && w == nullptr) || out == nullptr))
        return fail(SEP_ERR_INVALID_ARG, weighted ? "y_pool, topk_weight or out is NULL"
                                                  : "grad_recv or grad_x is NULL");
    if (!aligned16(y) || !aligned16(out))
        return fail(SEP_ERR_INVALID_ARG, "pool rows and output must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(w) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "topk_weight must be 4-byte aligned");
    const int64_t need = needed_rows(h);
    if (y_rows < need)
        return fail(SEP_ERR_CAPACITY, "the pool array holds %lld rows, the layout needs %lld",
                    (long long)y_rows, (long long)need);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    *empty = h->T == 0;
    if (*empty)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;

    *p = sep::CombineParams{};
    p->y = y;
    p->T = h->T;
    p->H = (int)hidden;
    p->k = h->k;
    p->src_pool_row = h->src_pool_row;
    p->w = weighted ? w : nullptr;
    p->out = out;
    p->max_ctas = h->max_ctas;
    p->error_epoch = h->timeout_epoch;
    p->epoch = h->epoch;
    return SEP_OK;
}

uint32_t poll_budget(uint64_t timeout_ns)
{
    const uint64_t polls = timeout_ns / 128 + 1024;
    return polls > 0xffffffffull ? 0xffffffffu : (uint32_t)polls;
}

}  // namespace

sep_status sep_combine(const sep_handle *h, uint32_t layout_epoch, const void *y_pool, int64_t hidden,
                       int64_t y_capacity_rows, const float *topk_weight, void *out, void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sep::CombineParams p;
    bool empty = false;
    sep_status st = prepare_combine(h, layout_epoch, y_pool, hidden, y_capacity_rows, topk_weight, true, out, s,
                                    &p, &empty);
    if (st != SEP_OK || empty)
        return st;
    cudaError_t e = sep::launch_combine(p, s, sep::device_sm_count(), 0);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "combine launch");
}

sep_status sep_combine_scatter(const sep_handle *h, uint32_t layout_epoch, const void *y_pool, int64_t hidden,
                               int64_t y_capacity_rows, const float *topk_weight, void *out, void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sep::CombineParams c;
    bool empty = false;
    sep_status st = prepare_combine(h, layout_epoch, y_pool, hidden, y_capacity_rows, topk_weight, true, out, s,
                                    &c, &empty);
    if (st != SEP_OK || empty)
        return st;
    cudaError_t e = cudaMemsetAsync(out, 0, (size_t)h->T * (size_t)hidden * 2, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync (out)");
    const int num_sms = sep::device_sm_count();
    sep::ScatterParams p{};
    p.y = y_pool;
    p.H = (int)hidden;
    p.k = h->k;
    p.pool_recv_token = h->pool_recv_token;
    p.pool_recv_slot = h->pool_recv_slot;
    p.w = topk_weight;
    p.out = out;
    p.num_pool_rows = h->sizes;
    p.rows_cap = needed_rows(h);
    e = sep::launch_combine_scatter(p, s, num_sms);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "scatter combine launch");
}

sep_status sep_combine_grads(const sep_handle *h, uint32_t layout_epoch, const void *grad_recv, int64_t hidden,
                             int64_t capacity_rows, void *grad_x, void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sep::CombineParams p;
    bool empty = false;
    sep_status st = prepare_combine(h, layout_epoch, grad_recv, hidden, capacity_rows, nullptr, false, grad_x, s,
                                    &p, &empty);
    if (st != SEP_OK || empty)
        return st;
    cudaError_t e = sep::launch_combine(p, s, sep::device_sm_count(), 0);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "combine_grads launch");
}

sep_status sep_combine_gated(const sep_handle *h, uint32_t layout_epoch, const void *y_pool, int64_t hidden,
                             int64_t y_capacity_rows, const float *topk_weight, void *out, const uint32_t *y_done,
                             int64_t y_done_len, uint32_t done_seq, int num_ctas, uint64_t timeout_ns,
                             uint32_t *status, void *stream)
{
    if (h != nullptr) {
        if (y_done == nullptr || status == nullptr)
            return fail(SEP_ERR_INVALID_ARG, "NULL y_done or status");
        if (((reinterpret_cast<uintptr_t>(y_done) | reinterpret_cast<uintptr_t>(status)) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "y_done and status must be 4-byte aligned");
        if (done_seq == 0)
            return fail(SEP_ERR_INVALID_ARG, "done_seq must be nonzero");
        if (num_ctas < 1 || num_ctas > 1024)
            return fail(SEP_ERR_INVALID_ARG, "num_ctas must be in 1..1024");
        if (y_done_len < h->T)
            return fail(SEP_ERR_CAPACITY, "y_done holds %lld entries, the layout has %lld tokens",
                        (long long)y_done_len, (long long)h->T);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sep::CombineParams p;
    bool empty = false;
    sep_status st = prepare_combine(h, layout_epoch, y_pool, hidden, y_capacity_rows, topk_weight, true, out, s,
                                    &p, &empty);
    if (st != SEP_OK)
        return st;
    cudaError_t e = cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync (status)");
    if (empty)
        return SEP_OK;
    p.y_done = y_done;
    p.done_seq = done_seq;
    p.timeout_ns = timeout_ns ? timeout_ns : 1000000000ull;
    p.max_polls = poll_budget(p.timeout_ns);
    p.status = status;
    e = sep::launch_combine(p, s, sep::device_sm_count(), num_ctas);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "gated combine launch");
}

sep_status sep_dispatch_grads(const sep_handle *h, uint32_t layout_epoch, const void *grad_out, int64_t hidden,
                              const float *topk_weight, const void *y_pool, int64_t y_capacity_rows, void *grad_y,
                              int64_t grad_y_capacity_rows, float *grad_w, void *stream)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    if (layout_epoch != h->epoch)
        return fail(SEP_ERR_HANDLE_MISMATCH, "handle epoch is %u, caller's routing has epoch %u",
                    h->epoch, layout_epoch);
    if ((st = check_not_leased(h)) != SEP_OK)
        return st;
    if (hidden < 1 || hidden > 65536 || hidden % 8 != 0)
        return fail(SEP_ERR_INVALID_ARG, "hidden must be a multiple of 8 in 1..65536 (got %lld)",
                    (long long)hidden);
    if (h->T > 0 && (grad_out == nullptr || topk_weight == nullptr || grad_y == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "grad_out, topk_weight or grad_y is NULL");
    if (h->T > 0 && grad_w != nullptr && y_pool == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "grad_w needs y_pool (the forward expert outputs)");
    if (!aligned16(grad_out) || !aligned16(grad_y) || !aligned16(y_pool))
        return fail(SEP_ERR_INVALID_ARG, "grad_out, grad_y and y_pool must be 16-byte aligned");
    if (((reinterpret_cast<uintptr_t>(topk_weight) | reinterpret_cast<uintptr_t>(grad_w)) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "topk_weight and grad_w must be 4-byte aligned");
    const int64_t need = needed_rows(h);
    if (grad_y_capacity_rows < need)
        return fail(SEP_ERR_CAPACITY, "grad_y holds %lld rows, the layout needs %lld",
                    (long long)grad_y_capacity_rows, (long long)need);
    if (grad_w != nullptr && y_capacity_rows < need)
        return fail(SEP_ERR_CAPACITY, "y_pool holds %lld rows, the layout needs %lld",
                    (long long)y_capacity_rows, (long long)need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    if (h->T == 0)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;

    const int num_sms = sep::device_sm_count();
    sep::DispatchGradsParams p{};
    p.g = grad_out;
    p.w = topk_weight;
    p.y = grad_w ? y_pool : nullptr;
    p.grad_y = grad_y;
    p.grad_w = grad_w;
    p.T = h->T;
    p.H = (int)hidden;
    p.k = h->k;
    p.src_pool_row = h->src_pool_row;
    cudaError_t e = sep::launch_dispatch_grads(p, s, num_sms);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "dispatch_grads launch");
}

namespace {

sep_status consume(const sep_handle *h, const void *recv_x, int64_t row_bytes, int64_t capacity_rows,
                   const uint32_t *tile_ready, int64_t tile_ready_len, uint32_t dispatch_seq, void *dst, int num_ctas,
                   uint64_t timeout_ns, uint32_t *status, uint32_t *y_done, uint32_t done_seq, cudaStream_t s)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    if (tile_ready == nullptr || status == nullptr || (h->T > 0 && (recv_x == nullptr || dst == nullptr)))
        return fail(SEP_ERR_INVALID_ARG, "NULL tile_ready, status, recv_x or dst");
    if (row_bytes < 16 || row_bytes % 16 != 0 || row_bytes > (1LL << 20))
        return fail(SEP_ERR_INVALID_ARG, "row_bytes must be a multiple of 16 in 16..2^20");
    if (!aligned16(recv_x) || !aligned16(dst))
        return fail(SEP_ERR_INVALID_ARG, "recv_x and dst must be 16-byte aligned");
    if (((reinterpret_cast<uintptr_t>(tile_ready) | reinterpret_cast<uintptr_t>(status) |
          reinterpret_cast<uintptr_t>(y_done)) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "tile_ready, status and y_done must be 4-byte aligned");
    if (dispatch_seq == 0)
        return fail(SEP_ERR_INVALID_ARG, "dispatch_seq must be nonzero");
    if (num_ctas < 1 || num_ctas > 1024)
        return fail(SEP_ERR_INVALID_ARG, "num_ctas must be in 1..1024");
    const int64_t need = needed_rows(h);
    if (capacity_rows < need)
        return fail(SEP_ERR_CAPACITY, "recv_x/dst hold %lld rows, the layout needs %lld",
                    (long long)capacity_rows, (long long)need);
    if (tile_ready_len < need / h->B)
        return fail(SEP_ERR_CAPACITY, "tile_ready holds %lld entries, the layout needs %lld",
                    (long long)tile_ready_len, (long long)(need / h->B));
    cudaError_t e = cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync (status)");
    if (h->T == 0)
        return SEP_OK;
    if (y_done != nullptr) {
        e = cudaMemsetAsync(h->token_arrivals, 0, (size_t)h->T * 4, s);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaMemsetAsync (token counters)");
    }
    sep::ConsumeParams p{};
    p.src = static_cast<const uint8_t *>(recv_x);
    p.dst = static_cast<uint8_t *>(dst);
    p.row_bytes = row_bytes;
    p.E = h->E;
    p.B = h->B;
    p.expert_pool_block_offset = h->expert_pool_block_offset;
    p.pool_recv_token = h->pool_recv_token;
    p.tile_ready = tile_ready;
    p.seq = dispatch_seq;
    p.timeout_ns = timeout_ns ? timeout_ns : 1000000000ull;
    p.max_polls = poll_budget(p.timeout_ns);
    p.status = status;
    p.abort_flag = status;
    p.y_done = y_done;
    p.token_arrivals = h->token_arrivals;
    p.src_pool_row = h->src_pool_row;
    p.k = h->k;
    p.done_seq = done_seq;
    e = sep::launch_consume(p, num_ctas, s);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "consumer launch");
}

}  // namespace

sep_status sep_consume_tiles(const sep_handle *h, const void *recv_x, int64_t row_bytes,
                             int64_t capacity_rows, const uint32_t *tile_ready, int64_t tile_ready_len,
                             uint32_t dispatch_seq, void *dst, int num_ctas, uint64_t timeout_ns,
                             uint32_t *status, void *stream)
{
    return consume(h, recv_x, row_bytes, capacity_rows, tile_ready, tile_ready_len, dispatch_seq, dst, num_ctas,
                   timeout_ns, status, nullptr, 0, static_cast<cudaStream_t>(stream));
}

sep_status sep_consume_tiles_stamp(const sep_handle *h, const void *recv_x, int64_t row_bytes,
                                   int64_t capacity_rows, const uint32_t *tile_ready, int64_t tile_ready_len,
                                   uint32_t dispatch_seq, void *dst, int num_ctas, uint64_t timeout_ns,
                                   uint32_t *status, uint32_t *y_done, int64_t y_done_len, uint32_t done_seq,
                                   void *stream)
{
    if (h != nullptr) {
        if (y_done == nullptr)
            return fail(SEP_ERR_INVALID_ARG, "NULL y_done");
        if (done_seq == 0)
            return fail(SEP_ERR_INVALID_ARG, "done_seq must be nonzero");
        if (y_done_len < h->T)
            return fail(SEP_ERR_CAPACITY, "y_done holds %lld entries, the layout has %lld tokens",
                        (long long)y_done_len, (long long)h->T);
    }
    return consume(h, recv_x, row_bytes, capacity_rows, tile_ready, tile_ready_len, dispatch_seq, dst, num_ctas,
                   timeout_ns, status, y_done, done_seq, static_cast<cudaStream_t>(stream));
}

sep_status sep_dispatch_borrow(sep_handle *h, const void *x, int64_t hidden, int payload, sep_recv_view *view)
{
    if (h == nullptr || view == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle or view");
    sep_status st = check_device(h);
    if (st == SEP_OK)
        st = check_not_leased(h);
    if (st != SEP_OK)
        return st;
    if (payload != SEP_PAYLOAD_BF16)
        return fail(SEP_ERR_INVALID_ARG, "a borrowed view supports the bf16 payload only (FP8 must quantise)");
    if (!h->synced)
        return fail(SEP_ERR_INVALID_ARG, "a borrowed view needs CPU counts: sync the layout first");
    if (hidden < 1 || hidden > 65536 || hidden % 8 != 0)
        return fail(SEP_ERR_INVALID_ARG, "hidden must be a multiple of 8 in 1..65536 (got %lld)", (long long)hidden);
    if (h->T > 0 && x == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "x is NULL");
    if (!aligned16(x))
        return fail(SEP_ERR_INVALID_ARG, "x must be 16-byte aligned");
    view->slab = x;
    view->row_indices = h->pool_recv_token;
    view->num_rows = h->P;
    view->row_bytes = hidden * 2;
    view->indexed = 1;
    view->epoch = h->epoch;
    h->leased = 1;
    return SEP_OK;
}

sep_status sep_view_release(sep_handle *h, void *const *streams, int num_streams)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    if (!h->leased)
        return fail(SEP_ERR_INVALID_ARG, "the handle has no active borrowed view");
    if (num_streams < 0 || num_streams > 8 || (num_streams > 0 && streams == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "num_streams must be in 0..8");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    for (int i = 0; i < num_streams; ++i) {
        if (i >= h->release_events_made) {
            const cudaError_t e = cudaEventCreateWithFlags(&h->release_events[i], cudaEventDisableTiming);
            if (e != cudaSuccess)
                return cuda_fail(e, "cudaEventCreateWithFlags (view release)");
            h->release_events_made = i + 1;
        }
        const cudaError_t e = cudaEventRecord(h->release_events[i], static_cast<cudaStream_t>(streams[i]));
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaEventRecord (view release)");
    }
    h->n_release = num_streams;
    h->leased = 0;
    return SEP_OK;
}

sep_status sep_gather_rows(const sep_recv_view *view, void *dst, int64_t dst_rows, void *stream)
{
    if (view == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL view");
    const sep_recv_view &v = *view;
    if (v.num_rows < 0 || v.row_bytes < 16 || v.row_bytes % 16 != 0 || v.row_bytes > (1LL << 20))
        return fail(SEP_ERR_INVALID_ARG, "view needs num_rows >= 0 and row_bytes a multiple of 16 in 16..2^20");
    if (v.num_rows > 0 && (v.slab == nullptr || v.row_indices == nullptr || dst == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "NULL slab, row_indices or dst");
    if (!aligned16(v.slab) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(v.row_indices) & 3u))
        return fail(SEP_ERR_INVALID_ARG, "slab and dst must be 16-byte aligned, row_indices 4-byte aligned");
    if (dst_rows < v.num_rows)
        return fail(SEP_ERR_CAPACITY, "dst holds %lld rows, the view has %lld", (long long)dst_rows,
                    (long long)v.num_rows);
    sep::GatherParams p{};
    p.slab = static_cast<const uint8_t *>(v.slab);
    p.row_indices = v.row_indices;
    p.dst = static_cast<uint8_t *>(dst);
    p.rows = v.num_rows;
    p.row_bytes = v.row_bytes;
    p.indexed = v.indexed ? 1 : 0;
    const cudaError_t e = sep::launch_gather(p, static_cast<cudaStream_t>(stream), sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "gather launch");
}

// ------------------------------------------------------- expert parallelism


sep_status sep_ep_plan(const int32_t *all_counts, int num_ranks, int num_experts, int block_m, int rank,
                       int32_t *delta, int64_t *owner_rows, int32_t *owner_block_offset,
                       int32_t *owner_expert_counts)
{
    if (all_counts == nullptr || delta == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL all_counts or delta");
    if (num_ranks < 1 || num_ranks > 1024 || num_experts < 1 || num_experts > 1024 ||
        num_experts % num_ranks != 0)
        return fail(SEP_ERR_INVALID_ARG, "need 1 <= num_ranks <= 1024, num_experts in 1..1024 divisible by num_ranks");
    if (block_m < 1 || block_m > 1024)
        return fail(SEP_ERR_INVALID_ARG, "block_m must be in 1..1024");
    if (rank < 0 || rank >= num_ranks)
        return fail(SEP_ERR_INVALID_ARG, "rank %d outside 0..%d", rank, num_ranks - 1);
    const int R = num_ranks, E = num_experts, El = E / R, B = block_m;
    for (int64_t i = 0; i < (int64_t)R * E; ++i)
        if (all_counts[i] < 0)
            return fail(SEP_ERR_INVALID_ARG, "all_counts[%lld] is negative", (long long)i);
    int64_t loff = 0;                                    // this rank's local block offset (tiles), running over e
    int64_t gboff = 0;                                   // owner-local block offset of e (tiles)
    for (int e = 0; e < E; ++e) {
        if (e % El == 0) {
            if (e > 0 && owner_rows != nullptr)
                owner_rows[e / El - 1] = gboff * B;
            gboff = 0;
        }
        int64_t N = 0, before = 0;
        for (int r = 0; r < R; ++r) {
            const int64_t c = all_counts[(int64_t)r * E + e];
            if (r < rank)
                before += c;
            N += c;
        }
        const int64_t own = all_counts[(int64_t)rank * E + e];
        const int64_t d = gboff * B + before - loff * B;
        if (N > INT32_MAX || d > INT32_MAX || d < INT32_MIN || (gboff + (N + B - 1) / B) * B > INT32_MAX)
            return fail(SEP_ERR_INVALID_ARG, "counts too large for 32-bit pool rows");
        delta[e] = (int32_t)d;
        if (e / El == rank) {
            if (owner_block_offset != nullptr)
                owner_block_offset[e % El] = (int32_t)gboff;
            if (owner_expert_counts != nullptr)
                owner_expert_counts[e % El] = (int32_t)N;
        }
        gboff += (N + B - 1) / B;
        loff += (own + B - 1) / B;
        if (e == E - 1) {
            if (owner_rows != nullptr)
                owner_rows[R - 1] = gboff * B;
        }
        if (e / El == rank && e % El == El - 1 && owner_block_offset != nullptr)
            owner_block_offset[El] = (int32_t)gboff;
    }
    return SEP_OK;
}

namespace {

// Checks shared by sep_ep_dispatch and sep_ep_combine, and the rank-group
// part of their parameters.
struct EpCommon {
    int64_t T;
    int H, k, B, E_loc, R;
    const int32_t *src_pool_row, *tile_expert, *delta;
    uint32_t *error;
    int64_t pool_rows[sep::kEpMaxRanks];
};

sep_status ep_common(const sep_handle *h, uint32_t layout_epoch, int64_t hidden, const int32_t *delta,
                     const int64_t *pool_rows, uint32_t *error, EpCommon *c)
{
    if (h == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL handle");
    sep_status st = check_device(h);
    if (st != SEP_OK)
        return st;
    if (layout_epoch != h->epoch)
        return fail(SEP_ERR_HANDLE_MISMATCH, "handle epoch is %u, caller's routing has epoch %u",
                    h->epoch, layout_epoch);
    if ((st = check_not_leased(h)) != SEP_OK)
        return st;
    if (h->R > sep::kEpMaxRanks)
        return fail(SEP_ERR_INVALID_ARG, "an expert-parallel group has at most %d ranks (the handle has %d owners)",
                    sep::kEpMaxRanks, h->R);
    if (hidden < 1 || hidden > 65536 || hidden % 8 != 0)
        return fail(SEP_ERR_INVALID_ARG, "hidden must be a multiple of 8 in 1..65536 (got %lld)",
                    (long long)hidden);
    if (delta == nullptr || pool_rows == nullptr || error == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL delta, pool_rows or error");
    if (((reinterpret_cast<uintptr_t>(delta) | reinterpret_cast<uintptr_t>(error)) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "delta and error must be 4-byte aligned");
    c->T = h->T;
    c->H = (int)hidden;
    c->k = h->k;
    c->B = h->B;
    c->E_loc = h->E / h->R;
    c->R = h->R;
    c->src_pool_row = h->src_pool_row;
    c->tile_expert = h->tile_expert;
    c->delta = delta;
    c->error = error;
    for (int r = 0; r < h->R; ++r) {
        if (pool_rows[r] < 0 || pool_rows[r] > INT32_MAX)
            return fail(SEP_ERR_INVALID_ARG, "pool_rows[%d] = %lld is outside 0..2^31-1", r, (long long)pool_rows[r]);
        c->pool_rows[r] = pool_rows[r];
    }
    return SEP_OK;
}

}  // namespace

sep_status sep_ep_dispatch(const sep_handle *h, uint32_t layout_epoch, const void *x, int64_t hidden, int rank,
                           const int32_t *delta, void *const *pools, const int64_t *pool_rows,
                           int32_t *const *recv_token, int32_t *const *recv_rank, int32_t *const *recv_slot,
                           uint32_t *error, void *stream)
{
    EpCommon c{};
    sep_status st = ep_common(h, layout_epoch, hidden, delta, pool_rows, error, &c);
    if (st != SEP_OK)
        return st;
    sep::EpDispatchParams p{};
    p.T = c.T;
    p.H = c.H;
    p.k = c.k;
    p.B = c.B;
    p.E_loc = c.E_loc;
    p.R = c.R;
    p.src_pool_row = c.src_pool_row;
    p.tile_expert = c.tile_expert;
    p.delta = c.delta;
    p.error = c.error;
    memcpy(p.pool_rows, c.pool_rows, sizeof(p.pool_rows));
    if (rank < 0 || rank >= h->R)
        return fail(SEP_ERR_INVALID_ARG, "rank %d outside 0..%d", rank, h->R - 1);
    if (pools == nullptr || (h->T > 0 && x == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "NULL pools or x");
    if (!aligned16(x))
        return fail(SEP_ERR_INVALID_ARG, "x must be 16-byte aligned");
    for (int r = 0; r < h->R; ++r) {
        if ((pool_rows[r] > 0 && pools[r] == nullptr) || !aligned16(pools[r]))
            return fail(SEP_ERR_INVALID_ARG, "pools[%d] must be non-NULL (if it has rows) and 16-byte aligned", r);
        p.pools[r] = pools[r];
        p.recv_token[r] = recv_token ? recv_token[r] : nullptr;
        p.recv_rank[r] = recv_rank ? recv_rank[r] : nullptr;
        p.recv_slot[r] = recv_slot ? recv_slot[r] : nullptr;
        if (((reinterpret_cast<uintptr_t>(p.recv_token[r]) | reinterpret_cast<uintptr_t>(p.recv_rank[r]) |
              reinterpret_cast<uintptr_t>(p.recv_slot[r])) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "receive maps of rank %d must be 4-byte aligned", r);
    }
    p.x = x;
    p.rank = rank;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    if (h->T == 0)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;
    const cudaError_t e = sep::launch_ep_dispatch(p, s, sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel dispatch launch");
}

sep_status sep_ep_dispatch_fp8(const sep_handle *h, uint32_t layout_epoch, const void *x, int64_t hidden, int rank,
                               int scale, const int32_t *delta, void *const *pools, void *const *scales,
                               const int64_t *pool_rows, int32_t *const *recv_token, int32_t *const *recv_rank,
                               int32_t *const *recv_slot, uint32_t *error, void *stream)
{
    EpCommon c{};
    sep_status st = ep_common(h, layout_epoch, hidden, delta, pool_rows, error, &c);
    if (st != SEP_OK)
        return st;
    if (rank < 0 || rank >= h->R)
        return fail(SEP_ERR_INVALID_ARG, "rank %d outside 0..%d", rank, h->R - 1);
    if (hidden % 128 != 0)
        return fail(SEP_ERR_INVALID_ARG, "the FP8 payload needs hidden to be a multiple of 128 (got %lld)",
                    (long long)hidden);
    if (scale != SEP_SCALE_F32 && scale != SEP_SCALE_UE8M0 && scale != SEP_SCALE_F32_POW2)
        return fail(SEP_ERR_INVALID_ARG, "the FP8 payload needs an fp32, UE8M0 or power-of-two fp32 scale");
    if (pools == nullptr || scales == nullptr || (h->T > 0 && x == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "NULL pools, scales or x");
    if (!aligned16(x))
        return fail(SEP_ERR_INVALID_ARG, "x must be 16-byte aligned");
    sep::EpDispatchParams p{};
    p.T = c.T;
    p.H = c.H;
    p.k = c.k;
    p.B = c.B;
    p.E_loc = c.E_loc;
    p.R = c.R;
    p.src_pool_row = c.src_pool_row;
    p.tile_expert = c.tile_expert;
    p.delta = c.delta;
    p.error = c.error;
    memcpy(p.pool_rows, c.pool_rows, sizeof(p.pool_rows));
    const uintptr_t scale_align = scale == SEP_SCALE_UE8M0 ? 0u : 3u;
    for (int r = 0; r < h->R; ++r) {
        if ((pool_rows[r] > 0 && (pools[r] == nullptr || scales[r] == nullptr)) || !aligned16(pools[r]) ||
            (reinterpret_cast<uintptr_t>(scales[r]) & scale_align) != 0)
            return fail(SEP_ERR_INVALID_ARG, "pools[%d] / scales[%d] must be non-NULL (if it has rows), "
                                             "16-byte and scale-size aligned", r, r);
        p.pools[r] = pools[r];
        p.scales[r] = scales[r];
        p.recv_token[r] = recv_token ? recv_token[r] : nullptr;
        p.recv_rank[r] = recv_rank ? recv_rank[r] : nullptr;
        p.recv_slot[r] = recv_slot ? recv_slot[r] : nullptr;
        if (((reinterpret_cast<uintptr_t>(p.recv_token[r]) | reinterpret_cast<uintptr_t>(p.recv_rank[r]) |
              reinterpret_cast<uintptr_t>(p.recv_slot[r])) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "receive maps of rank %d must be 4-byte aligned", r);
    }
    p.x = x;
    p.rank = rank;
    p.scale = scale;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    if (h->T == 0)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;
    const cudaError_t e = sep::launch_ep_dispatch_fp8(p, s, sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel FP8 dispatch launch");
}

sep_status sep_ep_mark_padding(int num_local_experts, int block_m, const int32_t *owner_block_offset,
                               const int32_t *owner_expert_counts, int64_t pool_rows, int32_t *recv_token,
                               int32_t *recv_rank, int32_t *recv_slot, void *stream)
{
    if (num_local_experts < 1 || num_local_experts > 1024 || block_m < 1 || block_m > 1024)
        return fail(SEP_ERR_INVALID_ARG, "need num_local_experts and block_m in 1..1024");
    if (pool_rows < 0 || pool_rows > INT32_MAX)
        return fail(SEP_ERR_INVALID_ARG, "pool_rows outside 0..2^31-1");
    if (pool_rows > 0 && (owner_block_offset == nullptr || owner_expert_counts == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "NULL owner_block_offset or owner_expert_counts");
    if (((reinterpret_cast<uintptr_t>(owner_block_offset) | reinterpret_cast<uintptr_t>(owner_expert_counts) |
          reinterpret_cast<uintptr_t>(recv_token) | reinterpret_cast<uintptr_t>(recv_rank) |
          reinterpret_cast<uintptr_t>(recv_slot)) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "arrays must be 4-byte aligned");
    int dev = -1;
    sep_status st = current_device(&dev);
    if (st != SEP_OK)
        return st;
    if ((st = preload_once(dev)) != SEP_OK)
        return st;
    sep::EpPaddingParams p{};
    p.E_loc = num_local_experts;
    p.B = block_m;
    p.block_offset = owner_block_offset;
    p.expert_counts = owner_expert_counts;
    p.pool_rows = pool_rows;
    p.recv_token = recv_token;
    p.recv_rank = recv_rank;
    p.recv_slot = recv_slot;
    const cudaError_t e = sep::launch_ep_mark_padding(p, static_cast<cudaStream_t>(stream), sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "padding launch");
}

sep_status sep_ep_plan_device(const int32_t *all_counts, int num_ranks, int num_experts, int block_m, int rank,
                              int32_t *delta, int64_t *owner_rows, int32_t *owner_block_offset,
                              int32_t *owner_expert_counts, int32_t *expert_rows, int32_t *expert_tile_offset,
                              uint32_t *error, void *stream)
{
    if (all_counts == nullptr || delta == nullptr || error == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL all_counts, delta or error");
    if (num_ranks < 1 || num_ranks > sep::kEpMaxRanks || num_experts < 1 || num_experts > 1024 ||
        num_experts % num_ranks != 0)
        return fail(SEP_ERR_INVALID_ARG, "need 1 <= num_ranks <= %d, num_experts in 1..1024 divisible by num_ranks",
                    sep::kEpMaxRanks);
    if (block_m < 1 || block_m > 1024)
        return fail(SEP_ERR_INVALID_ARG, "block_m must be in 1..1024");
    if (rank < 0 || rank >= num_ranks)
        return fail(SEP_ERR_INVALID_ARG, "rank %d outside 0..%d", rank, num_ranks - 1);
    if (((reinterpret_cast<uintptr_t>(all_counts) | reinterpret_cast<uintptr_t>(delta) |
          reinterpret_cast<uintptr_t>(owner_block_offset) | reinterpret_cast<uintptr_t>(owner_expert_counts) |
          reinterpret_cast<uintptr_t>(expert_rows) | reinterpret_cast<uintptr_t>(expert_tile_offset) |
          reinterpret_cast<uintptr_t>(error)) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(owner_rows) & 7u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "misaligned array");
    int dev = -1;
    sep_status st = current_device(&dev);
    if (st != SEP_OK || (st = preload_once(dev)) != SEP_OK)
        return st;
    sep::EpPlanParams p{};
    p.all_counts = all_counts;
    p.R = num_ranks;
    p.E = num_experts;
    p.B = block_m;
    p.rank = rank;
    p.delta = delta;
    p.owner_rows = owner_rows;
    p.owner_block_offset = owner_block_offset;
    p.owner_expert_counts = owner_expert_counts;
    p.expert_rows = expert_rows;
    p.expert_tile_offset = expert_tile_offset;
    p.error = error;
    const cudaError_t e = sep::launch_ep_plan(p, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel plan launch");
}

sep_status sep_ep_dispatch_publish(const sep_handle *h, uint32_t layout_epoch, const void *x, int64_t hidden,
                                   int rank, int payload, int scale, const int32_t *delta, void *const *pools,
                                   void *const *scales, const int64_t *pool_rows, int32_t *const *recv_token,
                                   int32_t *const *recv_rank, int32_t *const *recv_slot, uint32_t *const *tile_ready,
                                   uint32_t *const *arrival_count, const int32_t *expert_rows,
                                   const int32_t *expert_tile_offset, uint32_t dispatch_seq, uint32_t *error,
                                   void *stream)
{
    EpCommon c{};
    sep_status st = ep_common(h, layout_epoch, hidden, delta, pool_rows, error, &c);
    if (st != SEP_OK)
        return st;
    if (rank < 0 || rank >= h->R)
        return fail(SEP_ERR_INVALID_ARG, "rank %d outside 0..%d", rank, h->R - 1);
    const bool fp8 = payload == SEP_PAYLOAD_FP8_E4M3;
    if (payload != SEP_PAYLOAD_BF16 && !fp8)
        return fail(SEP_ERR_INVALID_ARG, "unknown payload %d", payload);
    if (!fp8 && scale != SEP_SCALE_NONE)
        return fail(SEP_ERR_INVALID_ARG, "bf16 payload takes SEP_SCALE_NONE");
    if (fp8 && (hidden % 128 != 0 ||
                (scale != SEP_SCALE_F32 && scale != SEP_SCALE_UE8M0 && scale != SEP_SCALE_F32_POW2)))
        return fail(SEP_ERR_INVALID_ARG, "the FP8 payload needs hidden % 128 == 0 and an fp32, UE8M0 or "
                                         "power-of-two fp32 scale");
    if (pools == nullptr || (fp8 && scales == nullptr) || (h->T > 0 && x == nullptr))
        return fail(SEP_ERR_INVALID_ARG, "NULL pools, scales or x");
    if (tile_ready == nullptr || arrival_count == nullptr || expert_rows == nullptr || expert_tile_offset == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL tile_ready, arrival_count, expert_rows or expert_tile_offset");
    if (dispatch_seq == 0)
        return fail(SEP_ERR_INVALID_ARG, "dispatch_seq must be nonzero");
    if (!aligned16(x) || ((reinterpret_cast<uintptr_t>(expert_rows) | reinterpret_cast<uintptr_t>(expert_tile_offset)) &
                          3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "x must be 16-byte aligned, expert_rows / expert_tile_offset 4-byte");
    sep::EpDispatchParams p{};
    p.T = c.T;
    p.H = c.H;
    p.k = c.k;
    p.B = c.B;
    p.E_loc = c.E_loc;
    p.R = c.R;
    p.src_pool_row = c.src_pool_row;
    p.tile_expert = c.tile_expert;
    p.delta = c.delta;
    p.error = c.error;
    memcpy(p.pool_rows, c.pool_rows, sizeof(p.pool_rows));
    const uintptr_t scale_align = scale == SEP_SCALE_UE8M0 ? 0u : 3u;
    for (int r = 0; r < h->R; ++r) {
        if ((pool_rows[r] > 0 && pools[r] == nullptr) || !aligned16(pools[r]))
            return fail(SEP_ERR_INVALID_ARG, "pools[%d] must be non-NULL (if it has rows) and 16-byte aligned", r);
        if (fp8 && ((pool_rows[r] > 0 && scales[r] == nullptr) ||
                    (reinterpret_cast<uintptr_t>(scales[r]) & scale_align) != 0))
            return fail(SEP_ERR_INVALID_ARG, "scales[%d] must be non-NULL (if it has rows) and scale-size aligned", r);
        if (tile_ready[r] == nullptr || arrival_count[r] == nullptr ||
            ((reinterpret_cast<uintptr_t>(tile_ready[r]) | reinterpret_cast<uintptr_t>(arrival_count[r])) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "tile_ready[%d] / arrival_count[%d] must be non-NULL, 4-byte aligned", r,
                        r);
        p.pools[r] = pools[r];
        p.scales[r] = fp8 ? scales[r] : nullptr;
        p.recv_token[r] = recv_token ? recv_token[r] : nullptr;
        p.recv_rank[r] = recv_rank ? recv_rank[r] : nullptr;
        p.recv_slot[r] = recv_slot ? recv_slot[r] : nullptr;
        if (((reinterpret_cast<uintptr_t>(p.recv_token[r]) | reinterpret_cast<uintptr_t>(p.recv_rank[r]) |
              reinterpret_cast<uintptr_t>(p.recv_slot[r])) & 3u) != 0)
            return fail(SEP_ERR_INVALID_ARG, "receive maps of rank %d must be 4-byte aligned", r);
        p.tile_ready[r] = tile_ready[r];
        p.arrival_count[r] = arrival_count[r];
    }
    p.x = x;
    p.rank = rank;
    p.scale = scale;
    p.expert_rows = expert_rows;
    p.expert_tile_offset = expert_tile_offset;
    p.seq = dispatch_seq;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    if (h->T == 0)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;
    const int sms = sep::device_sm_count();
    const cudaError_t e = fp8 ? sep::launch_ep_dispatch_fp8(p, s, sms) : sep::launch_ep_dispatch(p, s, sms);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel publishing dispatch launch");
}

sep_status sep_ep_consume_tiles(int num_local_experts, int block_m, const int32_t *owner_block_offset,
                                const void *pool, const int32_t *recv_token, int64_t row_bytes, int64_t pool_rows,
                                const uint32_t *tile_ready, uint32_t *arrival_count, uint32_t dispatch_seq,
                                void *dst, int num_ctas, uint64_t timeout_ns, uint32_t *status, void *stream)
{
    if (num_local_experts < 1 || num_local_experts > 1024 || block_m < 1 || block_m > 1024)
        return fail(SEP_ERR_INVALID_ARG, "need num_local_experts and block_m in 1..1024");
    if (pool_rows < 0 || pool_rows > INT32_MAX)
        return fail(SEP_ERR_INVALID_ARG, "pool_rows outside 0..2^31-1");
    if (owner_block_offset == nullptr || tile_ready == nullptr || arrival_count == nullptr || status == nullptr ||
        recv_token == nullptr || (pool_rows > 0 && (pool == nullptr || dst == nullptr)))
        return fail(SEP_ERR_INVALID_ARG, "NULL owner_block_offset, tile_ready, arrival_count, status, recv_token, "
                                         "pool or dst");
    if (row_bytes < 16 || row_bytes % 16 != 0 || row_bytes > (1LL << 20))
        return fail(SEP_ERR_INVALID_ARG, "row_bytes must be a multiple of 16 in 16..2^20");
    if (!aligned16(pool) || !aligned16(dst))
        return fail(SEP_ERR_INVALID_ARG, "pool and dst must be 16-byte aligned");
    if (((reinterpret_cast<uintptr_t>(owner_block_offset) | reinterpret_cast<uintptr_t>(tile_ready) |
          reinterpret_cast<uintptr_t>(arrival_count) | reinterpret_cast<uintptr_t>(status) |
          reinterpret_cast<uintptr_t>(recv_token)) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "arrays must be 4-byte aligned");
    if (dispatch_seq == 0)
        return fail(SEP_ERR_INVALID_ARG, "dispatch_seq must be nonzero");
    if (num_ctas < 1 || num_ctas > 1024)
        return fail(SEP_ERR_INVALID_ARG, "num_ctas must be in 1..1024");
    int dev = -1;
    sep_status st = current_device(&dev);
    if (st != SEP_OK || (st = preload_once(dev)) != SEP_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), s);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMemsetAsync (status)");
    sep::ConsumeParams p{};
    p.src = static_cast<const uint8_t *>(pool);
    p.dst = static_cast<uint8_t *>(dst);
    p.row_bytes = row_bytes;
    p.E = num_local_experts;
    p.B = block_m;
    p.expert_pool_block_offset = owner_block_offset;
    p.pool_recv_token = recv_token;
    p.tile_ready = tile_ready;
    p.seq = dispatch_seq;
    p.timeout_ns = timeout_ns ? timeout_ns : 1000000000ull;
    p.max_polls = poll_budget(p.timeout_ns);
    p.status = status;
    p.abort_flag = status;
    p.arrival_count = arrival_count;
    p.max_tiles = pool_rows / block_m;
    e = sep::launch_consume(p, num_ctas, s);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel consumer launch");
}

sep_status sep_ep_combine(const sep_handle *h, uint32_t layout_epoch, const void *const *y_pools,
                          const int64_t *pool_rows, int64_t hidden, const int32_t *delta, const float *topk_weight,
                          void *out, uint32_t *error, void *stream)
{
    EpCommon c{};
    sep_status st = ep_common(h, layout_epoch, hidden, delta, pool_rows, error, &c);
    if (st != SEP_OK)
        return st;
    sep::EpCombineParams p{};
    p.T = c.T;
    p.H = c.H;
    p.k = c.k;
    p.B = c.B;
    p.E_loc = c.E_loc;
    p.R = c.R;
    p.src_pool_row = c.src_pool_row;
    p.tile_expert = c.tile_expert;
    p.delta = c.delta;
    p.error = c.error;
    memcpy(p.pool_rows, c.pool_rows, sizeof(p.pool_rows));
    if (y_pools == nullptr || (h->T > 0 && (topk_weight == nullptr || out == nullptr)))
        return fail(SEP_ERR_INVALID_ARG, "NULL y_pools, topk_weight or out");
    if (!aligned16(out) || (reinterpret_cast<uintptr_t>(topk_weight) & 3u) != 0)
        return fail(SEP_ERR_INVALID_ARG, "out must be 16-byte aligned, topk_weight 4-byte aligned");
    for (int r = 0; r < h->R; ++r) {
        if ((pool_rows[r] > 0 && y_pools[r] == nullptr) || !aligned16(y_pools[r]))
            return fail(SEP_ERR_INVALID_ARG, "y_pools[%d] must be non-NULL (if it has rows) and 16-byte aligned", r);
        p.y_pools[r] = y_pools[r];
    }
    p.w = topk_weight;
    p.out = out;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = wait_for_release(const_cast<sep_handle *>(h), s, false)) != SEP_OK)
        return st;
    if (h->T == 0)
        return SEP_OK;
    const_cast<sep_handle *>(h)->last_stream = s;
    const cudaError_t e = sep::launch_ep_combine(p, s, sep::device_sm_count());
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, "expert-parallel combine launch");
}

sep_status sep_ep_buffer_alloc(int64_t bytes, void **ptr, void *ipc_handle)
{
    if (ptr == nullptr || ipc_handle == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL ptr or ipc_handle");
    if (bytes < 1)
        return fail(SEP_ERR_INVALID_ARG, "bytes must be positive");
    *ptr = nullptr;
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, (size_t)bytes);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaMalloc (expert-parallel buffer)");
    cudaIpcMemHandle_t hd;
    e = cudaIpcGetMemHandle(&hd, p);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "cudaIpcGetMemHandle");
    }
    static_assert(sizeof(cudaIpcMemHandle_t) == SEP_IPC_HANDLE_BYTES, "IPC handle size");
    memcpy(ipc_handle, &hd, sizeof(hd));
    *ptr = p;
    return SEP_OK;
}

sep_status sep_ep_buffer_open(const void *ipc_handle, void **ptr)
{
    if (ptr == nullptr || ipc_handle == nullptr)
        return fail(SEP_ERR_INVALID_ARG, "NULL ptr or ipc_handle");
    *ptr = nullptr;
    cudaIpcMemHandle_t hd;
    memcpy(&hd, ipc_handle, sizeof(hd));
    void *p = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&p, hd, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaIpcOpenMemHandle");
    *ptr = p;
    return SEP_OK;
}

sep_status sep_ep_buffer_close(void *ptr, int opened)
{
    if (ptr == nullptr)
        return SEP_OK;
    const cudaError_t e = opened ? cudaIpcCloseMemHandle(ptr) : cudaFree(ptr);
    return e == cudaSuccess ? SEP_OK : cuda_fail(e, opened ? "cudaIpcCloseMemHandle" : "cudaFree");
}

void sep_handle_free(sep_handle *h)
{
    if (h == nullptr)
        return;
    if (h->leased) {
        fail(SEP_ERR_HANDLE_MISMATCH, "sep_handle_free: a borrowed view is active; the handle was not freed");
        return;
    }
    int prev = -1;
    const bool switched = cudaGetDevice(&prev) == cudaSuccess && prev != h->device &&
                          cudaSetDevice(h->device) == cudaSuccess;
    // consumers of the last borrowed view still read the row map: the free
    // waits for the streams its release recorded; if that ordering cannot be
    // enqueued, the host waits for those consumers instead
    if (wait_for_release(h, h->last_stream, false) != SEP_OK) {
        for (int i = 0; i < h->n_release; ++i)
            cudaEventSynchronize(h->release_events[i]);
        fail(SEP_ERR_CUDA, "sep_handle_free: could not order the free after the view's consumers on the stream; "
                           "waited for them on the host");
    }
    h->n_release = 0;
    if (h->block != nullptr)
        cudaFreeAsync(h->block, h->last_stream);
    if (h->host_mirror != nullptr)
        mirror_pool().give(h->host_mirror);
    for (int i = 0; i < h->release_events_made; ++i)
        cudaEventDestroy(h->release_events[i]);
    if (switched)
        cudaSetDevice(prev);
    delete h;
}

}  // extern "C"
