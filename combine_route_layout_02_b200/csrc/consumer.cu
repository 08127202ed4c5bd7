// Reference consumer of a streaming dispatch (StreamEP README, "Streaming
// dispatch in one paragraph": a consumer kernel on another stream spins on
// the acquire-load of tile_ready[tile] >= dispatch_seq and proceeds; padding
// rows are predicated out by pool_recv_token >= 0).
//
// Persistent CTAs walk the tiles in the order a token-major dispatch finishes
// them: tile i of every expert before tile i+1 of any.  Position n of that
// order belongs to CTA n % gridDim.x.  Thread 0 waits (acquire load, bounded by
// %globaltimer and a poll budget, with nanosleep back-off), the CTA barrier
// passes the acquired view to the other threads, and the CTA copies the tile's
// valid rows with L2-coherent loads, eight 16-byte loads in flight per lane.  When a wait gives up, status[0] becomes
// SEP_ERR_TIMEOUT; every CTA then stops waiting and counts its remaining tiles
// in status[1].  No wait is unbounded.
//
// With per-token stamps the consumer stands in for the expert compute that
// feeds a gated combine (identity experts: the copy is the expert output):
// once a tile's rows are stored, each row adds one arrival to its token's
// counter and the arrival that completes the token release-stores done_seq
// into y_done[token] (StreamEP README, opening section: y_done_per_token).
#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxExperts = 1024;
constexpr int kCopyUnroll = 8;       // 16-byte loads in flight per lane while copying a row

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *ptr)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_acquire_sys(const unsigned *ptr)
{
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_time_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 1 once tile_ready[tile] has reached seq; 0 if this or another CTA gave up.
template <bool SYS>
__device__ int wait_tile(const ConsumeParams &p, int tile)
{
    const uint64_t t0 = global_time_ns();
    for (uint32_t polls = 0;; ++polls) {
        const unsigned v = SYS ? ld_acquire_sys(p.tile_ready + tile) : ld_acquire_gpu(p.tile_ready + tile);
        if ((int32_t)(v - p.seq) >= 0)
            return 1;
        if (*reinterpret_cast<volatile const uint32_t *>(p.abort_flag) != 0u)
            return 0;
        if (polls >= p.max_polls || global_time_ns() - t0 > p.timeout_ns) {
            atomicCAS(p.abort_flag, 0u, (uint32_t)SEP_ERR_TIMEOUT);
            return 0;
        }
        __nanosleep(256);
    }
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

// After the CTA has copied a tile: one arrival per valid row on its token's
// counter; the arrival that completes the token (all its valid assignments)
// release-stores done_seq into y_done[token].
__device__ void stamp_tokens(const ConsumeParams &p, int tile)
{
    for (int r = threadIdx.x; r < p.B; r += blockDim.x) {
        const int tok = __ldg(p.pool_recv_token + (int64_t)tile * p.B + r);
        if (tok < 0)
            continue;
        unsigned need = 0;
        for (int j = 0; j < p.k; ++j)
            need += __ldg(p.src_pool_row + (int64_t)tok * p.k + j) >= 0 ? 1u : 0u;
        if (atom_add_acq_rel_gpu(p.token_arrivals + tok, 1u) + 1u == need)
            st_release_gpu(p.y_done + tok, p.done_seq);
    }
}

// SYS: an expert-parallel owner's pool, written by other GPUs' dispatches.
template <bool SYS>
__global__ void __launch_bounds__(kThreads) consume_tiles_kernel(ConsumeParams p)
{
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_go;
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x)
        s_off[e] = p.expert_pool_block_offset[e];
    __syncthreads();
    int max_tau = 0;
    for (int e = 0; e < p.E; ++e)
        max_tau = max(max_tau, s_off[e + 1] - s_off[e]);

    const int64_t vecs = p.row_bytes / 16;
    long long pos = 0;
    for (int i = 0; i < max_tau; ++i) {
        for (int e = 0; e < p.E; ++e) {
            if (s_off[e + 1] - s_off[e] <= i)
                continue;
            if (pos++ % gridDim.x != blockIdx.x)
                continue;
            const int tile = s_off[e] + i;
            if (SYS && tile >= p.max_tiles) {            // a plan larger than the owner's arrays
                if (threadIdx.x == 0) {
                    atomicCAS(p.status, 0u, (uint32_t)SEP_ERR_CAPACITY);
                    atomicAdd(p.status + 1, 1u);
                }
                continue;
            }
            if (threadIdx.x == 0)
                s_go = wait_tile<SYS>(p, tile);
            __syncthreads();
            const int go = s_go;
            if (go) {
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
                for (int r = warp; r < p.B; r += kThreads / 32) {
                    const int64_t row = (int64_t)tile * p.B + r;
                    const int tok = SYS ? __ldcg(p.pool_recv_token + row) : __ldg(p.pool_recv_token + row);
                    if (tok < 0)
                        continue;                        // padding: never read
                    const uint4 *src = reinterpret_cast<const uint4 *>(p.src) + row * vecs;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.dst) + row * vecs;
                    for (int64_t v0 = lane; v0 < vecs; v0 += 32 * kCopyUnroll) {
                        uint4 buf[kCopyUnroll];
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u) {
                            const int64_t v = v0 + u * 32;
                            buf[u] = v < vecs ? __ldcg(src + v) : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                        for (int u = 0; u < kCopyUnroll; ++u) {
                            const int64_t v = v0 + u * 32;
                            if (v < vecs)
                                dst[v] = buf[u];
                        }
                    }
                }
                if (p.y_done)
                    __threadfence();                     // this thread's rows before the CTA barrier
            } else if (threadIdx.x == 0) {
                atomicAdd(p.status + 1, 1u);
            }
            __syncthreads();
            if (go && p.y_done)
                stamp_tokens(p, tile);
            if (SYS && go && threadIdx.x == 0)
                p.arrival_count[tile] = 0u;              // complete: no more arrivals this step
        }
    }
}

}  // namespace

cudaError_t launch_consume(const ConsumeParams &p, int num_ctas, cudaStream_t s)
{
    count_launch();
    if (p.arrival_count != nullptr)
        consume_tiles_kernel<true><<<num_ctas, kThreads, 0, s>>>(p);
    else
        consume_tiles_kernel<false><<<num_ctas, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t preload_consumer_kernels()
{
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(consume_tiles_kernel<false>));
    if (e == cudaSuccess)
        e = cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(consume_tiles_kernel<true>));
    return e;
}

}  // namespace sep
