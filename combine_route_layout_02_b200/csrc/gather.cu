// Indexed consumer of a receive view (PR #769 "Add opt-in borrowed receive
// storage for compact BF16 dispatch", "Description": an indexed consumer reads
// the borrowed slab through the row map instead of a copied pool).
//
// dst[r] = slab[indexed ? row_indices[r] : r] for every pool row r whose
// row_indices[r] >= 0.  One warp per row; each lane keeps eight 16-byte loads
// in flight.  Padding rows are neither read nor written.
#include "sep_internal.cuh"

namespace sep {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(kWarps * 32) gather_rows_kernel(GatherParams p)
{
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t vecs = p.row_bytes / 16;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < p.rows; r += nwarps) {
        const int idx = __ldg(p.row_indices + r);
        if (idx < 0)
            continue;                                    // padding: never read
        const uint4 *src = reinterpret_cast<const uint4 *>(p.slab) + (p.indexed ? (int64_t)idx : r) * vecs;
        uint4 *dst = reinterpret_cast<uint4 *>(p.dst) + r * vecs;
        for (int64_t v0 = lane; v0 < vecs; v0 += 32 * kUnroll) {
            uint4 buf[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + u * 32;
                buf[u] = v < vecs ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t v = v0 + u * 32;
                if (v < vecs)
                    dst[v] = buf[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_gather(const GatherParams &p, cudaStream_t s, int)
{
    if (p.rows <= 0)
        return cudaSuccess;
    return launch_kernel(gather_rows_kernel, dim3((unsigned)((p.rows + kWarps - 1) / kWarps)), dim3(kWarps * 32),
                         0, s, p);
}

cudaError_t preload_gather_kernels()
{
    cudaFuncAttributes a;
    return cudaFuncGetAttributes(&a, reinterpret_cast<const void *>(gather_rows_kernel));
}

}  // namespace sep
