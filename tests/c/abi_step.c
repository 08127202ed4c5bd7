/*
 * A plain C caller of the library: one layout -> dispatch -> combine step
 * through include/sep.h, with no Python in between.
 *
 * usage: abi_step <dir> T k E R B H
 *   reads  <dir>/topk_idx.bin (int32 [T][k]), x.bin (bf16 bits [T][H]),
 *          topk_weight.bin (float32 [T][k])
 *   writes <dir>/src_pool_row.bin (int32 [T][k]), recv.bin (bf16 bits [P][H]),
 *          out.bin (bf16 bits [T][H]), sizes.txt ("P NT")
 * Exits non-zero, with the library's message on stderr, if any call fails.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "sep.h"

static void *read_file(const char *dir, const char *name, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    void *buf = malloc(bytes ? bytes : 1);
    if (f == NULL || buf == NULL || fread(buf, 1, bytes, f) != bytes) {
        fprintf(stderr, "cannot read %s\n", path);
        exit(2);
    }
    fclose(f);
    return buf;
}

static void write_file(const char *dir, const char *name, const void *buf, size_t bytes)
{
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (f == NULL || fwrite(buf, 1, bytes, f) != bytes) {
        fprintf(stderr, "cannot write %s\n", path);
        exit(2);
    }
    fclose(f);
}

#define CHECK_SEP(call)                                                                   \
    do {                                                                                  \
        sep_status st_ = (call);                                                          \
        if (st_ != SEP_OK) {                                                              \
            fprintf(stderr, "%s: %s: %s\n", #call, sep_status_string(st_), sep_last_error()); \
            return 1;                                                                     \
        }                                                                                 \
    } while (0)

#define CHECK_CUDA(call)                                                           \
    do {                                                                           \
        cudaError_t e_ = (call);                                                   \
        if (e_ != cudaSuccess) {                                                   \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));            \
            return 1;                                                              \
        }                                                                          \
    } while (0)

int main(int argc, char **argv)
{
    if (argc != 8) {
        fprintf(stderr, "usage: %s dir T k E R B H\n", argv[0]);
        return 2;
    }
    const char *dir = argv[1];
    const int64_t T = atoll(argv[2]);
    const int k = atoi(argv[3]), E = atoi(argv[4]), R = atoi(argv[5]), B = atoi(argv[6]);
    const int64_t H = atoll(argv[7]);
    if (sep_abi_version() != SEP_ABI_VERSION) {
        fprintf(stderr, "ABI version mismatch\n");
        return 1;
    }
    int32_t *idx_h = read_file(dir, "topk_idx.bin", (size_t)(T * k * 4));
    uint16_t *x_h = read_file(dir, "x.bin", (size_t)(T * H * 2));
    float *w_h = read_file(dir, "topk_weight.bin", (size_t)(T * k * 4));

    cudaStream_t s;
    CHECK_CUDA(cudaStreamCreate(&s));
    void *idx_d, *x_d, *w_d, *out_d;
    CHECK_CUDA(cudaMalloc(&idx_d, (size_t)(T * k * 4 + 16)));
    CHECK_CUDA(cudaMalloc(&x_d, (size_t)(T * H * 2 + 16)));
    CHECK_CUDA(cudaMalloc(&w_d, (size_t)(T * k * 4 + 16)));
    CHECK_CUDA(cudaMalloc(&out_d, (size_t)(T * H * 2 + 16)));
    CHECK_CUDA(cudaMemcpy(idx_d, idx_h, (size_t)(T * k * 4), cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(x_d, x_h, (size_t)(T * H * 2), cudaMemcpyHostToDevice));
    CHECK_CUDA(cudaMemcpy(w_d, w_h, (size_t)(T * k * 4), cudaMemcpyHostToDevice));

    sep_handle *h = NULL;
    CHECK_SEP(sep_layout(idx_d, 4, T, k, E, R, B, SEP_LAYOUT_SYNC_COUNTS, s, &h));
    sep_layout_info info;
    CHECK_SEP(sep_handle_info(h, &info));
    const int64_t P = info.num_pool_rows;
    void *recv_d;
    CHECK_CUDA(cudaMalloc(&recv_d, (size_t)((P > 0 ? P : 1) * H * 2)));
    CHECK_SEP(sep_dispatch(h, x_d, H, SEP_PAYLOAD_BF16, SEP_SCALE_NONE, recv_d, NULL, P, NULL, 0, 0, s));
    CHECK_SEP(sep_combine(h, info.epoch, recv_d, H, P, (const float *)w_d, out_d, s));
    CHECK_CUDA(cudaStreamSynchronize(s));

    int32_t *spr_h = malloc((size_t)(T * k * 4 + 4));
    uint16_t *recv_h = malloc((size_t)((P > 0 ? P : 1) * H * 2));
    uint16_t *out_h = malloc((size_t)(T * H * 2 + 2));
    CHECK_CUDA(cudaMemcpy(spr_h, info.src_pool_row, (size_t)(T * k * 4), cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(recv_h, recv_d, (size_t)(P * H * 2), cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(out_h, out_d, (size_t)(T * H * 2), cudaMemcpyDeviceToHost));
    write_file(dir, "src_pool_row.bin", spr_h, (size_t)(T * k * 4));
    write_file(dir, "recv.bin", recv_h, (size_t)(P * H * 2));
    write_file(dir, "out.bin", out_h, (size_t)(T * H * 2));
    char sizes[64];
    int n = snprintf(sizes, sizeof sizes, "%lld %lld\n", (long long)P, (long long)info.num_tiles);
    write_file(dir, "sizes.txt", sizes, (size_t)n);

    sep_handle_free(h);
    cudaFree(recv_d);
    cudaFree(out_d);
    cudaFree(w_d);
    cudaFree(x_d);
    cudaFree(idx_d);
    cudaStreamDestroy(s);
    free(idx_h);
    free(x_h);
    free(w_h);
    free(spr_h);
    free(recv_h);
    free(out_h);
    return 0;
}
