/*
 * CPU oracle for MoE dispatch + combine.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, single-threaded C that states what the dispatch/combine path
 * computes.  Only the tests, the smoke check and the benchmark's CPU baseline
 * may load it; the product path never does.  It shares no code, header, table
 * or helper with the CUDA library.
 *
 * Sources (page title, section):
 *  - StreamEP README, "Streaming dispatch in one paragraph": the expert-major,
 *    BLOCK_M-padded pool; expert e's block starts at row
 *    expert_pool_block_offset[e] * tile_m; every slot belongs to one expert and
 *    one tile; pool_arrival_target per tile; padding rows carry
 *    pool_recv_token < 0 and are never read.
 *  - "DeepEP MoE dispatch/combine" (charlestar blog), section "一轮 DeepEP 数据流"
 *    (one round of data flow): count assignments by destination/expert,
 *    compute layout and offsets, move hidden states, recv_x grouped by local
 *    expert; combine restores source token / top-k slot and reduces the
 *    routing-weighted expert outputs.
 *  - same blog, "Imbalance 决定 buffer 与尾延迟": per-owner load L_r = sum of n_e
 *    over the owner's experts.
 *  - same blog, "Router 权重什么时候应用": y_t = sum_j p_{t,j} o_{t,j}.
 *  - same blog, "FP8 Dispatch 减少的是 payload": N_a = N_t * k assignments.
 *  - "DeepEP Low-Latency Dispatch and Combine Kernels for Inference Decoding",
 *    "FP8 and Quantization Support": float8_e4m3fn payload with fp32 or UE8M0
 *    scales (use_fp8 / use_ue8m0 / round_scale flags).
 *  - OCP 8-bit floating point format, E4M3 ("fn": no infinities, one NaN
 *    mantissa pattern, max finite 448, exponent bias 7, subnormals m * 2^-9).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  1. Slots inside an expert are filled in ascending assignment order
 *     a = t*k + j (a stable counting sort).
 *  2. Padding rows are not written; pool_recv_token = pool_recv_slot = -1 there.
 *  3. topk_idx < 0 means "no assignment"; topk_idx >= E is an error: it is
 *     reported and the entry is treated as no assignment.
 *  4. Duplicate experts inside one token's top-k are distinct assignments.
 *  5. Weights are applied only in combine; dispatch copies rows unscaled.
 *  6. FP8: amax over each 128-channel group; fp32 scale s = amax / 448
 *     (s = 1 when amax == 0); UE8M0 scale s = 2^E* with E* the smallest integer
 *     such that 448 * 2^E* >= amax (E* = 0 when amax == 0), clamped to
 *     [-127, 127]; "round_scale" stores that power of two as fp32.  Codes are
 *     e4m3(x / s), rounded to nearest even and saturated to +-448.
 *  7. Scales are row-major [pool_rows, H/128], aligned with pool rows.
 *  8. Combine accumulates in fp32, ascending j, separate multiply and add,
 *     starting from +0, then rounds once to bf16 (nearest even).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

enum { OR_OK = 0, OR_BAD_EXPERT_ID = 1, OR_CAPACITY = 2, OR_INVALID = 3 };
enum { OR_SCALE_F32 = 1, OR_SCALE_UE8M0 = 2, OR_SCALE_F32_POW2 = 3 };

/* ------------------------------------------------------------------ bf16 */

float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN stays a quiet NaN). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xffffu;
    /* round up when the dropped half is above one half, or exactly one half
     * and the kept part is odd */
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))
        upper += 1u;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------ e4m3 */

/* Value of an e4m3 ("fn") code; NaN for S.1111.111. */
float oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xf, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* Round a non-negative double to an integer, ties to even. */
static double rne_int(double q)
{
    double f = floor(q);
    double d = q - f;
    if (d > 0.5)
        return f + 1.0;
    if (d < 0.5)
        return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* fp32 -> e4m3 code, round to nearest even, saturating to +-448 (finite input). */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (isnan(v))
        return 0x7f;
    if (a >= 448.0)
        return sign | 0x7e;                       /* E=15, m=6: 448 */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: spacing 2^-9; n == 8 lands on the smallest normal,
         * whose code (E=1, m=0) is also 8 */
        double n = rne_int(a * 512.0);
        return sign | (uint8_t)n;
    }
    int e;
    frexp(a, &e);                                 /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                       /* a in [2^e, 2^(e+1)) */
    double n = rne_int(ldexp(a, 3 - e));          /* a / 2^(e-3), in [8, 16] */
    if (n == 16.0) {
        n = 8.0;
        e += 1;
    }
    /* a < 448 keeps (e, n) at or below (8, 14), i.e. at most 448 */
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* Smallest integer E with 448 * 2^E >= amax, clamped to [-127, 127]; 0 for amax == 0. */
int oracle_ue8m0_exponent(float amax)
{
    double a = (double)amax;
    if (!(a > 0.0))
        return 0;
    int e;
    frexp(a / 448.0, &e);                         /* first guess, then fix exactly */
    while (ldexp(448.0, e) < a)
        e++;
    while (ldexp(448.0, e - 1) >= a)
        e--;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    return e;
}

/* ---------------------------------------------------------------- layout */

/*
 * Layout of one routing.
 *   topk_idx          [T*k]   expert id per assignment (int64 values)
 * outputs (caller-allocated):
 *   expert_counts     [E]     n_e
 *   owner_counts      [R]     L_r = sum of n_e over owner r's experts
 *   owner_token_counts[R]     tokens with at least one assignment on owner r
 *   is_token_in_rank  [T*R]   1 if token t has an assignment on owner r (may be NULL)
 *   expert_pool_block_offset [E+1]  tile offset of expert e; [E] = total tiles NT
 *   owner_pool_row_offset    [R+1]  first pool row of owner r; [R] = pool rows P
 *   tile_expert, pool_arrival_target [cap_rows / B]
 *   src_pool_row      [T*k]   pool row of assignment (t,j), -1 if none
 *   pool_recv_token, pool_recv_slot [cap_rows]  source (t, j) of each pool row, -1 for padding
 *   num_pool_rows, num_tiles  P and NT
 * Returns OR_OK, OR_BAD_EXPERT_ID (outputs still complete, bad ids skipped),
 * OR_CAPACITY (P > cap_rows; nothing past the counts is written) or OR_INVALID.
 */
int oracle_layout(const int64_t *topk_idx, int64_t T, int k, int E, int R, int B,
                  int32_t *expert_counts, int32_t *owner_counts, int32_t *owner_token_counts,
                  uint8_t *is_token_in_rank, int32_t *expert_pool_block_offset,
                  int32_t *owner_pool_row_offset, int32_t *tile_expert,
                  int32_t *pool_arrival_target, int32_t *src_pool_row,
                  int32_t *pool_recv_token, int32_t *pool_recv_slot, int64_t cap_rows,
                  int64_t *num_pool_rows, int64_t *num_tiles)
{
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0 || B < 1)
        return OR_INVALID;
    const int E_loc = E / R;
    const int64_t Na = T * (int64_t)k;
    int bad = 0;

    /* step 1: count assignments per expert, ascending a */
    for (int e = 0; e < E; e++)
        expert_counts[e] = 0;
    for (int64_t a = 0; a < Na; a++) {
        int64_t e = topk_idx[a];
        if (e < 0)
            continue;
        if (e >= E) {
            bad = 1;
            continue;
        }
        expert_counts[e]++;
    }

    /* per-owner assignment load */
    for (int r = 0; r < R; r++) {
        owner_counts[r] = 0;
        for (int e = r * E_loc; e < (r + 1) * E_loc; e++)
            owner_counts[r] += expert_counts[e];
    }

    /* per-owner token membership (a token counts once per owner) */
    for (int r = 0; r < R; r++)
        owner_token_counts[r] = 0;
    for (int64_t t = 0; t < T; t++) {
        for (int r = 0; r < R; r++) {
            int in = 0;
            for (int j = 0; j < k; j++) {
                int64_t e = topk_idx[t * k + j];
                if (e >= 0 && e < E && e / E_loc == r)
                    in = 1;
            }
            if (is_token_in_rank)
                is_token_in_rank[t * R + r] = (uint8_t)in;
            owner_token_counts[r] += in;
        }
    }

    /* step 2: tiles per expert and their exclusive prefix sum */
    expert_pool_block_offset[0] = 0;
    for (int e = 0; e < E; e++) {
        int32_t tiles = (expert_counts[e] + B - 1) / B;
        expert_pool_block_offset[e + 1] = expert_pool_block_offset[e] + tiles;
    }
    const int64_t NT = expert_pool_block_offset[E];
    const int64_t P = NT * B;
    *num_tiles = NT;
    *num_pool_rows = P;
    for (int r = 0; r <= R; r++)
        owner_pool_row_offset[r] = (int32_t)((int64_t)expert_pool_block_offset[r * E_loc] * B);
    if (P > cap_rows)
        return OR_CAPACITY;

    for (int e = 0; e < E; e++) {
        for (int32_t i = expert_pool_block_offset[e]; i < expert_pool_block_offset[e + 1]; i++) {
            int32_t left = expert_counts[e] - (i - expert_pool_block_offset[e]) * B;
            tile_expert[i] = e;
            pool_arrival_target[i] = left < B ? left : B;
        }
    }

    /* step 3: stable slots, ascending a, one cursor per expert */
    for (int64_t row = 0; row < P; row++) {
        pool_recv_token[row] = -1;
        pool_recv_slot[row] = -1;
    }
    for (int e = 0; e < E; e++)
        expert_counts[e] = 0;                     /* reused as cursors */
    for (int64_t a = 0; a < Na; a++) {
        int64_t e = topk_idx[a];
        if (e < 0 || e >= E) {
            src_pool_row[a] = -1;
            continue;
        }
        int64_t row = (int64_t)expert_pool_block_offset[e] * B + expert_counts[e];
        expert_counts[e]++;
        src_pool_row[a] = (int32_t)row;
        pool_recv_token[row] = (int32_t)(a / k);
        pool_recv_slot[row] = (int32_t)(a % k);
    }
    /* the cursors end at n_e: the counts are restored */
    return bad ? OR_BAD_EXPERT_ID : OR_OK;
}

/* -------------------------------------------------------------- dispatch */

/* recv[src_pool_row[a]] = x[a / k] for every valid assignment; rows are H bf16. */
void oracle_dispatch_bf16(const uint16_t *x, int64_t T, int64_t H, int k,
                          const int32_t *src_pool_row, uint16_t *recv)
{
    for (int64_t t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int32_t row = src_pool_row[t * k + j];
            if (row < 0)
                continue;
            for (int64_t h = 0; h < H; h++)
                recv[(int64_t)row * H + h] = x[t * H + h];
        }
}

/*
 * Quantise one token row (H bf16, H % 128 == 0) to e4m3 codes and one scale per
 * 128-channel group.  scale_kind: OR_SCALE_F32 (fp32 amax/448),
 * OR_SCALE_UE8M0 (byte E*+127), OR_SCALE_F32_POW2 (fp32 2^E*).
 * codes [H]; scales_f32 [H/128] or scales_u8 [H/128] depending on the kind.
 */
void oracle_quant_row(const uint16_t *xrow, int64_t H, int scale_kind, uint8_t *codes,
                      float *scales_f32, uint8_t *scales_u8)
{
    for (int64_t g = 0; g < H / 128; g++) {
        const uint16_t *xg = xrow + g * 128;
        float amax = 0.0f;
        for (int i = 0; i < 128; i++) {
            float a = fabsf(oracle_bf16_to_f32(xg[i]));
            if (a > amax)
                amax = a;
        }
        float s;
        if (scale_kind == OR_SCALE_F32) {
            s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
            scales_f32[g] = s;
        } else {
            int E = oracle_ue8m0_exponent(amax);
            s = (float)ldexp(1.0, E);
            if (scale_kind == OR_SCALE_UE8M0)
                scales_u8[g] = (uint8_t)(E + 127);
            else
                scales_f32[g] = s;
        }
        for (int i = 0; i < 128; i++)
            codes[g * 128 + i] = oracle_e4m3_encode(oracle_bf16_to_f32(xg[i]) / s);
    }
}

/* FP8 dispatch: quantise x[t] once per token, write its codes and scales into
 * every pool row the token was assigned to. */
void oracle_dispatch_fp8(const uint16_t *x, int64_t T, int64_t H, int k,
                         const int32_t *src_pool_row, int scale_kind, uint8_t *recv,
                         float *recv_scales_f32, uint8_t *recv_scales_u8,
                         uint8_t *codes_tmp, float *sf_tmp, uint8_t *su_tmp)
{
    const int64_t G = H / 128;
    for (int64_t t = 0; t < T; t++) {
        oracle_quant_row(x + t * H, H, scale_kind, codes_tmp, sf_tmp, su_tmp);
        for (int j = 0; j < k; j++) {
            int32_t row = src_pool_row[t * k + j];
            if (row < 0)
                continue;
            memcpy(recv + (int64_t)row * H, codes_tmp, (size_t)H);
            if (scale_kind == OR_SCALE_UE8M0)
                memcpy(recv_scales_u8 + (int64_t)row * G, su_tmp, (size_t)G);
            else
                memcpy(recv_scales_f32 + (int64_t)row * G, sf_tmp, (size_t)G * sizeof(float));
        }
    }
}

/* Dequantise pool rows back to fp32: x_hat = decode(code) * s. */
void oracle_dequant_rows(const uint8_t *codes, int64_t rows, int64_t H, int scale_kind,
                         const float *scales_f32, const uint8_t *scales_u8, float *out)
{
    const int64_t G = H / 128;
    for (int64_t r = 0; r < rows; r++)
        for (int64_t h = 0; h < H; h++) {
            float s = (scale_kind == OR_SCALE_UE8M0)
                          ? (float)ldexp(1.0, (int)scales_u8[r * G + h / 128] - 127)
                          : scales_f32[r * G + h / 128];
            out[r * H + h] = oracle_e4m3_decode(codes[r * H + h]) * s;
        }
}

/* --------------------------------------------------------------- combine */

/* out[t] = bf16( sum_j w[t,j] * y[src_pool_row[t,j]] ), fp32, ascending j. */
void oracle_combine(const uint16_t *y_pool, int64_t T, int64_t H, int k,
                    const int32_t *src_pool_row, const float *topk_weight, uint16_t *out)
{
    for (int64_t t = 0; t < T; t++)
        for (int64_t h = 0; h < H; h++) {
            float acc = 0.0f;
            for (int j = 0; j < k; j++) {
                int32_t row = src_pool_row[t * k + j];
                if (row < 0)
                    continue;
                float prod = topk_weight[t * k + j] * oracle_bf16_to_f32(y_pool[(int64_t)row * H + h]);
                acc = acc + prod;
            }
            out[t * H + h] = oracle_f32_to_bf16(acc);
        }
}

/* ------------------------------------------------------------- backward */

/*
 * Backward of combine ("StreamEP" README, "What's in the box": dispatch_grads,
 * the backward symmetry of combine).  With out[t] = sum_j w[t,j] * y[row(t,j)]:
 *   grad_y[row(t,j)] = bf16( w[t,j] * grad_out[t] )      (fp32 product, one rounding)
 *   grad_w[t,j]      = sum_h grad_out[t,h] * y[row(t,j),h] (fp64 here: the exact sum
 *                                                            up to one final rounding)
 * Masked assignments get no row and grad_w = 0.  grad_w may be NULL (then y may be too).
 */
void oracle_dispatch_grads(const uint16_t *grad_out, int64_t T, int64_t H, int k, const int32_t *src_pool_row,
                           const float *topk_weight, const uint16_t *y_pool, uint16_t *grad_y, double *grad_w)
{
    for (int64_t t = 0; t < T; t++)
        for (int j = 0; j < k; j++) {
            int32_t row = src_pool_row[t * k + j];
            float w = topk_weight[t * k + j];
            double dot = 0.0;
            if (row >= 0) {
                for (int64_t h = 0; h < H; h++) {
                    float g = oracle_bf16_to_f32(grad_out[t * H + h]);
                    float prod = w * g;
                    grad_y[(int64_t)row * H + h] = oracle_f32_to_bf16(prod);
                    if (grad_w)
                        dot += (double)g * (double)oracle_bf16_to_f32(y_pool[(int64_t)row * H + h]);
                }
            }
            if (grad_w)
                grad_w[t * k + j] = dot;
        }
}

/*
 * Backward of dispatch (combine_grads): with recv[row(t,j)] = x[t],
 *   grad_x[t] = bf16( sum over valid j, ascending, of grad_recv[row(t,j)] )
 * in fp32 with one rounding at the end: the combine of oracle_combine with
 * every weight equal to 1.
 */
void oracle_combine_grads(const uint16_t *grad_recv, int64_t T, int64_t H, int k, const int32_t *src_pool_row,
                          uint16_t *grad_x)
{
    for (int64_t t = 0; t < T; t++)
        for (int64_t h = 0; h < H; h++) {
            float acc = 0.0f;
            for (int j = 0; j < k; j++) {
                int32_t row = src_pool_row[t * k + j];
                if (row < 0)
                    continue;
                acc = acc + oracle_bf16_to_f32(grad_recv[(int64_t)row * H + h]);
            }
            grad_x[t * H + h] = oracle_f32_to_bf16(acc);
        }
}
