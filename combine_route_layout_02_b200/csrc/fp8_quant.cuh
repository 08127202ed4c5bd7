// FP8 e4m3 quantisation of a 128-channel group held by 8 lanes (16 channels
// each), shared by the single-GPU and the expert-parallel dispatch kernels.
//
// Per group ("DeepEP Low-Latency Dispatch and Combine Kernels for Inference
// Decoding", "FP8 and Quantization Support"): amax = max |x| by xor shuffles
// over the 8 lanes; SEP_SCALE_F32: s = amax / 448 (IEEE division; 1 when
// amax = 0), codes e4m3(x / s); UE8M0 and power-of-two fp32: s = 2^E with E
// the smallest integer such that 448 * 2^E >= amax, codes e4m3(x * 2^-E)
// (exact, the same as the division).  Codes round to nearest even and
// saturate to +-448 (the hardware e4m3x2 conversion).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "sep_internal.cuh"

namespace sep {

// Smallest E with 448 * 2^E >= amax (0 for amax == 0), clamped to [-127, 127].
// amax = m * 2^x with m in [1, 2): 448 = 1.75 * 2^8, so E = x - 8 when
// m <= 1.75 (mantissa field <= 0x600000) and x - 7 otherwise.  Every subnormal
// amax is below 448 * 2^-134 and clamps to -127.
__device__ __forceinline__ int ue8m0_exponent(float amax)
{
    const uint32_t u = __float_as_uint(amax);
    if (u == 0u)
        return 0;
    const int ex = (int)(u >> 23);
    if (ex == 0)
        return -127;
    const int e = ex - 127 - 8 + ((u & 0x7fffffu) > 0x600000u ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^e as fp32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float *f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Quantise this lane's 16 channels; every lane of the warp must call it (the
// amax shuffles).  Returns the 16 codes and the group's scale (fp32 value and
// UE8M0 exponent).
template <int SCALE>
__device__ __forceinline__ uint4 quantize_lane16(const float *f, float &scale_f, int &expo)
{
    float amax = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q)
        amax = fmaxf(amax, fabsf(f[q]));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(kFullMask, amax, 4));

    float inv = 1.f;
    scale_f = 1.f;
    expo = 0;
    if (SCALE == SEP_SCALE_F32) {
        scale_f = amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
    } else {
        expo = ue8m0_exponent(amax);
        scale_f = exp2_int(expo);
        inv = exp2_int(-expo);                           // exact: x * 2^-E == x / 2^E
    }
    uint32_t packed[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float a[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
            a[r] = SCALE == SEP_SCALE_F32 ? __fdiv_rn(f[4 * q + r], scale_f) : __fmul_rn(f[4 * q + r], inv);
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a[0], a[1]), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a[2], a[3]), __NV_SATFINITE, __NV_E4M3);
        packed[q] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return make_uint4(packed[0], packed[1], packed[2], packed[3]);
}

}  // namespace sep
