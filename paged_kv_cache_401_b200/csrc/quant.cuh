// Per-row quantisation of a new K or V row by one warp, shared by the cache
// write and the fused append+decode so both store identical codes.
//
// "KV Cache 深度解析" §四 (fp16 -> fp8 E4M3 with a per-token scale to hold
// outliers); k1-blog "KV Cache 量化" (INT8 halves the cache like FP8).  For a
// row x of D elements (one token, one kv head):
//   FP8 : a = max|x|; scale = a / 448 (IEEE fp32 division);
//         code = E4M3(x / scale) (IEEE division, round to nearest even, saturating)
//   INT8: a = max|x|; scale = a / 127;
//         code = clamp(round_to_nearest_even(x / scale), -127, 127)
//   a == 0 -> scale 0 and every code 0.
// Lane l holds elements [l * D/32, (l + 1) * D/32) of the row.
#pragma once

#include "common.cuh"

namespace pkv {

// Load a lane's D/32 consecutive source elements (fp32 or bf16) widened to fp32.
template <int D>
__device__ __forceinline__ void load_row_part(const void* row, int32_t src_dtype, int32_t lane,
                                              float* x) {
    constexpr int kPer = D / 32;
    if (src_dtype == KV_F32) {
        const float* p = static_cast<const float*>(row) + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; ++e) x[e] = p[e];
    } else {
        const uint16_t* p = static_cast<const uint16_t*>(row) + lane * kPer;
#pragma unroll
        for (int e = 0; e < kPer; ++e) x[e] = __uint_as_float(static_cast<uint32_t>(p[e]) << 16);
    }
}

// Quantise the row held by the warp; returns this lane's D/32 codes packed
// little-endian (first element in the low byte) and the row scale in *scale.
template <int KV_T, int D>
__device__ __forceinline__ uint32_t quantize_row_warp(const float* x, float* scale) {
    constexpr int kPer = D / 32;
    constexpr float kMaxCode = KV_T == KV_INT8 ? 127.0f : 448.0f;
    static_assert(KV_T == KV_FP8_E4M3 || KV_T == KV_INT8, "8-bit codes");
    static_assert(kPer == 2 || kPer == 4, "head_dim 64 or 128");
    float a = 0.0f;
#pragma unroll
    for (int e = 0; e < kPer; ++e) a = fmaxf(a, fabsf(x[e]));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, m));
    const float s = __fdiv_rn(a, kMaxCode);
    uint32_t codes = 0;
#pragma unroll
    for (int e = 0; e < kPer; e += 2) {
        uint32_t pair = 0;
        if (a != 0.0f) {
            if constexpr (KV_T == KV_INT8) {
                const int c0 = max(-127, min(127, __float2int_rn(__fdiv_rn(x[e], s))));
                const int c1 = max(-127, min(127, __float2int_rn(__fdiv_rn(x[e + 1], s))));
                pair = (static_cast<uint32_t>(c0) & 0xffu) | ((static_cast<uint32_t>(c1) & 0xffu) << 8);
            } else {
                pair = float2_to_e4m3x2(__fdiv_rn(x[e], s), __fdiv_rn(x[e + 1], s));
            }
        }
        codes |= pair << (8 * e);
    }
    *scale = (a == 0.0f) ? 0.0f : s;
    return codes;
}

// INT4 ("llm-inference-optimization" notes §四: the printed 4-bit routine,
// asymmetric with a zero point), in IEEE fp32, on a group of values:
//   hi = max x, lo = min x, scale = (hi - lo) / 15, zero = rint(-lo / scale),
//   code = clamp(rint(x / scale) + zero, 0, 15); value = (code - zero) * scale.
// A constant group (where the routine would divide by zero) is stored exactly:
// scale = |lo|, zero = -1 / +1 / 0 for lo > 0 / < 0 / == 0, every code 0.
// The group is a row (INT4 pools), or for KIVI pools one channel of a full
// block's keys and one value row.
__device__ __forceinline__ bool int4_params(float hi, float lo, float* scale, float* zero) {
    if (hi == lo) {
        *scale = fabsf(lo);
        *zero = lo > 0.0f ? -1.0f : (lo < 0.0f ? 1.0f : 0.0f);
        return false;  // every code 0
    }
    const float s = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
    *scale = s;
    *zero = rintf(__fdiv_rn(-lo, s));
    return true;
}

__device__ __forceinline__ uint32_t int4_code(float x, float s, float z) {
    return static_cast<uint32_t>(fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(x, s)), z), 0.0f), 15.0f));
}

// One row held by the warp (lane l: elements 4l .. 4l+3 of a 128-element row).
// Returns the lane's 4 codes packed two per byte, its first element in the low
// nibble of the low byte.
template <int D>
__device__ __forceinline__ uint32_t quantize_row_int4_warp(const float* x, float* scale,
                                                           float* zero) {
    constexpr int kPer = D / 32;
    static_assert(kPer == 4, "4-bit rows: head_dim 128");
    float hi = x[0], lo = x[0];
#pragma unroll
    for (int e = 1; e < kPer; ++e) {
        hi = fmaxf(hi, x[e]);
        lo = fminf(lo, x[e]);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) {
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, m));
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, m));
    }
    float s, z;
    uint32_t codes = 0;
    if (int4_params(hi, lo, &s, &z)) {
#pragma unroll
        for (int e = 0; e < kPer; ++e) codes |= int4_code(x[e], s, z) << (4 * e);
    }
    *scale = s;
    *zero = z;
    return codes;
}

// One group of 16 values held by one thread (a KIVI key channel over a block);
// codes[t] for value t.
__device__ __forceinline__ void quantize_group16_int4(const float* x, uint32_t* codes,
                                                      float* scale, float* zero) {
    float hi = x[0], lo = x[0];
#pragma unroll
    for (int t = 1; t < 16; ++t) {
        hi = fmaxf(hi, x[t]);
        lo = fminf(lo, x[t]);
    }
    float s, z;
    const bool any = int4_params(hi, lo, &s, &z);
#pragma unroll
    for (int t = 0; t < 16; ++t) codes[t] = any ? int4_code(x[t], s, z) : 0u;
    *scale = s;
    *zero = z;
}

// Store a lane's packed codes (D/32 bytes) at dst.
template <int D>
__device__ __forceinline__ void store_codes(uint8_t* dst, uint32_t codes) {
    if constexpr (D / 32 == 4) {
        *reinterpret_cast<uint32_t*>(dst) = codes;
    } else {
        *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(codes);
    }
}

}  // namespace pkv
