// One K or V row of one (token, KV head) written into its cache slot by one
// warp: a bit copy, or the int8 / FP8 E4M3 quantisers.  Shared by the append
// kernel and the fused decode step.
//
// INT8 follows the symmetric absmax quantiser of "KV Cache Engineering for LLM
// Serving", section 8, at 8 bits with one float32 scale per (token, head):
// scale = max|x| / 127, code = clamp(rint(x / scale), -127, 127), divisions
// IEEE round-to-nearest, rint ties-to-even; an all-zero row stores scale 0.
// INT4 is the same quantiser at 4 bits (scale = max|x| / 7, codes -7..7), two
// codes per byte: element 2j in the low nibble of byte j, two's complement.
// FP8 stores the E4M3 (or E5M2) value of x / scale_h, nearest-even, saturated
// at the largest finite value (448, or 57344).
#pragma once

#include "pkv_device.cuh"

namespace pkv {

enum WriteKind : int { WK_COPY = 0, WK_INT8 = 1, WK_FP8 = 2, WK_E5M2 = 3, WK_INT4 = 4 };

template <int BYTES>
__device__ __forceinline__ void copy_lane(void* dst, const void* src) {
  if constexpr (BYTES == 4) {
    *static_cast<uint32_t*>(dst) = __ldg(static_cast<const uint32_t*>(src));
  } else if constexpr (BYTES == 8) {
    *static_cast<uint2*>(dst) = __ldg(static_cast<const uint2*>(src));
  } else if constexpr (BYTES == 16) {
    *static_cast<uint4*>(dst) = __ldg(static_cast<const uint4*>(src));
  } else {
    static_assert(BYTES == 32, "lane copy size");
    static_cast<uint4*>(dst)[0] = __ldg(static_cast<const uint4*>(src));
    static_cast<uint4*>(dst)[1] = __ldg(static_cast<const uint4*>(src) + 1);
  }
}

template <bool BF16, int EPL>
__device__ __forceinline__ void load_lane(float (&x)[EPL], const void* src) {
  if constexpr (BF16) {
    const uint32_t* w = static_cast<const uint32_t*>(src);
#pragma unroll
    for (int k = 0; k < EPL / 2; ++k) {
      const uint32_t v = __ldg(w + k);
      x[2 * k] = __uint_as_float(v << 16);
      x[2 * k + 1] = __uint_as_float(v & 0xFFFF0000u);
    }
  } else {
    const float* f = static_cast<const float*>(src);
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[e] = __ldg(f + e);
  }
}

template <int EPL>
__device__ __forceinline__ void store_bytes(void* dst, const uint8_t (&b)[EPL]) {
  if constexpr (EPL == 2) {
    *static_cast<uint16_t*>(dst) = (uint16_t)(b[0] | (b[1] << 8));
  } else {
    uint32_t w[EPL / 4];
#pragma unroll
    for (int k = 0; k < EPL / 4; ++k)
      w[k] = (uint32_t)b[4 * k] | ((uint32_t)b[4 * k + 1] << 8) | ((uint32_t)b[4 * k + 2] << 16) |
             ((uint32_t)b[4 * k + 3] << 24);
    if constexpr (EPL == 4) *static_cast<uint32_t*>(dst) = w[0];
    else *static_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  }
}

template <bool BF16, int KIND, int EPL>
__device__ __forceinline__ void write_row(const void* src_row, void* cache, float* scales, size_t dst_row, int h,
                                          int n_kv, int lane) {
  constexpr int D = EPL * 32;
  constexpr int AB = BF16 ? 2 : 4;  // bytes per input value
  if constexpr (KIND == WK_COPY) {
    copy_lane<EPL * AB>(static_cast<uint8_t*>(cache) + dst_row * D * AB + lane * EPL * AB,
                        static_cast<const uint8_t*>(src_row) + lane * EPL * AB);
  } else {
    float x[EPL];
    load_lane<BF16, EPL>(x, static_cast<const uint8_t*>(src_row) + lane * EPL * AB);
    if constexpr (KIND == WK_INT4) {
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
      amax = warp_max(amax);
      const float scale = __fdiv_rn(amax, 7.0f);
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        float q = scale == 0.f ? 0.f : rintf(__fdiv_rn(x[e], scale));
        q = fminf(fmaxf(q, -7.f), 7.f);
        packed |= ((uint32_t)(int)q & 0xFu) << (4 * e);
      }
      if (lane == 0) scales[dst_row] = scale;
      uint8_t* dst = static_cast<uint8_t*>(cache) + dst_row * (D / 2) + lane * (EPL / 2);
      if constexpr (EPL == 2) *dst = (uint8_t)packed;
      else if constexpr (EPL == 4) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
      else *reinterpret_cast<uint32_t*>(dst) = packed;
      return;
    }
    uint8_t code[EPL];
    if constexpr (KIND == WK_INT8) {
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
      amax = warp_max(amax);
      const float scale = __fdiv_rn(amax, 127.0f);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        float q = scale == 0.f ? 0.f : rintf(__fdiv_rn(x[e], scale));
        q = fminf(fmaxf(q, -127.f), 127.f);
        code[e] = (uint8_t)(int8_t)(int)q;
      }
      if (lane == 0) scales[dst_row] = scale;  // dst_row = slot * n_kv + h
    } else {
      const float scale = __ldg(scales + h);
      constexpr __nv_fp8_interpretation_t fmt = KIND == WK_E5M2 ? __NV_E5M2 : __NV_E4M3;
#pragma unroll
      for (int e = 0; e < EPL; ++e)
        code[e] = scale == 0.f ? (uint8_t)0 : (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(x[e], scale), __NV_SATFINITE, fmt);
    }
    store_bytes<EPL>(static_cast<uint8_t*>(cache) + dst_row * D + lane * EPL, code);
  }
}

}  // namespace pkv
