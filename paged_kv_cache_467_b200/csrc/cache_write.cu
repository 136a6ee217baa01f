// Cache append (reshape_and_cache): each new token's K and V rows go to their
// slot, row slot % 16 of physical block slot / 16 ("Chapter 18 - KV-Cache
// Optimization Strategies", How PagedAttention Works: new tokens fill the
// current block).  One warp per (token, KV head); lanes split the head
// dimension so every row is read and written with one coalesced access.
//
// INT8 rows use the symmetric absmax quantiser of "KV Cache Engineering for
// LLM Serving", section 8, at 8 bits with one float32 scale per (token, head):
// scale = max|x| / 127 and code = clamp(rint(x / scale), -127, 127), both
// divisions IEEE round-to-nearest, rint ties-to-even.  FP8 rows store the
// E4M3 value of x / scale_h, rounded to nearest-even and saturated at 448.
#include <cuda_runtime.h>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

enum WriteKind : int { WK_COPY = 0, WK_INT8 = 1, WK_FP8 = 2 };

struct WriteParams {
  const void* key;
  const void* value;
  void* key_cache;
  void* value_cache;
  float* k_scale;
  float* v_scale;
  const int64_t* slot_mapping;
  int* err;
  long long num_tokens;
  long long num_slots;
  int n_kv;
};

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
#pragma unroll
      for (int e = 0; e < EPL; ++e)
        code[e] = scale == 0.f ? (uint8_t)0 : (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(x[e], scale), __NV_SATFINITE, __NV_E4M3);
    }
    store_bytes<EPL>(static_cast<uint8_t*>(cache) + dst_row * D + lane * EPL, code);
  }
}

template <bool BF16, int KIND, int EPL>
__global__ void __launch_bounds__(256) cache_write_kernel(const WriteParams p) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.num_tokens * p.n_kv) return;
  const long long t = warp / p.n_kv;
  const int h = (int)(warp - t * p.n_kv);
  const int64_t slot = __ldg(p.slot_mapping + t);
  if (slot == -1) return;
  if (slot < -1 || slot >= p.num_slots) {
    if (lane == 0) flag_error(p.err, DEVERR_SLOT_RANGE);
    return;
  }
  constexpr int D = EPL * 32;
  constexpr int AB = BF16 ? 2 : 4;
  const size_t src_row = (size_t)t * p.n_kv + h;
  const size_t dst_row = (size_t)slot * p.n_kv + h;
  write_row<BF16, KIND, EPL>(static_cast<const uint8_t*>(p.key) + src_row * D * AB, p.key_cache, p.k_scale, dst_row, h,
                             p.n_kv, lane);
  write_row<BF16, KIND, EPL>(static_cast<const uint8_t*>(p.value) + src_row * D * AB, p.value_cache, p.v_scale, dst_row,
                             h, p.n_kv, lane);
}

template <bool BF16, int KIND>
static pkv_status launch_kind(const WriteParams& p, int head_dim, cudaStream_t stream) {
  const long long warps = p.num_tokens * p.n_kv;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  if (blocks > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  switch (head_dim) {
    case 64: cache_write_kernel<BF16, KIND, 2><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    case 128: cache_write_kernel<BF16, KIND, 4><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    case 256: cache_write_kernel<BF16, KIND, 8><<<(unsigned)blocks, threads, 0, stream>>>(p); break;
    default: return PKV_ERR_UNSUPPORTED;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "cache_write_kernel launch");
  return PKV_OK;
}

pkv_status launch_cache_write(const void* key, const void* value, void* key_cache, void* value_cache, float* k_scale,
                              float* v_scale, const int64_t* slot_mapping, int64_t num_tokens, int n_kv, int head_dim,
                              int block_size, int64_t num_blocks, pkv_dtype act, pkv_dtype cache, int32_t* device_error,
                              cudaStream_t stream) {
  WriteParams p;
  p.key = key;
  p.value = value;
  p.key_cache = key_cache;
  p.value_cache = value_cache;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.slot_mapping = slot_mapping;
  p.err = device_error;
  p.num_tokens = num_tokens;
  p.num_slots = num_blocks * block_size;
  p.n_kv = n_kv;
  const bool bf16 = act == PKV_BF16;
  if (cache == PKV_INT8)
    return bf16 ? launch_kind<true, WK_INT8>(p, head_dim, stream) : launch_kind<false, WK_INT8>(p, head_dim, stream);
  if (cache == PKV_FP8_E4M3)
    return bf16 ? launch_kind<true, WK_FP8>(p, head_dim, stream) : launch_kind<false, WK_FP8>(p, head_dim, stream);
  return bf16 ? launch_kind<true, WK_COPY>(p, head_dim, stream) : launch_kind<false, WK_COPY>(p, head_dim, stream);
}

}  // namespace pkv
