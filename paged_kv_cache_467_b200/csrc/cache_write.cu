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
#include "cache_row.cuh"
#include "pkv_device.cuh"

namespace pkv {

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
  if (cache == PKV_FP8_E5M2)
    return bf16 ? launch_kind<true, WK_E5M2>(p, head_dim, stream) : launch_kind<false, WK_E5M2>(p, head_dim, stream);
  if (cache == PKV_INT4)
    return bf16 ? launch_kind<true, WK_INT4>(p, head_dim, stream) : launch_kind<false, WK_INT4>(p, head_dim, stream);
  return bf16 ? launch_kind<true, WK_COPY>(p, head_dim, stream) : launch_kind<false, WK_COPY>(p, head_dim, stream);
}

}  // namespace pkv
