// Paged decode attention for an F32 cache on CUDA cores (no TF32), so float32
// inputs keep float32 accuracy.  One warp per (sequence, query head) walks the
// sequence's tokens in logical order through its block table ("KV-cache
// overview" page t13_4, block-table paragraph), keeping a running max / sum
// softmax in registers; lanes split the head dimension.
#include <cuda_runtime.h>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

struct F32Params {
  float* out;
  const float* query;
  const float* key_cache;
  const float* value_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* lse_out;
  int* err;
  // fused decode step: token L-1 comes from these rows and is stored to the cache
  const float* new_key;
  const float* new_value;
  long long num_blocks;
  int max_blocks_per_seq, cap_len, num_seqs, n_q, n_kv, G;
  int window, sinks;  // attend to [0, sinks) and [L - window, L) only; window 0 = every position
  const int32_t* pages;  // Quest: [num_seqs, n_kv, k_pages] logical pages to read (ascending, -1 past the count)
  int k_pages;
  float sm_scale;
};

template <int EPL>  // head_dim / 32 values per lane
__global__ void __launch_bounds__(128) decode_f32_kernel(const F32Params p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.num_seqs * p.n_q) return;
  const int s = warp / p.n_q, h = warp - s * p.n_q;
  const int kv = h / p.G;
  constexpr int D = EPL * 32;
  int L = __ldg(p.context_lens + s);
  if (L < 0 || L > p.cap_len) {
    if (h == 0) flag_error(p.err, DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : p.cap_len;
  }
  float q[EPL], acc[EPL];
  const float* qrow = p.query + ((size_t)s * p.n_q + h) * D + lane * EPL;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    q[e] = __ldg(qrow + e);
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int32_t* table = p.block_tables + (size_t)s * p.max_blocks_per_seq;
  // attended positions: [0, s_eff) then [lo_w, L) (one run when they touch)
  int s_eff = L, lo_w = L;
  if (p.window > 0 && L > p.window) {
    s_eff = min(p.sinks, L);
    lo_w = max(L - p.window, s_eff);
  }
  const int32_t* plist = p.pages ? p.pages + ((size_t)s * p.n_kv + kv) * p.k_pages : nullptr;
  const int plen = min(p.k_pages, (L + kBlockSize - 1) / kBlockSize);  // entries read at most
  int pi = 0;  // next listed page
  for (int pos = 0; pos < L; ++pos) {
    if (plist) {
      if (pos % kBlockSize == 0) {
        // next listed page; the list ends at k_pages entries or its first -1;
        // a page past the sequence (or out of order) is a range error
        int pg = -1;
        while (pi < plen) {
          pg = __ldg(plist + pi++);
          if (pg < 0) break;
          if ((long long)pg * kBlockSize >= pos && (long long)pg * kBlockSize < L) break;
          if (h % p.G == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
          pg = -1;
        }
        if (pg < 0) break;
        pos = pg * kBlockSize;
      }
    } else {
      if (pos == s_eff) pos = lo_w;
    }
    if (pos >= L) break;
    const int blk = __ldg(table + pos / kBlockSize);
    if (blk < 0 || (long long)blk >= p.num_blocks) {
      flag_error(p.err, DEVERR_BLOCK_RANGE);
      continue;
    }
    const size_t row = (((size_t)blk * kBlockSize + pos % kBlockSize) * p.n_kv + kv) * D + lane * EPL;
    const float* krow = p.key_cache + row;
    const float* vrow = p.value_cache + row;
    if (p.new_key && pos == L - 1) {
      // the appended token: read from the new rows; the group's first query
      // head's warp stores them into the cache (no warp reads them back there)
      const size_t nrow = ((size_t)s * p.n_kv + kv) * D + lane * EPL;
      krow = p.new_key + nrow;
      vrow = p.new_value + nrow;
      if (h % p.G == 0) {
        float* kc = const_cast<float*>(p.key_cache) + row;
        float* vc = const_cast<float*>(p.value_cache) + row;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          kc[e] = __ldg(krow + e);
          vc[e] = __ldg(vrow + e);
        }
      }
    }
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dot = fmaf(q[e], __ldg(krow + e), dot);
    dot = warp_sum(dot) * p.sm_scale;
    const float mn = fmaxf(m, dot);
    const float alpha = expf(m - mn);
    const float w = expf(dot - mn);
    l = l * alpha + w;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, __ldg(vrow + e), acc[e] * alpha);
    m = mn;
  }
  float* orow = p.out + ((size_t)s * p.n_q + h) * D + lane * EPL;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) orow[e] = acc[e] * inv;
  if (p.lse_out && lane == 0) p.lse_out[(size_t)s * p.n_q + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

pkv_status launch_decode_f32(const DecodeShape& sh, const TcArgs& a, cudaStream_t stream) {
  F32Params p;
  p.out = static_cast<float*>(a.out);
  p.query = static_cast<const float*>(a.query);
  p.key_cache = static_cast<const float*>(a.key_cache);
  p.value_cache = static_cast<const float*>(a.value_cache);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.lse_out = a.lse_out;
  p.err = a.device_error;
  p.new_key = static_cast<const float*>(a.new_key);
  p.new_value = static_cast<const float*>(a.new_value);
  p.num_blocks = a.num_blocks;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  const int64_t cap = (int64_t)a.max_blocks_per_seq * kBlockSize;
  p.cap_len = (int)(a.max_context_len < cap ? a.max_context_len : cap);
  p.num_seqs = sh.num_seqs;
  p.n_q = sh.n_q;
  p.n_kv = sh.n_kv;
  p.G = sh.n_q / sh.n_kv;
  p.sm_scale = a.sm_scale;
  p.window = a.window;
  p.sinks = a.sinks;
  p.pages = a.pages;
  p.k_pages = a.k_pages;
  const long long warps = (long long)sh.num_seqs * sh.n_q;
  const int threads = 128;
  const unsigned blocks = (unsigned)((warps * 32 + threads - 1) / threads);
  switch (sh.head_dim / 32) {
    case 1: decode_f32_kernel<1><<<blocks, threads, 0, stream>>>(p); break;
    case 2: decode_f32_kernel<2><<<blocks, threads, 0, stream>>>(p); break;
    case 3: decode_f32_kernel<3><<<blocks, threads, 0, stream>>>(p); break;
    case 4: decode_f32_kernel<4><<<blocks, threads, 0, stream>>>(p); break;
    case 5: decode_f32_kernel<5><<<blocks, threads, 0, stream>>>(p); break;
    case 6: decode_f32_kernel<6><<<blocks, threads, 0, stream>>>(p); break;
    case 7: decode_f32_kernel<7><<<blocks, threads, 0, stream>>>(p); break;
    case 8: decode_f32_kernel<8><<<blocks, threads, 0, stream>>>(p); break;
    default: return PKV_ERR_UNSUPPORTED;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode_f32_kernel launch");
  return PKV_OK;
}

}  // namespace pkv
