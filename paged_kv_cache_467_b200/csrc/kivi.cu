// 2-bit KIVI cache: block quantiser, residual pass (append + residual
// attention), host launchers.
//
// What it computes ("KV Cache Engineering for LLM Serving", section 8,
// Quantization: KIVI groups keys by channel and values by token, 2-bit cache;
// "Chapter 18 - KV-Cache Optimization Strategies", KV-Cache Quantization
// methods table): with the section's symmetric absmax quantiser at 2 bits
// (largest code 1, scale = max |x|, codes rint(x / scale) in {-1, 0, 1}),
//  * a key group is one channel of one KV head over the 16 tokens of a block,
//  * a value group is the 128 values of one token of one KV head.
// A channel group needs all 16 tokens, so only full blocks live in the pool;
// the rows of a sequence's partial last block stay in a BF16 residual
// [num_seqs, 16, n_kv, 128] until the row that fills the block arrives, and
// the block is then quantised at once.
//
// How (B200 design, not from the pages): one CTA of 128 threads per (sequence,
// KV head).  The residual pass appends the step's new row, quantises the block
// it completes (thread = channel for K, warp = token for V), and attends the
// group's query heads over the BF16 residual rows, one warp per head.  Its
// result per (KV head, query row) is the normalised output and base-2 lse,
// which the tensor-core decode over the quantised full blocks (queued behind
// it with programmatic serialisation) starts from, so a decode step is the
// residual pass, the decode and the merge of split units.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

namespace {

constexpr int kKiviD = 128;
constexpr int kKiviThreads = 128;

// Pools head-major inside a block, so a (block, KV head) tile is contiguous:
// 512 bytes of codes per pool, 512 of K scales, 64 of V scales.
struct KiviQuantTarget {
  uint8_t* key_cache;    // [num_blocks, n_kv, 16, 32]
  uint8_t* value_cache;
  float* k_scale;        // [num_blocks, n_kv, 128]
  float* v_scale;        // [num_blocks, n_kv, 16]
  int n_kv;
};

// Quantises the 16 rows of one (block, KV head): src_k / src_v point at row 0's
// head vector and rows are row_stride elements apart.  All 128 threads call.
__device__ void kivi_quantize_rows(const __nv_bfloat16* src_k, const __nv_bfloat16* src_v, size_t row_stride,
                                   long long phys, int kv, const KiviQuantTarget& t) {
  const int i = threadIdx.x, warp = i >> 5, lane = i & 31;
  // K: thread i is channel i; its scale is the channel's max |x| over the block
  float x[kBlockSize];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < kBlockSize; ++r) {
    x[r] = __bfloat162float(src_k[r * row_stride + i]);
    amax = fmaxf(amax, fabsf(x[r]));
  }
  t.k_scale[((size_t)phys * t.n_kv + kv) * kKiviD + i] = amax;
#pragma unroll
  for (int r = 0; r < kBlockSize; ++r) {
    int c = amax > 0.f ? (int)rintf(__fdiv_rn(x[r], amax)) : 0;
    c = max(-1, min(1, c));
    // element 4j + m of a row sits in bits [2m, 2m+1] of byte j: lanes 4j .. 4j+3 combine
    uint32_t bits = (uint32_t)(c & 3) << (2 * (i & 3));
    bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
    bits |= __shfl_xor_sync(0xffffffffu, bits, 2);
    if ((i & 3) == 0) t.key_cache[(((size_t)phys * t.n_kv + kv) * kBlockSize + r) * (kKiviD / 4) + (i >> 2)] = (uint8_t)bits;
  }
  // V: warp w takes tokens w, w+4, ...; lane l holds dims 4l .. 4l+3 (one code byte)
  for (int r = warp; r < kBlockSize; r += kKiviThreads / 32) {
    const uint2 w = *reinterpret_cast<const uint2*>(src_v + r * row_stride + 4 * lane);
    const float y[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u), __uint_as_float(w.y << 16),
                        __uint_as_float(w.y & 0xFFFF0000u)};
    const float vmax = warp_max(fmaxf(fmaxf(fabsf(y[0]), fabsf(y[1])), fmaxf(fabsf(y[2]), fabsf(y[3]))));
    uint32_t byte = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int c = vmax > 0.f ? (int)rintf(__fdiv_rn(y[e], vmax)) : 0;
      c = max(-1, min(1, c));
      byte |= (uint32_t)(c & 3) << (2 * e);
    }
    const size_t row = ((size_t)phys * t.n_kv + kv) * kBlockSize + r;
    t.value_cache[row * (kKiviD / 4) + lane] = (uint8_t)byte;
    if (lane == 0) t.v_scale[row] = vmax;
  }
}

struct ResidualParams {
  const __nv_bfloat16* query;      // [num_seqs, n_q, 128]
  const __nv_bfloat16* new_key;    // [num_seqs, n_kv, 128] or null
  const __nv_bfloat16* new_value;
  __nv_bfloat16* res_k;            // [num_seqs, 16, n_kv, 128]
  __nv_bfloat16* res_v;
  KiviQuantTarget q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* pre_o;    // [n_kv][num_seqs * G][128]
  float* pre_lse;  // [n_kv][num_seqs * G], base 2
  int* err;
  long long num_blocks;
  int max_blocks_per_seq, cap_len, num_seqs, n_q, n_kv, G;
  float scale_log2;
};

__global__ void __launch_bounds__(kKiviThreads) kivi_residual_kernel(const ResidualParams p) {
  grid_launch_dependents();  // the decode's prologue may start; it waits for this grid before reading
  constexpr int D = kKiviD;
  const int s = blockIdx.x / p.n_kv, kv = blockIdx.x - s * p.n_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L = __ldg(p.context_lens + s);
  if (L < 0 || L > p.cap_len) {
    if (tid == 0 && kv == 0) flag_error(p.err, DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : p.cap_len;
  }
  const size_t rstride = (size_t)p.n_kv * D;
  __nv_bfloat16* rk = p.res_k + (size_t)s * kBlockSize * rstride + (size_t)kv * D;
  __nv_bfloat16* rv = p.res_v + (size_t)s * kBlockSize * rstride + (size_t)kv * D;

  if (p.new_key && L > 0) {
    // the step's row is token L-1: residual row (L-1) % 16
    const int pos = L - 1, r = pos % kBlockSize;
    const size_t src = ((size_t)s * p.n_kv + kv) * D + tid;
    rk[r * rstride + tid] = p.new_key[src];
    rv[r * rstride + tid] = p.new_value[src];
    __syncthreads();
    if (r == kBlockSize - 1) {  // the block is full: quantise it into the pool
      const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + pos / kBlockSize);
      if (phys < 0 || (long long)phys >= p.num_blocks) {
        if (tid == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
      } else {
        kivi_quantize_rows(rk, rv, rstride, phys, kv, p.q);
      }
    }
  }

  // Attention of the group's query heads over the residual rows [L - L % 16, L):
  // base-2 scores z = sm_scale * log2(e) * <q, k>, m = max z, o = sum 2^(z-m) v / l,
  // lse = m + log2 l (no rows: o = 0, lse = -inf).
  const int r_att = L % kBlockSize;
  for (int h = warp; h < p.G; h += kKiviThreads / 32) {
    const size_t qrow = (size_t)s * p.n_q + (size_t)kv * p.G + h;
    const uint2 qw = *reinterpret_cast<const uint2*>(p.query + qrow * D + 4 * lane);
    const float q[4] = {__uint_as_float(qw.x << 16), __uint_as_float(qw.x & 0xFFFF0000u),
                        __uint_as_float(qw.y << 16), __uint_as_float(qw.y & 0xFFFF0000u)};
    float z[kBlockSize];
    float m = -INFINITY;
#pragma unroll
    for (int t = 0; t < kBlockSize; ++t) {
      z[t] = -INFINITY;
      if (t < r_att) {
        const uint2 kw = *reinterpret_cast<const uint2*>(rk + t * rstride + 4 * lane);
        float d = q[0] * __uint_as_float(kw.x << 16) + q[1] * __uint_as_float(kw.x & 0xFFFF0000u) +
                  q[2] * __uint_as_float(kw.y << 16) + q[3] * __uint_as_float(kw.y & 0xFFFF0000u);
        z[t] = warp_sum(d) * p.scale_log2;
        m = fmaxf(m, z[t]);
      }
    }
    float l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int t = 0; t < kBlockSize; ++t) {
      if (t < r_att) {
        const float w = exp2f(z[t] - m);
        const uint2 vw = *reinterpret_cast<const uint2*>(rv + t * rstride + 4 * lane);
        l += w;
        o[0] += w * __uint_as_float(vw.x << 16);
        o[1] += w * __uint_as_float(vw.x & 0xFFFF0000u);
        o[2] += w * __uint_as_float(vw.y << 16);
        o[3] += w * __uint_as_float(vw.y & 0xFFFF0000u);
      }
    }
    const float inv = r_att > 0 ? 1.f / l : 0.f;
    const size_t prow = (size_t)kv * ((size_t)p.num_seqs * p.G) + (size_t)s * p.G + h;
    reinterpret_cast<float4*>(p.pre_o + prow * D)[lane] = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    if (lane == 0) p.pre_lse[prow] = r_att > 0 ? m + log2f(l) : -INFINITY;
  }
}

__global__ void __launch_bounds__(kKiviThreads)
    kivi_quantize_blocks_kernel(const __nv_bfloat16* key_rows, const __nv_bfloat16* value_rows,
                                const int32_t* dst_blocks, long long n, KiviQuantTarget t, long long num_blocks,
                                int* err) {
  const long long b = blockIdx.x / t.n_kv;
  const int kv = (int)(blockIdx.x - b * t.n_kv);
  const int phys = __ldg(dst_blocks + b);
  if (phys == -1) return;
  if (phys < 0 || (long long)phys >= num_blocks) {
    if (threadIdx.x == 0 && kv == 0) flag_error(err, DEVERR_BLOCK_RANGE);
    return;
  }
  const size_t rstride = (size_t)t.n_kv * kKiviD;
  const size_t base = (size_t)b * kBlockSize * rstride + (size_t)kv * kKiviD;
  kivi_quantize_rows(key_rows + base, value_rows + base, rstride, phys, kv, t);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t kivi_state_bytes(int num_seqs, int n_q) {
  const size_t rows = (size_t)num_seqs * n_q;  // over all KV heads: n_kv * (num_seqs * G)
  return align256(rows * kKiviD * 4) + align256(rows * 4);
}

pkv_status launch_kivi_residual(const KiviArgs& a, void* state_ws, PrefixState* state, cudaStream_t stream) {
  ResidualParams p;
  p.query = static_cast<const __nv_bfloat16*>(a.query);
  p.new_key = static_cast<const __nv_bfloat16*>(a.new_key);
  p.new_value = static_cast<const __nv_bfloat16*>(a.new_value);
  p.res_k = static_cast<__nv_bfloat16*>(a.residual_k);
  p.res_v = static_cast<__nv_bfloat16*>(a.residual_v);
  p.q = KiviQuantTarget{static_cast<uint8_t*>(a.key_cache), static_cast<uint8_t*>(a.value_cache), a.k_scale,
                        a.v_scale, a.n_kv};
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  const size_t rows = (size_t)a.num_seqs * a.n_q;
  p.pre_o = static_cast<float*>(state_ws);
  p.pre_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(state_ws) + align256(rows * kKiviD * 4));
  p.err = a.device_error;
  p.num_blocks = a.num_blocks;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.cap_len = a.cap_len;
  p.num_seqs = a.num_seqs;
  p.n_q = a.n_q;
  p.n_kv = a.n_kv;
  p.G = a.n_q / a.n_kv;
  p.scale_log2 = (float)((double)a.sm_scale * 1.4426950408889634);
  kivi_residual_kernel<<<(unsigned)((size_t)a.num_seqs * a.n_kv), kKiviThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kivi_residual_kernel launch");
  state->o = p.pre_o;
  state->lse = p.pre_lse;
  state->splits = 1;
  state->rows = a.num_seqs * p.G;
  return PKV_OK;
}

pkv_status launch_kivi_quantize_blocks(const void* key_rows, const void* value_rows, const int32_t* dst_blocks,
                                       int64_t n, void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                                       int n_kv, int64_t num_blocks, int32_t* device_error, cudaStream_t stream) {
  KiviQuantTarget t{static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), k_scale, v_scale, n_kv};
  kivi_quantize_blocks_kernel<<<(unsigned)(n * n_kv), kKiviThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(key_rows), static_cast<const __nv_bfloat16*>(value_rows), dst_blocks, n, t,
      num_blocks, device_error);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kivi_quantize_blocks_kernel launch");
  return PKV_OK;
}

}  // namespace pkv
