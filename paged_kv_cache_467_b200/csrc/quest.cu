// Quest: query-aware page selection ("KV Cache Engineering for LLM Serving",
// section 7, Query-aware sparse reads).  A page is one cache block.  Each page
// keeps the element-wise minimum and maximum of its keys; a query scores a page
// by sum_i max(q_i * min_i, q_i * max_i), an upper bound of q . k for every key
// of the page, and only the best pages are read by the decode.
//
// Readings: pages are chosen per (sequence, KV head) by the largest score of
// the group's query heads; the k best pages are kept, ties toward the lower
// page index; the last page covers only rows below the sequence length.
//
//  * quest_summaries_kernel: warp per (block of a sequence, KV head); lanes
//    split the head dimension, rows are folded with min / max.  Summaries are
//    stored in the cache dtype (min / max of bf16 values are bf16 values).
//  * quest_score_tc_kernel (BF16): the page scores of a group as a tensor-core
//    product, pages streamed through shared memory; quest_score_simt_kernel
//    (F32 and wide groups): a warp per page.  Both write every page's score.
//  * quest_topk_kernel: CTA per (sequence, KV head); a 4-pass radix select over
//    order-preserving float keys finds the k-th score; an index-order
//    compaction keeps ties lowest-index first and writes the pages ascending.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

struct QuestSumParams {
  const void* key_cache;
  void* page_min;
  void* page_max;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int* err;
  long long num_blocks;
  int max_blocks_per_seq, num_seqs, n_kv;
  int last_page_only;  // one CTA per sequence, refreshing the page that holds token L-1
};

template <bool BF16, int EPL>
__device__ __forceinline__ void load_vals(float (&x)[EPL], const void* base, size_t elem_off) {
  if constexpr (BF16) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(base) + elem_off);
#pragma unroll
    for (int k = 0; k < EPL / 2; ++k) {
      const uint32_t v = __ldg(w + k);
      x[2 * k] = __uint_as_float(v << 16);
      x[2 * k + 1] = __uint_as_float(v & 0xFFFF0000u);
    }
  } else {
    const float* f = static_cast<const float*>(base) + elem_off;
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[e] = __ldg(f + e);
  }
}

template <bool BF16, int EPL>
__device__ __forceinline__ void store_vals(void* base, size_t elem_off, const float (&x)[EPL]) {
  if constexpr (BF16) {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(base) + elem_off;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = __float2bfloat16_rn(x[e]);  // exact: x holds bf16 values
  } else {
    float* o = static_cast<float*>(base) + elem_off;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = x[e];
  }
}

template <bool BF16, int EPL>
__global__ void __launch_bounds__(256) quest_summaries_kernel(const QuestSumParams p) {
  constexpr int D = EPL * 32;
  int s, j;
  const int L0 = __ldg(p.context_lens + (p.last_page_only ? blockIdx.x : blockIdx.x / p.max_blocks_per_seq));
  if (p.last_page_only) {
    s = blockIdx.x;
    j = (L0 - 1) / kBlockSize;
  } else {
    s = blockIdx.x / p.max_blocks_per_seq;
    j = blockIdx.x - s * p.max_blocks_per_seq;
  }
  const int cap = p.max_blocks_per_seq * kBlockSize;
  const int L = L0 < 0 ? 0 : min(L0, cap);
  if ((L0 < 0 || L0 > cap) && threadIdx.x == 0 && (p.last_page_only || j == 0)) flag_error(p.err, DEVERR_CONTEXT_LEN);
  if (L <= 0 || j < 0 || L <= j * kBlockSize || j >= p.max_blocks_per_seq) return;
  const int rows = min(kBlockSize, L - j * kBlockSize);
  const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + j);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (phys < 0 || (long long)phys >= p.num_blocks) {
    if (threadIdx.x == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
    return;
  }
  for (int h = warp; h < p.n_kv; h += blockDim.x >> 5) {
    float mn[EPL], mx[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      mn[e] = INFINITY;
      mx[e] = -INFINITY;
    }
    // rows in batches of 8 independent loads, then folded
#pragma unroll
    for (int r0 = 0; r0 < kBlockSize; r0 += 8) {
      float x[8][EPL];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r0 + r < rows)
          load_vals<BF16, EPL>(x[r], p.key_cache, (((size_t)phys * kBlockSize + r0 + r) * p.n_kv + h) * D + lane * EPL);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r0 + r < rows) {
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            mn[e] = fminf(mn[e], x[r][e]);
            mx[e] = fmaxf(mx[e], x[r][e]);
          }
        }
      }
    }
    const size_t off = ((size_t)phys * p.n_kv + h) * D + lane * EPL;
    store_vals<BF16, EPL>(p.page_min, off, mn);
    store_vals<BF16, EPL>(p.page_max, off, mx);
  }
}

pkv_status launch_quest_summaries(const void* key_cache, void* page_min, void* page_max, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int n_kv,
                                  int head_dim, int64_t num_blocks, pkv_dtype cache, int last_page_only,
                                  int32_t* device_error, cudaStream_t stream) {
  QuestSumParams p{key_cache, page_min, page_max, block_tables, context_lens, device_error, num_blocks,
                   max_blocks_per_seq, num_seqs, n_kv, last_page_only ? 1 : 0};
  const long long grid = last_page_only ? (long long)num_seqs : (long long)num_seqs * max_blocks_per_seq;
  if (grid == 0) return PKV_OK;
  if (grid > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  const bool bf16 = cache == PKV_BF16;
  switch (head_dim) {
    case 64:
      if (bf16) quest_summaries_kernel<true, 2><<<(unsigned)grid, 256, 0, stream>>>(p);
      else quest_summaries_kernel<false, 2><<<(unsigned)grid, 256, 0, stream>>>(p);
      break;
    case 128:
      if (bf16) quest_summaries_kernel<true, 4><<<(unsigned)grid, 256, 0, stream>>>(p);
      else quest_summaries_kernel<false, 4><<<(unsigned)grid, 256, 0, stream>>>(p);
      break;
    default:
      return PKV_ERR_UNSUPPORTED;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quest_summaries_kernel launch");
  return PKV_OK;
}

struct QuestSelParams {
  const void* query;
  const void* page_min;
  const void* page_max;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* selected;  // [num_seqs, n_kv, k_pages], ascending logical pages, -1 past the count
  float* scores;      // [num_seqs, n_kv, max_pages]: every page's score (scratch of the selection too)
  int* err;
  long long num_blocks;
  int max_blocks_per_seq, cap_len, num_seqs, n_q, n_kv, G, k_pages, max_pages;
  int act_bf16;
};

__device__ __forceinline__ int clamp_len(const QuestSelParams& p, int s) {
  const int L = __ldg(p.context_lens + s);
  return L < 0 ? 0 : min(L, p.cap_len);
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA of one int per thread; total returned too.
__device__ int cta_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < nw ? sh[lane] : 0;
    int incl = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < nw) sh[lane] = incl - w;
    if (lane == 31) sh[32] = incl;
  }
  __syncthreads();
  const int res = sh[warp] + x - v;
  *total = sh[32];
  __syncthreads();
  return res;
}

// ---------------------------------------------------------------- scoring
// CUDA-core scorer (F32 caches, F32 queries, groups of more than 8 query
// heads): CTA per (sequence, KV head); a warp scores a page with lanes over
// the head dimension, taking the largest score of the group's query heads.
template <bool CBF16, int EPL>
__global__ void __launch_bounds__(256) quest_score_simt_kernel(const QuestSelParams p) {
  constexpr int D = EPL * 32;
  extern __shared__ float qs[];  // [G][D] query rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int s = blockIdx.x / p.n_kv, kv = blockIdx.x - s * p.n_kv;
  const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
  if (P == 0) return;
  for (int i = tid; i < p.G * D; i += blockDim.x) {
    const size_t qi = ((size_t)s * p.n_q + kv * p.G + i / D) * D + i % D;
    qs[i] = p.act_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.query)[qi])
                       : static_cast<const float*>(p.query)[qi];
  }
  __syncthreads();
  float* out = p.scores + ((size_t)s * p.n_kv + kv) * p.max_pages;
  for (int j = warp; j < P; j += nwarps) {
    const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + j);
    float best = -INFINITY;
    if (phys < 0 || (long long)phys >= p.num_blocks) {
      if (lane == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
    } else {
      float mn[EPL], mx[EPL];
      const size_t off = ((size_t)phys * p.n_kv + kv) * D + lane * EPL;
      load_vals<CBF16, EPL>(mn, p.page_min, off);
      load_vals<CBF16, EPL>(mx, p.page_max, off);
      for (int h = 0; h < p.G; ++h) {
        const float* q = qs + h * D + lane * EPL;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) part += fmaxf(q[e] * mn[e], q[e] * mx[e]);
        best = fmaxf(best, warp_sum(part));
      }
    }
    if (lane == 0) out[j] = best;
  }
}

// Tensor-core scorer (BF16 queries and summaries, at most 8 query heads per
// KV head).  For a page, sum_i max(q_i * min_i, q_i * max_i) equals, term by
// term, sum_i (q+_i * max_i + q-_i * min_i) with q+ = max(q, 0) and
// q- = min(q, 0), so the scores of 16 pages for the group's query heads are one
// 16 x 8 x (2 * head_dim) product: A = the pages' [max | min] rows (staged in
// shared memory by cp.async), B = the heads' [q+ | q-] rows (registers).
// Products of two BF16 values are exact in the FP32 accumulator.
//
// Work: a tile is 16 pages of one (sequence, KV head); tiles are laid end to
// end (sequence-major) and every warp takes an equal contiguous range, with a
// ring of kScoreStages tiles in flight per warp.
constexpr int kScoreWarps = 4;
constexpr int kScoreStages = 3;
constexpr int kScoreMaxSeqs = 4096;  // tile prefix over sequences kept in shared memory

template <int D>
struct ScoreTile {
  static constexpr int kRow = 4 * D;            // staged bytes of a page: max row, then min row (BF16)
  static constexpr int kChunks = kRow / 16;     // 16-byte chunks of a staged page
  static constexpr int kBytes = 16 * kRow;      // 16 pages
  static constexpr int kKSteps = 2 * D / 16;    // MMA k-steps over [max | min]
  static constexpr int kRounds = 16 * kChunks / 32;  // cp.async rounds of a lane per tile
};

__host__ __device__ constexpr size_t score_tc_prefix_bytes(int num_seqs) {
  return ((size_t)(num_seqs + 1) * 4 + 127) / 128 * 128;
}

template <int D>
__global__ void __launch_bounds__(kScoreWarps * 32) quest_score_tc_kernel(const QuestSelParams p) {
  using T = ScoreTile<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  int* TP = reinterpret_cast<int*>(smem);  // TP[s] = tiles of sequences < s (all KV heads)
  __shared__ int scan_sh[33];
  __shared__ int info[kScoreWarps][kScoreStages][3];  // unit, tile in unit, mask of rejected pages
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, c = lane & 3;

  // ---- tile prefix over sequences (each thread a contiguous run)
  {
    const int per_t = (p.num_seqs + blockDim.x - 1) / blockDim.x;
    const int s0 = min(tid * per_t, p.num_seqs), s1 = min(s0 + per_t, p.num_seqs);
    int local = 0;
    for (int s = s0; s < s1; ++s) {
      const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
      local += p.n_kv * ((P + 15) / 16);
    }
    int total = 0;
    int run = cta_exclusive_scan(local, scan_sh, &total);
    for (int s = s0; s < s1; ++s) {
      TP[s] = run;
      const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
      run += p.n_kv * ((P + 15) / 16);
    }
    if (tid == 0) TP[p.num_seqs] = total;
    __syncthreads();
  }
  const int total = TP[p.num_seqs];
  const int nw = gridDim.x * kScoreWarps;
  const int per = (total + nw - 1) / nw;
  const int t0 = min((blockIdx.x * kScoreWarps + warp) * per, total), t1 = min(t0 + per, total);
  if (t0 >= t1) return;

  uint8_t* ring = smem + score_tc_prefix_bytes(p.num_seqs) + (size_t)warp * kScoreStages * T::kBytes;
  const uint32_t ring_addr = smem_addr(ring);

  // tile t -> (sequence, KV head, tile in unit, tiles per unit)
  auto locate = [&](int t, int& s, int& kv, int& i, int& tpu) {
    int lo = 0, hi = p.num_seqs;  // last s with TP[s] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (TP[mid] <= t) lo = mid; else hi = mid;
    }
    s = lo;
    tpu = (TP[s + 1] - TP[s]) / p.n_kv;
    const int r = t - TP[s];
    kv = r / tpu;
    i = r - kv * tpu;
  };

  auto issue = [&](int t, int stage) {
    int s, kv, i, tpu;
    locate(t, s, kv, i, tpu);
    const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
    int phys = -1, rejected = 0;
    if (lane < 16) {
      const int j = i * 16 + lane;
      if (j < P) {
        phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + j);
        if (phys < 0 || (long long)phys >= p.num_blocks) {
          flag_error(p.err, DEVERR_BLOCK_RANGE);
          phys = -1;
          rejected = 1;
        }
      }
    }
    const unsigned rej_mask = __ballot_sync(0xffffffffu, rejected);
    const uint32_t base = ring_addr + stage * T::kBytes;
    const char* pmax = static_cast<const char*>(p.page_max);
    const char* pmin = static_cast<const char*>(p.page_min);
#pragma unroll
    for (int r = 0; r < T::kRounds; ++r) {
      const int cidx = r * 32 + lane;
      const int m = cidx / T::kChunks, ch = cidx - m * T::kChunks;
      const int ph = __shfl_sync(0xffffffffu, phys, m);
      constexpr int half = T::kChunks / 2;
      const char* src = (ch < half ? pmax : pmin);
      uint32_t bytes = 0;
      if (ph >= 0) {
        src += (((size_t)ph * p.n_kv + kv) * D) * 2 + (size_t)(ch % half) * 16;
        bytes = 16;
      }
      cp_async16(base + m * T::kRow + ((ch ^ (m & 7)) << 4), src, bytes);
    }
    if (lane == 0) {
      info[warp][stage][0] = s * p.n_kv + kv;
      info[warp][stage][1] = i;
      info[warp][stage][2] = (int)rej_mask;
    }
  };

  // B fragments of the current unit's query heads: [q+ | q-] rows, head g of the 8
  uint32_t bq[T::kKSteps][2];
  int cur_unit = -1;
  auto load_query = [&](int u) {
    const int s = u / p.n_kv, kv = u - s * p.n_kv;
    const bool ok = g < p.G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        static_cast<const __nv_bfloat16*>(p.query) + ((size_t)s * p.n_q + kv * p.G + (ok ? g : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        const uint32_t x = ok ? __ldg(qrow + ks * 8 + c + hlf * 4) : 0u;
        const uint32_t neg = ((x & 0x8000u) ? 0x0000FFFFu : 0u) | ((x & 0x80000000u) ? 0xFFFF0000u : 0u);
        bq[ks][hlf] = x & ~neg;              // q+ against the max row
        bq[ks + D / 16][hlf] = x & neg;      // q- against the min row
      }
    }
  };

  const int row = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row (page) this lane addresses
  const int khalf = lane >> 4;                          // which 8 of the k-step's 16 columns

  int issued = t0;
#pragma unroll
  for (int k = 0; k < kScoreStages - 1; ++k) {
    if (issued < t1) issue(issued, k);
    ++issued;
    cp_async_commit();
  }
  for (int t = t0, it = 0; t < t1; ++t, ++it) {
    if (issued < t1) issue(issued, (it + kScoreStages - 1) % kScoreStages);
    ++issued;
    cp_async_commit();
    cp_async_wait<kScoreStages - 1>();
    __syncwarp();
    const int stage = it % kScoreStages;
    const int u = info[warp][stage][0], i = info[warp][stage][1];
    const unsigned rej = (unsigned)info[warp][stage][2];
    if (u != cur_unit) {
      load_query(u);
      cur_unit = u;
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t tile = ring_addr + stage * T::kBytes + row * T::kRow;
#pragma unroll
    for (int ks = 0; ks < T::kKSteps; ++ks) {
      uint32_t a[4];
      ldmatrix_x4(a, tile + (((ks * 2 + khalf) ^ (row & 7)) << 4));
      mma_bf16(acc, a, bq[ks][0], bq[ks][1]);
    }
    // acc: pages g (0, 1) and g + 8 (2, 3); heads 2c (0, 2) and 2c + 1 (1, 3)
    const bool h0 = 2 * c < p.G, h1 = 2 * c + 1 < p.G;
    float lo = fmaxf(h0 ? acc[0] : -INFINITY, h1 ? acc[1] : -INFINITY);
    float hi = fmaxf(h0 ? acc[2] : -INFINITY, h1 ? acc[3] : -INFINITY);
    lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 1));
    lo = fmaxf(lo, __shfl_xor_sync(0xffffffffu, lo, 2));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 1));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, 2));
    if (c == 0) {
      const int s = u / p.n_kv;
      const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
      float* out = p.scores + (size_t)u * p.max_pages + i * 16;
      if (i * 16 + g < P) out[g] = ((rej >> g) & 1) ? -INFINITY : lo;
      if (i * 16 + g + 8 < P) out[g + 8] = ((rej >> (g + 8)) & 1) ? -INFINITY : hi;
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------- top-k
// CTA per (sequence, KV head): the page scores become order-preserving keys
// in shared memory; a 4-pass radix select (8 bits a pass, from the top) finds
// the K-th largest key T and how many of its ties to keep; an index-order
// compaction keeps keys > T and the first ties, writing the pages ascending.
constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) quest_topk_kernel(const QuestSelParams p) {
  extern __shared__ uint32_t keys[];  // [max_pages]
  __shared__ int hist[256];
  __shared__ int scan_sh[33];
  __shared__ uint32_t sel_prefix;
  __shared__ int sel_need;
  const int tid = threadIdx.x, bd = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int s = blockIdx.x / p.n_kv, kv = blockIdx.x - s * p.n_kv;
  const int Lraw = __ldg(p.context_lens + s);
  if ((Lraw < 0 || Lraw > p.cap_len) && tid == 0 && kv == 0) flag_error(p.err, DEVERR_CONTEXT_LEN);
  const int P = (clamp_len(p, s) + kBlockSize - 1) / kBlockSize;
  const int K = min(p.k_pages, P);
  int32_t* out = p.selected + ((size_t)s * p.n_kv + kv) * p.k_pages;
  for (int i = K + tid; i < p.k_pages; i += bd) out[i] = -1;
  if (K == 0) return;
  const float* sc = p.scores + ((size_t)s * p.n_kv + kv) * p.max_pages;
  if (K == P) {  // every page
    for (int j = tid; j < P; j += bd) out[j] = j;
    return;
  }
  for (int j = tid; j < P; j += bd) keys[j] = order_key(sc[j]);
  __syncthreads();

  uint32_t prefix = 0, mask = 0;
  int need = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += bd) hist[i] = 0;
    __syncthreads();
    // scores cluster in few digits (the top ones especially): lanes of a warp
    // with the same digit add once
    for (int j0 = warp * 32; j0 < P; j0 += bd) {
      const int j = j0 + lane;
      const uint32_t k = j < P ? keys[j] : 0u;
      const bool in = j < P && (k & mask) == prefix;
      const int digit = in ? (int)((k >> shift) & 255) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (in && (__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 8l .. 8l+7; find the largest digit whose count of
      // keys at or above it reaches `need`
      int cnt[8], sum = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt[e] = hist[lane * 8 + e];
        sum += cnt[e];
      }
      int above = sum;  // keys in lanes >= this one (inclusive suffix sum)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, above, o);
        if (lane + o < 32) above += y;
      }
      const unsigned ok = __ballot_sync(0xffffffffu, above >= need);
      const int hl = 31 - __clz(ok);  // `need` <= keys matching the prefix, so some lane qualifies
      if (lane == hl) {
        int acc = above - sum;  // keys in higher lanes
        int dgt = lane * 8 + 7;
        for (int e = 7; e > 0; --e, --dgt) {
          if (acc + cnt[e] >= need) break;
          acc += cnt[e];
        }
        sel_prefix = prefix | ((uint32_t)dgt << shift);
        sel_need = need - acc;
      }
    }
    __syncthreads();
    prefix = sel_prefix;
    need = sel_need;
    mask |= 0xFFu << shift;
  }
  const uint32_t T = prefix;  // the K-th largest key; `need` of its ties are kept

  const int per = (P + bd - 1) / bd;
  const int j0 = min(tid * per, P), j1 = min(j0 + per, P);
  int gt = 0, eq = 0;
  for (int j = j0; j < j1; ++j) {
    gt += keys[j] > T;
    eq += keys[j] == T;
  }
  int eq_total = 0, tot = 0;
  const int eq_before = cta_exclusive_scan(eq, scan_sh, &eq_total);
  const int take_eq = max(0, min(eq, need - eq_before));
  int o = cta_exclusive_scan(gt + take_eq, scan_sh, &tot);
  int rank = eq_before;
  for (int j = j0; j < j1; ++j) {
    const uint32_t k = keys[j];
    bool pick = k > T;
    if (k == T) pick = rank++ < need;
    if (pick) out[o++] = j;
  }
}

pkv_status launch_quest_select(const void* query, const void* page_min, const void* page_max,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int64_t num_blocks,
                               pkv_dtype act, pkv_dtype cache, int k_pages, int32_t* selected, float* scores,
                               int32_t* device_error, cudaStream_t stream) {
  QuestSelParams p;
  p.query = query;
  p.page_min = page_min;
  p.page_max = page_max;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.selected = selected;
  p.scores = scores;
  p.err = device_error;
  p.num_blocks = num_blocks;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.cap_len = (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * kBlockSize);
  p.num_seqs = num_seqs;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.G = n_q / n_kv;
  p.k_pages = k_pages;
  p.max_pages = (p.cap_len + kBlockSize - 1) / kBlockSize;
  p.act_bf16 = act == PKV_BF16;
  const long long units = (long long)num_seqs * n_kv;
  if (units == 0) return PKV_OK;
  if (units > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  const int optin = device_smem_optin();
  const size_t topk_smem = (size_t)p.max_pages * 4;
  if (topk_smem > (size_t)optin - 4096) return PKV_ERR_UNSUPPORTED;

  cudaError_t e;
  const bool tc = cache == PKV_BF16 && act == PKV_BF16 && p.G <= 8 && num_seqs <= kScoreMaxSeqs;
  if (tc) {
    auto run = [&](auto kern, int tile_bytes) -> pkv_status {
      const size_t smem = score_tc_prefix_bytes(num_seqs) + (size_t)kScoreWarps * kScoreStages * tile_bytes;
      cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return cuda_fail(err, "cudaFuncSetAttribute(quest_score_tc)");
      int per_sm = (int)std::max<size_t>(1, (size_t)(optin) / (smem + 1024));
      per_sm = std::min(per_sm, 4);
      kern<<<device_sm_count() * per_sm, kScoreWarps * 32, smem, stream>>>(p);
      err = cudaGetLastError();
      if (err != cudaSuccess) return cuda_fail(err, "quest_score_tc_kernel launch");
      return PKV_OK;
    };
    pkv_status st = PKV_ERR_UNSUPPORTED;
    if (head_dim == 64) st = run(quest_score_tc_kernel<64>, ScoreTile<64>::kBytes);
    if (head_dim == 128) st = run(quest_score_tc_kernel<128>, ScoreTile<128>::kBytes);
    if (st != PKV_OK) return st;
  } else {
    const size_t smem = (size_t)p.G * head_dim * 4;
    if (smem > (size_t)optin - 2048) return PKV_ERR_UNSUPPORTED;
    auto run = [&](auto kern) -> pkv_status {
      cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return cuda_fail(err, "cudaFuncSetAttribute(quest_score_simt)");
      kern<<<(unsigned)units, 256, smem, stream>>>(p);
      err = cudaGetLastError();
      if (err != cudaSuccess) return cuda_fail(err, "quest_score_simt_kernel launch");
      return PKV_OK;
    };
    const bool bf16 = cache == PKV_BF16;
    pkv_status st = PKV_ERR_UNSUPPORTED;
    if (head_dim == 64) st = bf16 ? run(quest_score_simt_kernel<true, 2>) : run(quest_score_simt_kernel<false, 2>);
    if (head_dim == 128) st = bf16 ? run(quest_score_simt_kernel<true, 4>) : run(quest_score_simt_kernel<false, 4>);
    if (st != PKV_OK) return st;
  }
  e = cudaFuncSetAttribute(quest_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)topk_smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(quest_topk)");
  quest_topk_kernel<<<(unsigned)units, kTopkThreads, topk_smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quest_topk_kernel launch");
  return PKV_OK;
}

}  // namespace pkv
