// Paged decode attention on the tensor-core path: BF16, INT8, INT4, FP8 E4M3,
// FP8 E5M2 and 2-bit KIVI caches.
//
// What it computes: for every sequence s and query head h, softmax over the
// s-th sequence's cached keys of sm_scale * <q_h, K_p> weighting the cached
// values, with query heads grouped onto KV heads consecutively ("KV Cache
// Engineering for LLM Serving", section 1) and the rows found through the
// sequence's block table (KV-cache overview page t13_4, block-table paragraph;
// "Chapter 18 - KV-Cache Optimization Strategies", How PagedAttention Works).
//
// How (B200 design, not from the pages):
//  * Work unit = (sequence, group of HPC KV heads).  All units' 16-token blocks
//    are laid end to end and every persistent CTA takes an equal contiguous
//    share (split-K over context with no wave quantisation).  A unit cut by a
//    share boundary leaves one piece per CTA (normalised o, base-2 lse); the
//    merge kernel, queued behind this one with programmatic serialisation,
//    combines them in CTA order, so the result does not depend on timing.
//  * One producer warp streams each block's K and V tiles of the CTA's KV heads
//    into a ring of shared-memory stages, completing on mbarriers: TMA boxes of
//    [16 tokens x 128 bytes] with the 128-byte swizzle (INT4: 64-byte rows,
//    64-byte swizzle), or for the head-major 2-bit pools one bulk copy per pool
//    plus a swizzled TMA box of the per-channel K scales.  Block-table entries
//    are fetched 32 at a time by the producer's lanes.
//  * Consumer warp (KV head, chunk of 8 query heads): S^T[16 tok x 8 heads] =
//    K_blk * Q^T, an online base-2 softmax with warp shuffles, then
//    O^T[d x 8] += V^T * P^T with P^T via movmatrix.  BF16 uses m16n8k16 MMAs
//    fed by ldmatrix.  INT8 / INT4 scores run as m16n8k32 integer MMAs on the
//    stored codes against the query quantised per unit into two 8-bit parts;
//    E4M3 / E5M2 codes, and V codes of every quantised format, become exact f16
//    in registers.  Per-token scales multiply the scores and the
//    probabilities, per-head FP8 scales fold into constants, and the 2-bit
//    cache's per-(block, channel) K scales fold into the f16 query operand.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "cache_row.cuh"
#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

struct TcParams {
  void* out;
  const void* query;
  float* k_scale;  // written by the fused step's int8 append, read otherwise
  float* v_scale;
  // fused decode step: the new token's rows [num_seqs, n_kv, D] (act dtype),
  // appended as token L-1 of each sequence before it is attended; null = none
  const void* new_key;
  const void* new_value;
  void* key_cache;
  void* value_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* lse_out;
  int2* desc;  // per unit: (first CTA | second-slot flag << 30, pieces) for the merge launch
  float* part_o;
  float* part_lse;
  int* err;
  long long num_blocks;
  int max_blocks_per_seq;
  int cap_len;  // min(max_context_len, max_blocks_per_seq * 16)
  int max_context_len;
  int num_seqs, n_q, n_kv;
  int window, sinks;  // attend to [0, sinks) and [L - window, L) only; window 0 = every position
  // Quest: per (sequence, KV head) list of k_pages logical pages (ascending, -1
  // past the count) to read instead of every block; one KV head per unit
  const int32_t* pages;
  int k_pages;
  // shared-prefix decode: logical blocks < skip_blocks are attended by the
  // prefix pass, whose pieces the merge adds; every unit then leaves a piece
  // (merge_all), a unit finished inside one CTA in unit_o / unit_lse
  int skip_blocks;
  int merge_all;
  float* unit_o;    // [num_seqs * n_q][D], normalised
  float* unit_lse;  // [num_seqs * n_q], base 2
  // the prefix pass runs beside this kernel: wait for it (the previous
  // kernel) only before exiting, not before the work
  int late_wait;
  long long wait_limit;  // SM cycles a ring wait may spend before giving up
  // start state of each unit's first piece (the KIVI residual pass)
  const float* pre_o;    // [n_kv][rows][D], normalised
  const float* pre_lse;  // [n_kv][rows], base 2
  int pre_rows;
  int whole_blocks;  // only full 16-token blocks are in the pool (2-bit KIVI cache)
  int G, QC, HPC, HG, NCW, stages, units;
  float scale_log2;
  int act_bf16;
  uint32_t stage_bytes, tx_bytes;
};

constexpr float kLn2 = 0.6931471805599453f;
// Slack (log2 units) of the running softmax maximum before it is moved.
constexpr float kLazyLog2 = 8.f;

__device__ __forceinline__ float ex2(float x) { return ex2_approx(x); }

// Attended length of sequence s, clamped to what the launch and table cover.
__device__ __forceinline__ int seq_len(const TcParams& p, int s, bool report) {
  int L = __ldg(p.context_lens + s);
  if (L < 0 || L > p.cap_len) {
    if (report) flag_error(p.err, DEVERR_CONTEXT_LEN);
    L = L < 0 ? 0 : p.cap_len;
  }
  return L;
}

// The blocks a sequence of length L attends to, in order: all of them, or the
// blocks holding the sink positions [0, s_eff) followed by those holding the
// window [lo_w, L) (one contiguous run when the two touch).
struct AttendSet {
  int nb;           // blocks in the set
  int sink_blocks;  // set index j < sink_blocks is logical block j
  int win_first;    // set index j >= sink_blocks is logical block win_first + j - sink_blocks
  int s_eff, lo_w;  // attended positions: p < s_eff or lo_w <= p < L
};

__device__ __forceinline__ AttendSet attend_set(const TcParams& p, int L) {
  AttendSet a;
  const int nbl = p.whole_blocks ? L / kBlockSize : (L + kBlockSize - 1) / kBlockSize;
  a.nb = a.sink_blocks = a.win_first = nbl;
  a.s_eff = L;
  a.lo_w = 0;
  if (p.skip_blocks > 0) {  // positions [skip_blocks * 16, L) only
    a.s_eff = 0;
    a.sink_blocks = 0;
    a.win_first = min(p.skip_blocks, nbl);
    a.lo_w = min(p.skip_blocks * kBlockSize, L);
    a.nb = nbl - a.win_first;
    return a;
  }
  if (p.window > 0 && L > p.window) {
    a.lo_w = L - p.window;
    a.s_eff = min(p.sinks, L);
    if (a.lo_w <= a.s_eff) {
      a.s_eff = L;  // sinks reach the window: every position
      a.lo_w = 0;
    } else {
      const int sb = (a.s_eff + kBlockSize - 1) / kBlockSize, wb0 = a.lo_w / kBlockSize;
      if (wb0 >= sb) {
        a.sink_blocks = sb;
        a.win_first = wb0;
        a.nb = sb + (nbl - wb0);
      }
    }
  }
  return a;
}

__device__ __forceinline__ int logical_block(const AttendSet& a, int j) {
  return j < a.sink_blocks ? j : a.win_first + (j - a.sink_blocks);
}

// Rows of logical block lb that are attended: bit r <=> position lb*16 + r.
__device__ __forceinline__ uint32_t token_mask(const AttendSet& a, int L, int lb) {
  const int base = lb * kBlockSize;
  auto below = [](int n) -> uint32_t { return n <= 0 ? 0u : (n >= kBlockSize ? 0xFFFFu : (1u << n) - 1u); };
  uint32_t m = below(L - base);
  if (a.s_eff < L || a.lo_w > 0) m &= below(a.s_eff - base) | (0xFFFFu & ~below(a.lo_w - base));
  return m;
}

// Blocks of unit u (sequence length L): its attended set or, with a page list,
// the list's entries before its first -1, at most min(k_pages, pages of the
// sequence).  A full list (the usual case) costs one load.
__device__ __forceinline__ int unit_blocks(const TcParams& p, int u, int L) {
  const int nb = attend_set(p, L).nb;
  if (!p.pages) return nb;
  const int32_t* list = p.pages + (size_t)u * p.k_pages;  // one KV head per unit: u = s * n_kv + kv
  const int n = min(p.k_pages, nb);
  if (n == 0 || __ldg(list + n - 1) >= 0) return n;
  int lo = 0, hi = n - 1;  // listed pages (>= 0) come first, then -1
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(list + mid) >= 0) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// First index i in [0, n) with P[i] > x (n if none).
__device__ __forceinline__ int upper_bound_smem(const int* P, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (P[mid] <= x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// P[u] = number of blocks of units 0..u-1, P[units] = total.  All threads call.
__device__ void build_prefix(const TcParams& p, int* P, int* wsum) {
  const int nthreads = blockDim.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, nwarps = nthreads >> 5;
  const int units = p.units;
  const int per_t = (units + nthreads - 1) / nthreads;
  const int u0 = min(t * per_t, units), u1 = min(u0 + per_t, units);
  // counts into P[u]: four units at a time, so their loads are in flight together
  int local = 0;
  for (int u = u0; u < u1; u += 4) {
    int L[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) L[k] = u + k < u1 ? seq_len(p, (u + k) / p.HG, ((u + k) % p.HG) == 0) : 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (u + k < u1) {
        const int n = unit_blocks(p, u + k, L[k]);
        P[u + k] = n;
        local += n;
      }
    }
  }
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int v = lane < nwarps ? wsum[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < nwarps) wsum[lane] = incl - v;
  }
  __syncthreads();
  int run = wsum[warp] + x - local;
  for (int u = u0; u < u1; ++u) {  // this thread's own counts become offsets
    const int n = P[u];
    P[u] = run;
    run += n;
  }
  if (u1 == units && u0 < u1) P[units] = run;
  if (units == 0 && t == 0) P[0] = 0;
  __syncthreads();
}

template <int CACHE, int D>
struct TcTraits {
  static constexpr int kElem = CACHE == TC_BF16 ? 2 : 1;
  // bytes of one TMA box row: a 128-byte chunk, or a whole INT4 (64 bytes) or
  // 2-bit (32 bytes) head row
  static constexpr int kChunkBytes = CACHE == TC_INT4 ? D / 2 : CACHE == TC_KIVI ? D / 4 : 128;
  static constexpr int kChunks = (CACHE == TC_INT4 || CACHE == TC_KIVI) ? 1 : D * kElem / 128;  // chunks per head row
  static constexpr int kBox = kChunkBytes * 16;                            // one chunk of 16 rows
  static constexpr int kTile = kChunks * kBox;                             // one head's 16-row tile
  static constexpr int kSteps = D / 16;  // k-steps of Q.K and m-tiles of P.V
};

// Head dimension held in accumulator row g (hi = 0) or g + 8 (hi = 1) of P.V
// m-tile mt: the order in which each cache format's V fragments list the dims.
template <int CACHE, int D>
__device__ __forceinline__ int d_of(int mt, int hi, int g) {
  if constexpr (CACHE == TC_BF16) return mt * 16 + g + 8 * hi;
  else if constexpr (CACHE == TC_KIVI) return g * 16 + 8 * (mt >> 2) + 4 * hi + (mt & 3);
  else return g * 16 + 2 * mt + hi;
}

// Factor between an accumulator entry (m-tile mt, row g (hi = 0) or g + 8
// (hi = 1) of P.V) and the value it stands for: INT4 high nibbles and 2-bit
// codes are unpacked where they sit in their byte, so those entries hold 16
// (INT4, rows g + 8) or 4^(mt % 4) (2-bit, m-tile mt) times the sum.
template <int CACHE>
__device__ __forceinline__ float v_unscale(int mt, int hi) {
  if constexpr (CACHE == TC_INT4) return hi ? 1.f / 16.f : 1.f;
  else if constexpr (CACHE == TC_KIVI) return 1.f / (float)(1 << (2 * (mt & 3)));
  else return 1.f;
}

// ---------------------------------------------------------------- merge
// A unit split over several CTAs leaves one normalised partial output and its
// base-2 log-sum-exp per CTA ("piece").  A second launch, queued behind the
// decode kernel with programmatic serialisation, combines them: one CTA per
// unit (or several, see below), a thread per (query head, 4 dims).  A thread
// loads the lse and its 4 dims of up to kMergeBatch pieces at once, so a
// merge of that many pieces costs one L2 round trip, and combines them in a
// fixed order with a running maximum: M' = max(M, lse_k), the sums so far
// scaled by 2^(M - M'), then w_k = 2^(lse_k - M'); o = sum w_k o_k / sum w_k,
// lse = M + log2(sum w_k); with more pieces it takes the maximum first and
// then one weighted pass.  When units are expected to have more pieces than
// kMergeBatch, kMergeLanes lanes share a (query head, 4 dims): lane r takes
// pieces r, r + kMergeLanes, ..., and the lanes' sums meet in a fixed shuffle
// tree, over as many CTAs per unit as that takes.
// Under a shared prefix every unit is merged (decode_merge_all_kernel): its
// own piece(s) (CTA pieces, or the unit's whole piece) and then the prefix
// pass's split pieces of the same query row.
constexpr int kMergeBatch = 8;
constexpr int kMergeLanes = 8;

struct MergeParams {
  void* out;
  float* lse_out;
  const float* part_o;
  const float* part_lse;
  const int2* desc;
  int HG, QH, n_q, num_ctas, act_bf16;
  // shared prefix (merge_all): whole-unit pieces and the prefix pass's pieces
  int merge_all;
  const float* unit_o;
  const float* unit_lse;
  const float* pre_o;    // [n_kv][pre_splits][pre_rows][D]
  const float* pre_lse;  // [n_kv][pre_splits][pre_rows]
  int pre_rows, pre_splits, G, HPC;
};

// Running combination of pieces (lse base 2, o normalised) in the order given.
struct MergeAcc {
  float M = -INFINITY, wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // Pieces k = first, first + stride, ... below n; piece(k, lse_ptr, o_ptr)
  // names piece k's lse and this thread's 4 dims.
  template <typename PieceFn>
  __device__ __forceinline__ void add_pieces(int n, int first, int stride, PieceFn piece) {
    const int cnt = first < n ? (n - first + stride - 1) / stride : 0;
    if (cnt > kMergeBatch) {
      // many pieces: the maximum over all lse first, then one pass of weights
      float mb = M;
#pragma unroll 8
      for (int k = first; k < n; k += stride) {
        const float* lp;
        const float4* op;
        piece(k, lp, op);
        mb = fmaxf(mb, __ldcg(lp));
      }
      if (mb == -INFINITY) return;
      const float sc = ex2(M - mb);
      wsum *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
#pragma unroll 8
      for (int k = first; k < n; k += stride) {
        const float* lp;
        const float4* op;
        piece(k, lp, op);
        const float lv = __ldcg(lp);
        const float4 ov = __ldcg(op);
        if (lv > -INFINITY) {
          const float w = ex2(lv - mb);
          wsum += w;
          acc.x += w * ov.x;
          acc.y += w * ov.y;
          acc.z += w * ov.z;
          acc.w += w * ov.w;
        }
      }
      M = mb;
      return;
    }
    if (cnt > 0) {
      float lv[kMergeBatch];
      float4 ov[kMergeBatch];
#pragma unroll
      for (int i = 0; i < kMergeBatch; ++i) {
        lv[i] = -INFINITY;
        ov[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < cnt) {
          const float* lp;
          const float4* op;
          piece(first + i * stride, lp, op);
          lv[i] = __ldcg(lp);
          ov[i] = __ldcg(op);
        }
      }
      float mb = M;
#pragma unroll
      for (int i = 0; i < kMergeBatch; ++i) mb = fmaxf(mb, lv[i]);
      if (mb == -INFINITY) return;  // no piece with any weight
      const float sc = ex2(M - mb);   // 0 while M is -inf
      wsum *= sc;
      acc.x *= sc;
      acc.y *= sc;
      acc.z *= sc;
      acc.w *= sc;
#pragma unroll
      for (int i = 0; i < kMergeBatch; ++i) {
        if (lv[i] > -INFINITY) {
          const float w = ex2(lv[i] - mb);
          wsum += w;
          acc.x += w * ov[i].x;
          acc.y += w * ov[i].y;
          acc.z += w * ov[i].z;
          acc.w += w * ov[i].w;
        }
      }
      M = mb;
    }
  }
  // The sums of the `lanes` lanes that share this thread's (query head, 4
  // dims), combined in a fixed tree; every lane ends with the total.
  template <int lanes>
  __device__ __forceinline__ void reduce_lanes() {
    if constexpr (lanes == 1) return;
    float Mt = M;
#pragma unroll
    for (int o = 1; o < lanes; o <<= 1) Mt = fmaxf(Mt, __shfl_xor_sync(0xffffffffu, Mt, o));
    if (Mt == -INFINITY) return;  // no lane has a piece with weight
    const float sc = M == -INFINITY ? 0.f : ex2(M - Mt);
    wsum *= sc;
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
#pragma unroll
    for (int o = 1; o < lanes; o <<= 1) {
      wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    M = Mt;
  }
  // out row (bf16 or f32) and lse (natural log; -inf and zeros if nothing had weight)
  __device__ __forceinline__ void store(const MergeParams& p, long long row, int v, int D) const {
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    if (p.act_bf16) {
      __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.out) + row * D + 4 * v);
      o[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      o[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    } else {
      reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * D)[v] =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (p.lse_out && v == 0) p.lse_out[row] = wsum > 0.f ? (M + log2f(wsum)) * kLn2 : -INFINITY;
  }
};

template <int D, int L>
__global__ void __launch_bounds__(512, 2) decode_merge_kernel(const MergeParams p) {
  grid_launch_dependents();
  grid_wait_prerequisites();  // the decode kernel's pieces and descriptors are complete
  const int u = blockIdx.x;
  const int2 d = p.desc[u];
  const int c0 = d.x & 0x3FFFFFFF, n = d.y;
  const bool c0_slot1 = (d.x >> 30) & 1;
  // whole unit in one CTA (written there), or no pieces; a descriptor out of
  // range (only after a timed-out decode) is skipped
  if (n < 2 || n > p.num_ctas || c0 >= p.num_ctas || c0 + n > p.num_ctas) return;
  const int s = u / p.HG, hg = u - s * p.HG;
  constexpr int V = D / 4;
  const int r = threadIdx.x % L;  // L lanes per (query head, 4 dims); L divides the block
  const int pairs = p.QH * V, step = gridDim.y * blockDim.x / L;
  for (int idx = (blockIdx.y * blockDim.x + threadIdx.x) / L; idx - (int)(threadIdx.x / L) < pairs; idx += step) {
    const bool live = idx < pairs;  // a lane group past the end still joins the shuffles
    const int h = live ? idx / V : 0, v = live ? idx - h * V : 0;
    MergeAcc m;
    // CTA c0 + k's piece: slot 1 for k == 0 when the unit starts inside CTA c0's range
    if (live)
      m.add_pieces(n, r, L, [&](int k, const float*& lp, const float4*& op) {
        const size_t piece = ((size_t)(c0 + k) * 2 + ((k == 0 && c0_slot1) ? 1 : 0)) * p.QH + h;
        lp = p.part_lse + piece;
        op = reinterpret_cast<const float4*>(p.part_o + piece * D) + v;
      });
    m.reduce_lanes<L>();
    if (live && r == 0) m.store(p, (long long)s * p.n_q + hg * p.QH + h, v, D);
  }
}

template <int D, int L>
__global__ void __launch_bounds__(512, 2) decode_merge_all_kernel(const MergeParams p) {
  grid_launch_dependents();
  grid_wait_prerequisites();  // the decode kernel's pieces and descriptors are complete
  const int u = blockIdx.x;
  const int2 d = p.desc[u];
  const int c0 = d.x & 0x3FFFFFFF;
  int n = d.y;
  const bool c0_slot1 = (d.x >> 30) & 1;
  // a descriptor out of range (only after a timed-out decode) contributes nothing
  if (n < 0 || n > p.num_ctas || c0 >= p.num_ctas || c0 + n > p.num_ctas) n = 0;
  const int s = u / p.HG, hg = u - s * p.HG;
  const int npre = p.pre_splits;
  const int own = n;  // the unit's own pieces: n CTA pieces, its one whole piece (n == 1), or none
  constexpr int V = D / 4;
  const int r = threadIdx.x % L;  // L lanes per (query head, 4 dims); L divides the block
  const int pairs = p.QH * V, step = gridDim.y * blockDim.x / L;
  for (int idx = (blockIdx.y * blockDim.x + threadIdx.x) / L; idx - (int)(threadIdx.x / L) < pairs; idx += step) {
    const bool live = idx < pairs;  // a lane group past the end still joins the shuffles
    const int h = live ? idx / V : 0, v = live ? idx - h * V : 0;
    const long long row = (long long)s * p.n_q + hg * p.QH + h;
    // own piece k: the whole unit's (own == 1, written by one CTA), or CTA
    // c0 + k's slot (slot 1 of CTA c0 when the unit starts inside its range,
    // slot 0 after that: 2 QH lse apart)
    const size_t own0 = own == 1 ? 0 : ((size_t)c0 * 2 + (c0_slot1 ? 1 : 0)) * p.QH + h;
    const float* own_l = own == 1 ? p.unit_lse + row : p.part_lse + own0;
    const float* own_o = own == 1 ? p.unit_o + row * D : p.part_o + own0 * D;
    const long long own_back = c0_slot1 ? p.QH : 0;
    // the prefix pass's splits of this query row, pre_rows apart
    const int kvh = hg * p.HPC + h / p.G;
    const size_t pre_row = (size_t)kvh * npre * p.pre_rows + (size_t)s * p.G + h % p.G;
    const float* pre_l = p.pre_lse + pre_row;
    const float* pre_o = p.pre_o + pre_row * D;
    MergeAcc m;
    if (live)
      m.add_pieces(own + npre, r, L, [&](int k, const float*& lp, const float4*& op) {
      if (k < own) {
        const long long off = k == 0 ? 0 : (long long)k * 2 * p.QH - own_back;
        lp = own_l + off;
        op = reinterpret_cast<const float4*>(own_o + off * D) + v;
      } else {
        const size_t off = (size_t)(k - own) * p.pre_rows;
        lp = pre_l + off;
        op = reinterpret_cast<const float4*>(pre_o + off * D) + v;
      }
    });
    m.reduce_lanes<L>();
    if (live && r == 0) m.store(p, row, v, D);
  }
}

template <int CACHE, int D, int MAXW, int MINB>
__global__ void __launch_bounds__((MAXW + 1) * 32, MINB)
    decode_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap smap, const TcParams p) {
  using Tr = TcTraits<CACHE, D>;
  constexpr int KS = Tr::kSteps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)p.stages * p.stage_bytes);
  uint64_t* empty = full + p.stages;
  uint64_t* append_done = empty + p.stages;  // fused step: the new rows are in the cache
  int* wsum = reinterpret_cast<int*>(append_done + 1);
  int* P = wsum + 32;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = p.units;

  grid_launch_dependents();
  if (threadIdx.x == 0) {
    for (int k = 0; k < p.stages; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], p.NCW);
    }
    mbar_init(append_done, p.HPC);  // one arrival per KV head of the CTA
    fence_barrier_init();
  }
  if (warp == p.NCW && lane == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    if constexpr (CACHE == TC_KIVI) prefetch_tensormap(&smap);
  }
  build_prefix(p, P, wsum);  // ends with __syncthreads()

  const int total = P[units];
  const int per = max(1, (total + (int)gridDim.x - 1) / (int)gridDim.x);
  const int a = min((int)blockIdx.x * per, total);
  const int b = min(a + per, total);
  // Producer lanes look up the physical blocks of 32 consecutive entries of
  // the range: block i (lane's) of unit u, its KV head group, whether it is
  // the unit's last block; -1 (bad = true) for an entry out of the pool.
  auto lookup = [&](int base, int& phys, int& hg, int& unit_last, bool& bad) {
    const int i = base + lane;
    phys = -1;
    hg = 0;
    unit_last = 0;
    bad = false;
    if (i < b) {
      const int u = upper_bound_smem(P, units + 1, i) - 1;
      const int s = u / p.HG;
      hg = u - s * p.HG;
      unit_last = (i + 1 == P[u + 1]);
      const int Ls = seq_len(p, s, false);
      int lb;
      if (p.pages) {
        lb = __ldg(p.pages + ((size_t)s * p.n_kv + hg) * p.k_pages + (i - P[u]));
        if (lb < 0 || (long long)lb * kBlockSize >= Ls) lb = -1;  // not a page of this sequence
      } else {
        lb = logical_block(attend_set(p, Ls), i - P[u]);
      }
      phys = lb < 0 ? -1 : __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + lb);
      if (phys < 0 || (long long)phys >= p.num_blocks) {
        bad = true;
        phys = -1;
      }
    }
  };
  // The first lookup reads only block_tables (and context_lens): it may run
  // before the wait below (page lists may come from the previous kernel).
  int phys0 = -1, hg0 = 0, last0 = 0;
  bool bad0 = false, early = false;
  if (warp == p.NCW && a < b && !p.pages) {
    lookup(a, phys0, hg0, last0, bad0);
    early = true;
  }
  // Everything above read only context_lens and block_tables.  Under a
  // programmatic launch the previous kernel may still be running: wait for it
  // before touching queries, new rows, the cache, the workspace or outputs.
  // Beside the shared-prefix pass (late_wait) that kernel is the prefix pass,
  // which touches none of these (it let this grid start only after its own
  // wait for the kernel before it): the producer waits for it before exiting,
  // so that this grid completes after it and the merge sees its pieces.
  if (!p.late_wait) grid_wait_prerequisites();

  // ------------------------------------------------------------ producer
  if (warp == p.NCW) {
    if (a >= b) {
      if (p.late_wait) grid_wait_prerequisites();
      return;
    }
    int it = 0;
    int pstage = 0;       // ring stage of block `it`
    uint32_t ppass = 0;   // parity of the ring pass of block `it`
    bool abort = false, appended = false;
    for (int base = a; base < b && !abort; base += 32) {
      int phys, hg, unit_last;
      bool bad;
      if (base == a && early) {
        phys = phys0;
        hg = hg0;
        unit_last = last0;
        bad = bad0;
      } else {
        lookup(base, phys, hg, unit_last, bad);
      }
      if (bad) flag_error(p.err, DEVERR_BLOCK_RANGE);
      const int n = min(32, b - base);
      for (int k = 0; k < n; ++k) {
        const int ph = __shfl_sync(0xffffffffu, phys, k);
        const int hgk = __shfl_sync(0xffffffffu, hg, k);
        const int lastk = __shfl_sync(0xffffffffu, unit_last, k);
        int ok = 1;
        if (lane == 0) {
          const int stage = pstage;
          if (it >= p.stages && !mbar_wait(&empty[stage], ppass ^ 1u, p.wait_limit)) {
            flag_error(p.err, DEVERR_TIMEOUT);
            ok = 0;
          } else if (p.new_key && lastk && !appended && !(appended = mbar_wait(append_done, 0, p.wait_limit))) {
            // the block holding a new token is read only after the consumers wrote it
            flag_error(p.err, DEVERR_TIMEOUT);
            ok = 0;
          } else {
            uint8_t* st = smem + (size_t)stage * p.stage_bytes;
            mbar_arrive_expect_tx(&full[stage], p.tx_bytes);
            if constexpr (CACHE == TC_KIVI) {
              // head-major pools: the (block, head) tiles of the CTA's heads are
              // contiguous, as are their K scales and V scales (a rejected entry
              // reads block 0; its error bit is set)
              const size_t tile0 = (size_t)(ph >= 0 ? ph : 0) * p.n_kv + hgk * p.HPC;
              const uint32_t codes = p.HPC * Tr::kTile;
              bulk_load(st, static_cast<const uint8_t*>(p.key_cache) + tile0 * Tr::kTile, codes, &full[stage]);
              bulk_load(st + codes, static_cast<const uint8_t*>(p.value_cache) + tile0 * Tr::kTile, codes,
                        &full[stage]);
              // K scales: rows of 32 channels, 128-byte swizzle; V scales: 16 per head
              uint8_t* sc = st + 2 * codes;
              tma_load_2d(sc, &smap, 0, (int)(tile0 * (D / 32)), &full[stage]);
              bulk_load(sc + p.HPC * D * 4, p.v_scale + tile0 * kBlockSize, 64u * p.HPC, &full[stage]);
            } else {
              const int row = ph * kBlockSize;  // -16 for a rejected entry: the TMA zero-fills it
#pragma unroll 1
              for (int hl = 0; hl < p.HPC; ++hl) {
#pragma unroll
                for (int ch = 0; ch < Tr::kChunks; ++ch) {
                  const int c1 = (hgk * p.HPC + hl) * Tr::kChunks + ch;
                  tma_load_3d(st + (hl * Tr::kChunks + ch) * Tr::kBox, &kmap, 0, c1, row, &full[stage]);
                  tma_load_3d(st + (p.HPC + hl) * Tr::kTile + ch * Tr::kBox, &vmap, 0, c1, row, &full[stage]);
                }
              }
            }
            if constexpr (tc_row_scaled(CACHE)) {
              const size_t sb = (size_t)(ph >= 0 ? ph : 0) * kBlockSize * p.n_kv;
              const uint32_t bytes = 64u * p.n_kv;
              uint8_t* sc = st + 2 * p.HPC * Tr::kTile;
              bulk_load(sc, p.k_scale + sb, bytes, &full[stage]);
              bulk_load(sc + bytes, p.v_scale + sb, bytes, &full[stage]);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { abort = true; break; }
        ++it;
        if (++pstage == p.stages) {
          pstage = 0;
          ppass ^= 1u;
        }
      }
    }
    // Never leave with copies in flight: wait for the last stages issued
    // (with the full limit, whatever the ring waits were given).
    if (lane == 0) {
      for (int k = max(0, it - p.stages); k < it; ++k) mbar_wait(&full[k % p.stages], (k / p.stages) & 1);
    }
    if (p.late_wait) grid_wait_prerequisites();
    return;
  }

  // ------------------------------------------------------------ consumers
  const int head_local = warp / p.QC;
  const int qc = warp - head_local * p.QC;
  const int g = lane >> 2, c = lane & 3;
  const int QH = p.HPC * p.G;
  const int qbase_local = head_local * p.G + qc * 8;  // q head index inside the unit
  const bool head0_ok = qc * 8 + 2 * c < p.G, head1_ok = qc * 8 + 2 * c + 1 < p.G;

  // Units with no blocks (empty sequences, empty page lists): out = 0,
  // lse = -inf, or with a starting state (the KIVI residual pass) that state.
  // CTAs share the scan, 32 units per warp step.
  for (int u0 = blockIdx.x * 32; u0 < units; u0 += gridDim.x * 32) {
    const int uu = u0 + lane;
    unsigned empty_units = __ballot_sync(0xffffffffu, uu < units && P[uu] == P[uu + 1]);
    while (empty_units) {
      const int u = u0 + __ffs(empty_units) - 1;
      empty_units &= empty_units - 1;
      if (warp == 0 && lane == 0) p.desc[u] = make_int2(0, 0);
      if (p.merge_all) continue;  // the merge writes it (from the prefix pieces alone)
      const int s = u / p.HG, hg = u - s * p.HG;
      for (int n = 0; n < 8; ++n) {
        if (qc * 8 + n >= p.G) break;
        const long long row = (long long)s * p.n_q + hg * QH + qbase_local + n;
        const size_t pre_row = ((size_t)(hg * p.HPC + head_local) * p.pre_rows + (size_t)s * p.G + qc * 8 + n);
        for (int dd = lane; dd < D; dd += 32) {
          const float v = p.pre_o ? __ldcg(p.pre_o + pre_row * D + dd) : 0.f;
          if (p.act_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[row * D + dd] = __float2bfloat16_rn(v);
          else reinterpret_cast<float*>(p.out)[row * D + dd] = v;
        }
        if (p.lse_out && lane == 0) p.lse_out[row] = p.pre_o ? __ldcg(p.pre_lse + pre_row) * kLn2 : -INFINITY;
      }
    }
  }
  if (a >= b) return;

  // Fused step: this CTA reads the last block of every unit that ends inside
  // its range, so it writes those units' new rows (token L-1) into the cache
  // first, one warp per KV head, while the producer starts the ring.  The
  // proxy fence orders these generic stores before the TMA reads of the block.
  if (CACHE != TC_KIVI && p.new_key && qc == 0) {
    for (int uu = upper_bound_smem(P, units + 1, a) - 1; uu < units && P[uu] < b; ++uu) {
      if (P[uu + 1] > b) break;  // ends past this range: another CTA appends it
      if (P[uu] == P[uu + 1]) continue;
      const int ss = uu / p.HG, kv = (uu - ss * p.HG) * p.HPC + head_local;
      const int pos = seq_len(p, ss, false) - 1;
      const int phys = __ldg(p.block_tables + (size_t)ss * p.max_blocks_per_seq + pos / kBlockSize);
      if (phys < 0 || (long long)phys >= p.num_blocks) {
        if (lane == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
        continue;
      }
      const size_t dst_row = ((size_t)phys * kBlockSize + pos % kBlockSize) * p.n_kv + kv;
      const size_t src_row = (size_t)ss * p.n_kv + kv;
      constexpr int kind = CACHE == TC_BF16   ? WK_COPY
                           : CACHE == TC_INT8 ? WK_INT8
                           : CACHE == TC_INT4 ? WK_INT4
                           : CACHE == TC_E5M2 ? WK_E5M2
                                              : WK_FP8;
      if constexpr (CACHE == TC_KIVI) {
        // the KIVI residual pass appends (a row is quantised only with its block)
      } else if (p.act_bf16) {
        write_row<true, kind, D / 32>(static_cast<const uint8_t*>(p.new_key) + src_row * D * 2, p.key_cache, p.k_scale,
                                      dst_row, kv, p.n_kv, lane);
        write_row<true, kind, D / 32>(static_cast<const uint8_t*>(p.new_value) + src_row * D * 2, p.value_cache,
                                      p.v_scale, dst_row, kv, p.n_kv, lane);
      } else if constexpr (CACHE != TC_BF16) {
        write_row<false, kind, D / 32>(static_cast<const uint8_t*>(p.new_key) + src_row * D * 4, p.key_cache, p.k_scale,
                                       dst_row, kv, p.n_kv, lane);
        write_row<false, kind, D / 32>(static_cast<const uint8_t*>(p.new_value) + src_row * D * 4, p.value_cache,
                                       p.v_scale, dst_row, kv, p.n_kv, lane);
      }
    }
    fence_proxy_async_global();
    __syncwarp();
    if (lane == 0) mbar_arrive(append_done);
  }

  // Per-lane ldmatrix offsets inside a head tile (128-byte swizzle: the 16-byte
  // chunk j of row r lives at chunk j ^ (r & 7)).
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int k_cadd = lane >> 4;
  const int v_tok = (lane & 7) + ((lane >> 4) & 1) * 8;
  const int v_cadd = (lane >> 3) & 1;
  const int sw = lane & 7;
  // Byte offset of this lane's first 16-byte piece inside a head tile.  The
  // swizzle XORs address bits [6:4] with the row's low bits, so the piece for
  // chunk (base ^ x) sits at offset koff ^ (x << 4): one XOR per access.
  //  bf16: ldmatrix rows k_row / v_tok, chunk pair (ks & 3) * 2 (+ lane's half)
  //  int8/fp8: K rows g (+8 rows = +1024 B), chunks 2c (+1); V rows 2c (+1, +8, +9), chunk g
  uint32_t koff, voff;
  if constexpr (CACHE == TC_BF16) {
    koff = k_row * 128 + ((k_cadd ^ sw) << 4);
    voff = v_tok * 128 + ((v_cadd ^ sw) << 4);
  } else {
    koff = g * 128 + (((2 * c) ^ g) << 4);
    voff = (2 * c) * 128 + ((g ^ (2 * c)) << 4);
  }

  const int u_first = upper_bound_smem(P, units + 1, a) - 1;
  int u = u_first;
  int j = a - P[u];
  int s = 0, hg = 0, L = 0;
  AttendSet aset{};
  int last_page = 0;
  float head_k_scale = 1.f, head_v_scale = 1.f;

  uint32_t qf[KS][2];
  // INT8 / INT4: the queries as two 8-bit parts per dim for m16n8k32 MMAs
  // (q ~ qscale * (h + l / 254)), the per-column scales, and for INT4 the sums
  // of the parts times 8 (the stored codes are offset by 8)
  uint32_t qh[4][2], ql[4][2];
  float qs0 = 0.f, qs1 = 0.f;
  int ch0 = 0, ch1 = 0, cl0 = 0, cl1 = 0;
  float acc[KS][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // Query words of a unit as loaded (bf16 pairs), in the order of the MMA B
  // fragments.  BF16: dims ks*16 + 2c, +1 and ks*16 + 2c + 8, +9.  FP8: k-step
  // ks = h * 4 + k covers, for lane column c, dims (2c + h) * 16 + 4k + {0..3}
  // (the order in which the FP8 K fragments take the stored bytes).
  uint32_t qraw[KS][2];
  auto fetch_query = [&](int uu) {
    const int ss = uu / p.HG, hh = uu - ss * p.HG;
    const int kv = hh * p.HPC + head_local;
    const bool q_ok = qc * 8 + g < p.G;
    const size_t qoff = ((size_t)ss * p.n_q + kv * p.G + qc * 8 + g) * D;  // query head of fragment column g
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(p.query) + qoff);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      if constexpr (CACHE == TC_BF16) {
        qraw[ks][0] = q_ok ? __ldg(q32 + (ks * 16 + 2 * c) / 2) : 0u;
        qraw[ks][1] = q_ok ? __ldg(q32 + (ks * 16 + 2 * c + 8) / 2) : 0u;
      } else {
        const int d0 = (2 * c + (ks >> 2)) * 16 + 4 * (ks & 3);
        const uint2 w = q_ok ? __ldg(reinterpret_cast<const uint2*>(q32 + d0 / 2)) : make_uint2(0u, 0u);
        qraw[ks][0] = w.x;
        qraw[ks][1] = w.y;
      }
    }
  };

  // Scores of one 16-token block held in stage memory st: S^T = K Q^T
  // [16 tokens x 8 heads] in log2 units, -inf past the sequence end.
  // sv = (token g, head 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1); vsc = the
  // per-token V scales (INT8, INT4, 2-bit) of tokens g and g+8 (1 otherwise).
  auto block_scores = [&](const uint8_t* st, uint32_t vm, float (&sv)[4], float (&vsc)[2]) {
    const uint32_t kt = smem_addr(st + head_local * Tr::kTile);
    const int t0 = g, t1 = g + 8;
    // ---- S^T = K Q^T : [16 tokens x 8 heads]
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (CACHE == TC_BF16) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t af[4];
        ldmatrix_x4(af, kt + (koff ^ ((ks & 3) << 5)) + (ks >> 2) * 2048);
        if (ks & 1) mma_bf16(sb, af, qf[ks][0], qf[ks][1]);
        else mma_bf16(sa, af, qf[ks][0], qf[ks][1]);
      }
    } else if constexpr (CACHE == TC_INT4) {
      // lane (g, c) reads the 16-byte chunk c (dims 32c .. 32c+31) of rows g and
      // g+8; 64-byte rows under the 64-byte swizzle: chunk c of row r sits at
      // chunk c ^ ((r >> 1) & 3), the same for rows g and g+8
      const uint32_t kb = kt + g * 64 + ((uint32_t)(c ^ ((g >> 1) & 3)) << 4);
      const uint4 r0 = lds128(kb), r1 = lds128(kb + 512);
      // k-step kk: word kk of the chunk, its even nibbles (offset-binary codes
      // + 8, as unsigned bytes) and its odd nibbles, against the query parts
      int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t x0 = (&r0.x)[kk] ^ 0x88888888u, x1 = (&r1.x)[kk] ^ 0x88888888u;
        const uint32_t af[4] = {x0 & 0x0F0F0F0Fu, x1 & 0x0F0F0F0Fu, (x0 >> 4) & 0x0F0F0F0Fu,
                                (x1 >> 4) & 0x0F0F0F0Fu};
        mma_u8s8(ah, af, qh[kk][0], qh[kk][1]);
        mma_u8s8(al, af, ql[kk][0], ql[kk][1]);
      }
      // sum (code + 8) q = sum code q + 8 sum q: the offsets come back out exactly
      sa[0] = ((float)(ah[0] - ch0) + (float)(al[0] - cl0) * (1.f / 254.f)) * qs0;
      sa[1] = ((float)(ah[1] - ch1) + (float)(al[1] - cl1) * (1.f / 254.f)) * qs1;
      sa[2] = ((float)(ah[2] - ch0) + (float)(al[2] - cl0) * (1.f / 254.f)) * qs0;
      sa[3] = ((float)(ah[3] - ch1) + (float)(al[3] - cl1) * (1.f / 254.f)) * qs1;
    } else if constexpr (CACHE == TC_KIVI) {
      // 2-bit codes, 32-byte rows: lane (g, c) reads bytes 8c .. 8c+7 (dims
      // 32c .. 32c+31) of rows g and g+8.  The block's per-channel K scales
      // fold into the query: B = q * scale (f16) for the lane's channels, row
      // 4 * head_local + c of the scale tile, whose 16-byte chunk kk sits at
      // kk ^ (row & 7) under the 128-byte swizzle (conflict-free).
      const uint2 r0 = lds64(kt + g * 32 + 8 * c), r1 = lds64(kt + (g + 8) * 32 + 8 * c);
      const int srow = 4 * head_local + c;
      const uint32_t ksb = smem_addr(st + 2 * p.HPC * Tr::kTile) + srow * 128;
      float f[8][4];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint4 w = lds128(ksb + ((uint32_t)(kk ^ (srow & 7)) << 4));
        f[kk][0] = __uint_as_float(w.x);
        f[kk][1] = __uint_as_float(w.y);
        f[kk][2] = __uint_as_float(w.z);
        f[kk][3] = __uint_as_float(w.w);
      }
      // k-step ks: word m = ks >> 2 of the row, byte pair (t, t + 2) with
      // t = (ks >> 1) & 1, codes s0 = 2 (ks & 1) and s0 + 1 of each byte:
      // dims 32c + 16m + 4t + s and 32c + 16m + 8 + 4t + s.  The codes are
      // unpacked where they sit (times 4^s0, 4^(s0+1)); the query parts carry
      // 4^-s0 and 4^-(s0+1) (kivi_query_factor).
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int m = ks >> 2, t = (ks >> 1) & 1, s0 = 2 * (ks & 1);
        const uint32_t w0 = (m ? r0.y : r0.x) >> (8 * t), w1 = (m ? r1.y : r1.x) >> (8 * t);
        const uint32_t af[4] = {i2x2_at_to_f16x2(w0, s0), i2x2_at_to_f16x2(w1, s0), i2x2_at_to_f16x2(w0, s0 + 1),
                                i2x2_at_to_f16x2(w1, s0 + 1)};
        const uint32_t b0 = hmul2_u32(qf[ks][0], pack_f16(f[4 * m + t][s0], f[4 * m + t + 2][s0]));
        const uint32_t b1 = hmul2_u32(qf[ks][1], pack_f16(f[4 * m + t][s0 + 1], f[4 * m + t + 2][s0 + 1]));
        if (ks & 1) mma_f16(sb, af, b0, b1);
        else mma_f16(sa, af, b0, b1);
      }
    } else if constexpr (CACHE == TC_INT8) {
      // lane (g, c) reads rows g and g+8, chunks 2c and 2c+1 (16 bytes each); k-step
      // kk takes the bytes of dims 32c + 8kk + {0..3} and {4..7} as they are stored
      uint4 kr[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        kr[0][h] = lds128(kt + (koff ^ (h << 4)));
        kr[1][h] = lds128(kt + (koff ^ (h << 4)) + 1024);
      }
      int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int h = kk >> 1, wv = (kk & 1) * 2;
        const uint32_t af[4] = {(&kr[0][h].x)[wv], (&kr[1][h].x)[wv], (&kr[0][h].x)[wv + 1], (&kr[1][h].x)[wv + 1]};
        mma_s8s8(ah, af, qh[kk][0], qh[kk][1]);
        mma_s8s8(al, af, ql[kk][0], ql[kk][1]);
      }
      sa[0] = ((float)ah[0] + (float)al[0] * (1.f / 254.f)) * qs0;
      sa[1] = ((float)ah[1] + (float)al[1] * (1.f / 254.f)) * qs1;
      sa[2] = ((float)ah[2] + (float)al[2] * (1.f / 254.f)) * qs0;
      sa[3] = ((float)ah[3] + (float)al[3] * (1.f / 254.f)) * qs1;
    } else {
      // FP8: lane (g, c) reads rows g and g+8, chunks 2c and 2c+1 (16 bytes
      // each); k-step ks takes the byte pairs (0, 1) -> k = 2c, 2c+1 and (2, 3)
      // -> k = 2c+8, 2c+9 of word ks & 3 of chunk 2c + (ks >> 2), as f16 values
      uint4 kr[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        kr[0][h] = lds128(kt + (koff ^ (h << 4)));
        kr[1][h] = lds128(kt + (koff ^ (h << 4)) + 1024);
      }
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int h = ks >> 2, k = ks & 3;
        const uint32_t w0 = (&kr[0][h].x)[k], w1 = (&kr[1][h].x)[k];
        uint32_t af[4];
        if constexpr (CACHE == TC_E5M2) {
          // an E5M2 byte is the top byte of the f16 of the same value
          af[0] = prmt(w0, 0u, 0x1404);
          af[1] = prmt(w1, 0u, 0x1404);
          af[2] = prmt(w0, 0u, 0x3424);
          af[3] = prmt(w1, 0u, 0x3424);
        } else {
          // E4M3 pairs through the hardware conversion (exact values); a code
          // that reads as NaN sits in a row that is not attended, whose score
          // the select below replaces by -inf
          e4m3x4_to_f16x2x2(w0, af[0], af[2]);
          e4m3x4_to_f16x2x2(w1, af[1], af[3]);
        }
        if (ks & 1) mma_f16(sb, af, qf[ks][0], qf[ks][1]);
        else mma_f16(sa, af, qf[ks][0], qf[ks][1]);
      }
    }

    float sc0 = p.scale_log2, sc1 = p.scale_log2;
    vsc[0] = vsc[1] = 1.f;
    const int kvh = hg * p.HPC + head_local;
    if constexpr (tc_row_scaled(CACHE)) {
      const float* ksm = reinterpret_cast<const float*>(st + 2 * p.HPC * Tr::kTile);
      const float* vsm = ksm + kBlockSize * p.n_kv;
      sc0 *= ksm[t0 * p.n_kv + kvh];
      sc1 *= ksm[t1 * p.n_kv + kvh];
      vsc[0] = vsm[t0 * p.n_kv + kvh];
      vsc[1] = vsm[t1 * p.n_kv + kvh];
    } else if constexpr (CACHE == TC_KIVI) {
      const float* vsm = reinterpret_cast<const float*>(st + 2 * p.HPC * Tr::kTile + p.HPC * D * 4) + head_local * 16;
      vsc[0] = vsm[t0];
      vsc[1] = vsm[t1];
    } else if constexpr (tc_fp8(CACHE)) {
      sc0 *= head_k_scale;
      sc1 *= head_k_scale;
    }
    const bool ok0 = (vm >> t0) & 1u, ok1 = (vm >> t1) & 1u;
    sv[0] = ok0 ? (sa[0] + sb[0]) * sc0 : -INFINITY;
    sv[1] = ok0 ? (sa[1] + sb[1]) * sc0 : -INFINITY;
    sv[2] = ok1 ? (sa[2] + sb[2]) * sc1 : -INFINITY;
    sv[3] = ok1 ? (sa[3] + sb[3]) * sc1 : -INFINITY;
  };

  // O^T += V^T P^T for one block with probabilities pr (layout of the scores).
  auto block_pv = [&](const uint8_t* st, uint32_t vm, const float (&pr)[4], const float (&vsc)[2]) {
    const uint32_t vt = smem_addr(st + (p.HPC + head_local) * Tr::kTile);
    const bool ok0 = (vm >> g) & 1u, ok1 = (vm >> (g + 8)) & 1u;
    uint32_t pb0, pb1;
    if constexpr (CACHE == TC_BF16) {
      pb0 = movmatrix_trans(pack_bf16(pr[0], pr[1]));
      pb1 = movmatrix_trans(pack_bf16(pr[2], pr[3]));
    } else if constexpr (tc_v_row_scaled(CACHE)) {
      pb0 = movmatrix_trans(pack_f16(ok0 ? pr[0] * vsc[0] : 0.f, ok0 ? pr[1] * vsc[0] : 0.f));
      pb1 = movmatrix_trans(pack_f16(ok1 ? pr[2] * vsc[1] : 0.f, ok1 ? pr[3] * vsc[1] : 0.f));
    } else {
      pb0 = movmatrix_trans(pack_f16(pr[0], pr[1]));
      pb1 = movmatrix_trans(pack_f16(pr[2], pr[3]));
    }
    // token pairs of the A fragments: (2c, 2c+1) and (2c+8, 2c+9)
    uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
    const bool partial = vm != 0xFFFFu;
    if (partial) {
      mlo = ((vm >> (2 * c)) & 1u ? 0x0000FFFFu : 0u) | ((vm >> (2 * c + 1)) & 1u ? 0xFFFF0000u : 0u);
      mhi = ((vm >> (2 * c + 8)) & 1u ? 0x0000FFFFu : 0u) | ((vm >> (2 * c + 9)) & 1u ? 0xFFFF0000u : 0u);
    }
    if constexpr (CACHE == TC_BF16) {
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        uint32_t af[4];
        ldmatrix_x4_trans(af, vt + (voff ^ ((mt & 3) << 5)) + (mt >> 2) * 2048);
        af[0] &= mlo;
        af[1] &= mlo;
        af[2] &= mhi;
        af[3] &= mhi;
        mma_bf16(acc[mt], af, pb0, pb1);
      }
    } else if constexpr (CACHE == TC_KIVI) {
      // lane (g, c) reads word g (dims 16g .. 16g+15, byte j = dims 16g + 4j ..
      // + 3) of token rows 2c, 2c+1, 2c+8, 2c+9 (32-byte rows).  Bytes (2J,
      // 2J+1) of the row pair side by side; code s of byte 2J is dim 16g + 8J
      // + s (m-tile row g), of byte 2J+1 dim 16g + 8J + 4 + s (row g+8)
      const uint32_t vb = vt + 64 * c + 4 * g;
      const uint32_t x0 = lds32(vb), y0 = lds32(vb + 32), x1 = lds32(vb + 256), y1 = lds32(vb + 288);
#pragma unroll
      for (int J = 0; J < 2; ++J) {
        const uint32_t sel = J ? 0x7632u : 0x5410u;
        const uint32_t z0 = prmt(x0, y0, sel), z1 = prmt(x1, y1, sel);
        const uint32_t h0 = z0 >> 8, h1 = z1 >> 8;
#pragma unroll
        for (int s2 = 0; s2 < 4; ++s2) {
          // codes are finite and masked tokens carry P = 0: no V mask needed.
          // Unpacked where they sit, m-tile 4J + s2 holds 4^s2 times the
          // values (v_unscale takes the factor out at the end)
          const uint32_t af[4] = {i2x2_at_to_f16x2(z0, s2), i2x2_at_to_f16x2(h0, s2), i2x2_at_to_f16x2(z1, s2),
                                  i2x2_at_to_f16x2(h1, s2)};
          mma_f16(acc[4 * J + s2], af, pb0, pb1);
        }
      }
    } else if constexpr (CACHE == TC_INT4) {
      // lane (g, c) reads dims 16g .. 16g+15 (8 bytes at byte 8g, in chunk g/2)
      // of token rows 2c, 2c+1, 2c+8, 2c+9 (64-byte rows, 64-byte swizzle)
      auto row8 = [&](int r) {
        return lds64(vt + r * 64 + ((uint32_t)((g >> 1) ^ ((r >> 1) & 3)) << 4) + (g & 1) * 8);
      };
      const uint2 x0 = row8(2 * c), y0 = row8(2 * c + 1), x1 = row8(2 * c + 8), y1 = row8(2 * c + 9);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        // dims 16g + 2mt (+1): byte mt of the 8, low (high) nibble; tokens side by
        // side.  The high nibbles are unpacked where they sit, as 16 times the
        // codes (v_unscale takes the factor out of rows g + 8 at the end)
        const int wi = mt >> 2, b = mt & 3;
        const uint32_t sel = b | (b << 4) | ((4 + b) << 8) | ((4 + b) << 12);
        const uint32_t z0 = prmt((&x0.x)[wi], (&y0.x)[wi], sel);
        const uint32_t z1 = prmt((&x1.x)[wi], (&y1.x)[wi], sel);
        uint32_t af[4];
        // codes are finite and masked tokens carry P = 0: no V mask needed
        af[0] = i4x2_at_to_f16x2<false>(z0);
        af[1] = i4x2_at_to_f16x2<true>(z0);
        af[2] = i4x2_at_to_f16x2<false>(z1);
        af[3] = i4x2_at_to_f16x2<true>(z1);
        mma_f16(acc[mt], af, pb0, pb1);
      }
    } else {
      // lane (g, c) reads chunk g of token rows 2c, 2c+1, 2c+8, 2c+9
      const uint32_t mlo5 = mlo & 0xFF00FF00u, mhi5 = mhi & 0xFF00FF00u;
      const uint4 x0 = lds128(vt + voff);
      const uint4 y0 = lds128(vt + (voff ^ 16) + 128);
      const uint4 x1 = lds128(vt + voff + 1024);
      const uint4 y1 = lds128(vt + (voff ^ 16) + 1152);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int wi = mt >> 1;
        uint32_t af[4];
        if constexpr (CACHE == TC_INT8) {
          const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
          const uint32_t ta = prmt((&x0.x)[wi], (&y0.x)[wi], sel) ^ 0x80808080u;
          const uint32_t tb = prmt((&x1.x)[wi], (&y1.x)[wi], sel) ^ 0x80808080u;
          af[0] = i8x2_to_f16x2(ta, 0x4140);
          af[1] = i8x2_to_f16x2(ta, 0x4342);
          af[2] = i8x2_to_f16x2(tb, 0x4140);
          af[3] = i8x2_to_f16x2(tb, 0x4342);
        } else if constexpr (CACHE == TC_E5M2) {
          // byte A of the token-2c row into bits [15:8], of the token-2c+1 row into [31:24]
          const uint32_t A = 2 * (mt & 1);
          const uint32_t s0 = ((4 + A) << 12) | ((4 + A) << 8) | (A << 4) | A;
          const uint32_t s1 = s0 + 0x1111u;
          af[0] = prmt((&x0.x)[wi], (&y0.x)[wi], s0);
          af[1] = prmt((&x0.x)[wi], (&y0.x)[wi], s1);
          af[2] = prmt((&x1.x)[wi], (&y1.x)[wi], s0);
          af[3] = prmt((&x1.x)[wi], (&y1.x)[wi], s1);
          // E5M2 bytes are the f16 top bytes: clear the duplicated low bytes, and
          // the rows past the attended ones (their codes may be inf or NaN)
          af[0] &= mlo5;
          af[1] &= mlo5;
          af[2] &= mhi5;
          af[3] &= mhi5;
        } else {
          // E4M3: bytes A and A+1 of the token-2c and token-2c+1 rows as two
          // pairs [2c, 2c+1] through the hardware conversion; rows past the
          // attended ones may hold NaN codes, so partial blocks are masked
          const uint32_t A = 2 * (mt & 1);
          const uint32_t sel = A | ((4 + A) << 4) | ((A + 1) << 8) | ((5 + A) << 12);
          e4m3x4_to_f16x2x2(prmt((&x0.x)[wi], (&y0.x)[wi], sel), af[0], af[1]);
          e4m3x4_to_f16x2x2(prmt((&x1.x)[wi], (&y1.x)[wi], sel), af[2], af[3]);
          if (partial) {
            af[0] &= mlo;
            af[1] &= mlo;
            af[2] &= mhi;
            af[3] &= mhi;
          }
        }
        // INT8 values decode finite whatever the bytes, and masked tokens
        // carry P = 0, so they need no V mask
        mma_f16(acc[mt], af, pb0, pb1);
      }
    }
  };

  // One step over NB (1 or 2) consecutive blocks of the current unit: their
  // scores, one online-softmax update, then their P.V.  Two blocks give each
  // warp two independent MMA chains.  Returns false if a wait timed out.
  int it = 0;
  int cstage = 0;      // ring stage of block `it`
  uint32_t cpass = 0;  // parity of the ring pass of block `it`
  auto step = [&](auto nb_const) -> bool {
    constexpr int NB = decltype(nb_const)::value;
    const uint8_t* st[NB];
    int stage[NB];
    uint32_t valid[NB];  // attended-row masks
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      int sk = cstage + k;
      uint32_t pk = cpass;
      if (sk >= p.stages) {
        sk -= p.stages;
        pk ^= 1u;
      }
      stage[k] = sk;
      if (!mbar_wait(&full[sk], pk, p.wait_limit)) return false;
      st[k] = smem + (size_t)sk * p.stage_bytes;
      if constexpr (CACHE == TC_KIVI)
        valid[k] = 0xFFFFu;  // full blocks only
      else if (p.pages)
        valid[k] = (j + k + 1 == P[u + 1] - P[u]) ? token_mask(aset, L, last_page) : 0xFFFFu;
      else
        valid[k] = token_mask(aset, L, logical_block(aset, j + k));
    }
    float sv[NB][4], vsc[NB][2];
#pragma unroll
    for (int k = 0; k < NB; ++k) block_scores(st[k], valid[k], sv[k], vsc[k]);

    // The reference max m of each head moves only when some score exceeds it by
    // more than kLazyLog2, so probabilities stay <= 2^kLazyLog2 and most steps
    // skip the cross-lane max and the rescale of the accumulators; the final
    // o / l and lse = m + log2(l) do not depend on which m was used.
    float mx0 = fmaxf(sv[0][0], sv[0][2]), mx1 = fmaxf(sv[0][1], sv[0][3]);
#pragma unroll
    for (int k = 1; k < NB; ++k) {
      mx0 = fmaxf(mx0, fmaxf(sv[k][0], sv[k][2]));
      mx1 = fmaxf(mx1, fmaxf(sv[k][1], sv[k][3]));
    }
    if (__any_sync(0xffffffffu, mx0 > m0 + kLazyLog2 || mx1 > m1 + kLazyLog2)) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      l0 *= al0;
      l1 *= al1;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        acc[mt][0] *= al0;
        acc[mt][1] *= al1;
        acc[mt][2] *= al0;
        acc[mt][3] *= al1;
      }
    }
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      float pr[4];
      pr[0] = ex2(sv[k][0] - m0);
      pr[1] = ex2(sv[k][1] - m1);
      pr[2] = ex2(sv[k][2] - m0);
      pr[3] = ex2(sv[k][3] - m1);
      l0 += pr[0] + pr[2];
      l1 += pr[1] + pr[3];
      block_pv(st[k], valid[k], pr, vsc[k]);
    }
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < NB; ++k) mbar_arrive(&empty[stage[k]]);
    }
    return true;
  };

  int i = a;
  while (i < b) {
    if (i == a || j == 0) {
      // ---- unit start: this warp's 8 query rows as MMA B fragments
      if (j == 0 && warp == 0 && lane == 0) {
        // this CTA holds the unit's first block: record its pieces for the merge
        const int c1 = (P[u + 1] - 1) / per;
        p.desc[u] = make_int2((int)blockIdx.x | ((P[u] % per) != 0 ? (1 << 30) : 0), c1 - (int)blockIdx.x + 1);
      }
      s = u / p.HG;
      hg = u - s * p.HG;
      L = seq_len(p, s, false);
      aset = attend_set(p, L);
      if (p.pages)  // only the list's last entry can be the sequence's partial last page
        last_page = __ldg(p.pages + ((size_t)s * p.n_kv + hg) * p.k_pages + (P[u + 1] - P[u] - 1));
      if constexpr (CACHE == TC_BF16) {
        fetch_query(u);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qf[ks][0] = qraw[ks][0];
          qf[ks][1] = qraw[ks][1];
        }
      } else if constexpr (tc_fp8(CACHE)) {
        // the query as f16 pairs in the order of the FP8 K fragments; the codes
        // become f16 of their exact values, so the per-head scales apply as they are
        const int kv = hg * p.HPC + head_local;
        if (p.act_bf16) {
          fetch_query(u);
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            qf[ks][0] = pack_f16(__uint_as_float(qraw[ks][0] << 16), __uint_as_float(qraw[ks][0] & 0xFFFF0000u));
            qf[ks][1] = pack_f16(__uint_as_float(qraw[ks][1] << 16), __uint_as_float(qraw[ks][1] & 0xFFFF0000u));
          }
        } else {
          const bool q_ok = qc * 8 + g < p.G;
          const float* qrow = reinterpret_cast<const float*>(p.query) + ((size_t)s * p.n_q + kv * p.G + qc * 8 + g) * D;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int d0 = (2 * c + (ks >> 2)) * 16 + 4 * (ks & 3);
            float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q_ok) w = __ldg(reinterpret_cast<const float4*>(qrow + d0));
            qf[ks][0] = pack_f16(w.x, w.y);
            qf[ks][1] = pack_f16(w.z, w.w);
          }
        }
        head_k_scale = __ldg(p.k_scale + kv);
        head_v_scale = __ldg(p.v_scale + kv);
      }
      if constexpr (tc_row_scaled(CACHE)) {
        // this lane's 32 dims 32c .. 32c+31 of query head g, quantised per head:
        // t = q * 127 / max|q|, h = rint(t), l = rint((t - h) * 254), both in
        // [-127, 127], so q = max|q| / 127 * (h + l / 254) to 1 part in 32000
        const int kvq = hg * p.HPC + head_local;
        const bool q_ok = qc * 8 + g < p.G;
        const size_t qoff = ((size_t)s * p.n_q + kvq * p.G + qc * 8 + g) * D + 32 * c;
        float x[32];
        if (p.act_bf16) {
          const uint4* q4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.query) + qoff);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint4 w = q_ok ? __ldg(q4 + i) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              x[8 * i + 2 * k] = __uint_as_float(wv[k] << 16);
              x[8 * i + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
            }
          }
        } else {
          const float4* q4 = reinterpret_cast<const float4*>(static_cast<const float*>(p.query) + qoff);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w = q_ok ? __ldg(q4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            x[4 * i] = w.x;
            x[4 * i + 1] = w.y;
            x[4 * i + 2] = w.z;
            x[4 * i + 3] = w.w;
          }
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        int hsum = 0, lsum = 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          int hv[8], lv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float t = x[8 * kk + e] * inv;
            const float hq = rintf(t);
            hv[e] = (int)hq;
            lv[e] = (int)rintf((t - hq) * 254.f);
            hsum += hv[e];
            lsum += lv[e];
          }
          if constexpr (CACHE == TC_INT8) {
            // k-step kk: dims 32c + 8kk + {0..3} and {4..7}, as the stored bytes
            qh[kk][0] = pack_s8x4(hv[0], hv[1], hv[2], hv[3]);
            qh[kk][1] = pack_s8x4(hv[4], hv[5], hv[6], hv[7]);
            ql[kk][0] = pack_s8x4(lv[0], lv[1], lv[2], lv[3]);
            ql[kk][1] = pack_s8x4(lv[4], lv[5], lv[6], lv[7]);
          } else {
            // k-step kk: even and odd nibbles of the INT4 word kk (dims 32c + 8kk + {0,2,4,6}, {1,3,5,7})
            qh[kk][0] = pack_s8x4(hv[0], hv[2], hv[4], hv[6]);
            qh[kk][1] = pack_s8x4(hv[1], hv[3], hv[5], hv[7]);
            ql[kk][0] = pack_s8x4(lv[0], lv[2], lv[4], lv[6]);
            ql[kk][1] = pack_s8x4(lv[1], lv[3], lv[5], lv[7]);
          }
        }
        hsum += __shfl_xor_sync(0xffffffffu, hsum, 1);
        hsum += __shfl_xor_sync(0xffffffffu, hsum, 2);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
        lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
        // score columns are heads 2c and 2c+1: their values live on lanes 8c and 8c + 4
        const float qsc = amax * (1.f / 127.f);
        qs0 = __shfl_sync(0xffffffffu, qsc, 8 * c);
        qs1 = __shfl_sync(0xffffffffu, qsc, 8 * c + 4);
        if constexpr (CACHE == TC_INT4) {
          ch0 = 8 * __shfl_sync(0xffffffffu, hsum, 8 * c);
          ch1 = 8 * __shfl_sync(0xffffffffu, hsum, 8 * c + 4);
          cl0 = 8 * __shfl_sync(0xffffffffu, lsum, 8 * c);
          cl1 = 8 * __shfl_sync(0xffffffffu, lsum, 8 * c + 4);
        }
      }
      if constexpr (CACHE == TC_KIVI) {
        // this lane's dims 32c .. 32c+31 of query head g as f16 pairs in the
        // order of the 2-bit K fragments (see block_scores); the block's
        // channel scales multiply them per block
        const int kvq = hg * p.HPC + head_local;
        const bool q_ok = qc * 8 + g < p.G;
        const size_t qoff = ((size_t)s * p.n_q + kvq * p.G + qc * 8 + g) * D + 32 * c;
        const uint4* q4 = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.query) + qoff);
        float x[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 w = q_ok ? __ldg(q4 + i) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[8 * i + 2 * k] = __uint_as_float(wv[k] << 16);
            x[8 * i + 2 * k + 1] = __uint_as_float(wv[k] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          // the K codes of k-step ks come as 4^s0 and 4^(s0+1) times their values
          // (s0 = 2 (ks & 1)): the query parts take 4^-s0 and 4^-(s0+1)
          const int e = 16 * (ks >> 2) + 4 * ((ks >> 1) & 1) + 2 * (ks & 1);
          const float f0 = (ks & 1) ? 1.f / 16.f : 1.f, f1 = (ks & 1) ? 1.f / 64.f : 0.25f;
          qf[ks][0] = pack_f16(x[e] * f0, x[e + 8] * f0);
          qf[ks][1] = pack_f16(x[e + 1] * f1, x[e + 9] * f1);
        }
      }
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      if (p.pre_o != nullptr && j == 0) {
        // the piece holding the unit's first block starts from the shared-prefix
        // state (normalised o, base-2 lse) of this lane's heads 2c, 2c+1: m = lse,
        // acc = o, l = 1, the sum counted on lane g == 0 only
        const int kvh = hg * p.HPC + head_local;
        const size_t r0 = (size_t)kvh * p.pre_rows + (size_t)s * p.G + qc * 8 + 2 * c;
        const float* o0 = p.pre_o + r0 * D;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int dd = d_of<CACHE, D>(mt, hi, g);
            const float f = 1.f / v_unscale<CACHE>(mt, hi);
            if (head0_ok) acc[mt][2 * hi] = __ldcg(o0 + dd) * f;
            if (head1_ok) acc[mt][2 * hi + 1] = __ldcg(o0 + D + dd) * f;
          }
        }
        if (head0_ok) m0 = __ldcg(p.pre_lse + r0);
        if (head1_ok) m1 = __ldcg(p.pre_lse + r0 + 1);
        l0 = (g == 0 && head0_ok) ? 1.f : 0.f;
        l1 = (g == 0 && head1_ok) ? 1.f : 0.f;
      }
    }

    const int uend = P[u + 1];
    const int nb = (i + 1 < b && i + 1 < uend) ? 2 : 1;
    const bool ok = nb == 2 ? step(std::integral_constant<int, 2>{}) : step(std::integral_constant<int, 1>{});
    if (!ok) {
      flag_error(p.err, DEVERR_TIMEOUT);
      break;
    }
    i += nb;
    it += nb;
    j += nb;
    cstage += nb;
    if (cstage >= p.stages) {
      cstage -= p.stages;
      cpass ^= 1u;
    }

    // ---- unit end: finish here, or hand a piece to the merge
    const bool unit_end = (i == uend);
    if (unit_end || i == b) {
      float lt0 = l0, lt1 = l1;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        lt0 += __shfl_xor_sync(0xffffffffu, lt0, o);
        lt1 += __shfl_xor_sync(0xffffffffu, lt1, o);
      }
      if constexpr (CACHE == TC_INT4 || CACHE == TC_KIVI) {
        // the factors of the codes unpacked in place (the range ends here)
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            acc[mt][2 * hi] *= v_unscale<CACHE>(mt, hi);
            acc[mt][2 * hi + 1] *= v_unscale<CACHE>(mt, hi);
          }
        }
      }
      const float post = tc_fp8(CACHE) ? head_v_scale : 1.f;
      const float inv0 = post / lt0, inv1 = post / lt1;
      const float lse0 = m0 + log2f(lt0), lse1 = m1 + log2f(lt1);
      const bool contained = P[u] >= a && P[u + 1] <= b;
      const long long row0 = (long long)s * p.n_q + hg * QH + qbase_local + 2 * c;  // head 2c of this lane
      if (contained && p.merge_all) {
        // the whole unit's piece, for the merge with the shared prefix's pieces
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int dd = d_of<CACHE, D>(mt, hi, g);
            if (head0_ok) __stcg(p.unit_o + row0 * D + dd, acc[mt][2 * hi] * inv0);
            if (head1_ok) __stcg(p.unit_o + (row0 + 1) * D + dd, acc[mt][2 * hi + 1] * inv1);
          }
        }
        if (g == 0) {
          if (head0_ok) __stcg(p.unit_lse + row0, lse0);
          if (head1_ok) __stcg(p.unit_lse + row0 + 1, lse1);
        }
      } else if (contained) {
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int dd = d_of<CACHE, D>(mt, hi, g);
            const float v0 = acc[mt][2 * hi] * inv0, v1 = acc[mt][2 * hi + 1] * inv1;
            if (p.act_bf16) {
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(p.out);
              if (head0_ok) o[row0 * D + dd] = __float2bfloat16_rn(v0);
              if (head1_ok) o[(row0 + 1) * D + dd] = __float2bfloat16_rn(v1);
            } else {
              float* o = reinterpret_cast<float*>(p.out);
              if (head0_ok) o[row0 * D + dd] = v0;
              if (head1_ok) o[(row0 + 1) * D + dd] = v1;
            }
          }
        }
        if (p.lse_out && g == 0) {
          if (head0_ok) p.lse_out[row0] = lse0 * kLn2;
          if (head1_ok) p.lse_out[row0 + 1] = lse1 * kLn2;
        }
      } else {
        const int slot = (u == u_first) ? 0 : 1;
        const size_t pbase = ((size_t)blockIdx.x * 2 + slot) * QH + qbase_local + 2 * c;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int dd = d_of<CACHE, D>(mt, hi, g);
            if (head0_ok) __stcg(p.part_o + pbase * D + dd, acc[mt][2 * hi] * inv0);
            if (head1_ok) __stcg(p.part_o + (pbase + 1) * D + dd, acc[mt][2 * hi + 1] * inv1);
          }
        }
        if (g == 0) {
          if (head0_ok) __stcg(p.part_lse + pbase, lse0);
          if (head1_ok) __stcg(p.part_lse + pbase + 1, lse1);
        }
      }
    }
    if (unit_end) {
      ++u;
      while (u < units && P[u + 1] == P[u]) ++u;
      j = 0;
    }
  }
}

// ----------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Rank-3 view of a cache pool [num_blocks * 16 rows][n_kv * head_dim * elem
// bytes] as (elements of one chunk, chunk index, token row), box = 1 chunk x 16
// rows.  A chunk is 128 bytes (BF16 / INT8 / FP8 rows, 128-byte swizzle), or a
// whole head row: 64 bytes of INT4 (64-byte swizzle) or 32 bytes of 2-bit
// codes (no swizzle; the decode reads the head-major 2-bit pools with bulk
// copies, so that map is only passed along).
pkv_status make_pool_map(CUtensorMap* map, const void* base, int elem, int chunk_bytes, int row_bytes_i,
                              int64_t rows) {
  auto fn = encode_fn();
  if (!fn) return driver_fail(-1, "cuTensorMapEncodeTiled entry point");
  const cuuint64_t row_bytes = (cuuint64_t)row_bytes_i;
  const cuuint64_t cb = (cuuint64_t)chunk_bytes;
  cuuint64_t dims[3] = {cb / elem, row_bytes / cb, (cuuint64_t)rows};
  cuuint64_t strides[2] = {cb, row_bytes};
  cuuint32_t box[3] = {(cuuint32_t)(cb / elem), 1, (cuuint32_t)kBlockSize};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  chunk_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                  : chunk_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                      : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return driver_fail((int)r, "cuTensorMapEncodeTiled");
  return PKV_OK;
}

// The 2-bit cache's K scales [num_blocks * n_kv * 4 rows][32 floats] as a
// rank-2 map, box = 32 floats x (4 * heads_per_cta) rows, 128-byte swizzle.
static pkv_status make_kivi_scale_map(CUtensorMap* map, const float* k_scale, int64_t num_blocks, int n_kv, int hpc) {
  auto fn = encode_fn();
  if (!fn) return driver_fail(-1, "cuTensorMapEncodeTiled entry point");
  cuuint64_t dims[2] = {32, (cuuint64_t)num_blocks * n_kv * 4};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {32, (cuuint32_t)(4 * hpc)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(k_scale), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return driver_fail((int)r, "cuTensorMapEncodeTiled(k_scale)");
  return PKV_OK;
}

template <int CACHE, int D, int MAXW, int MINB = 1>
static pkv_status launch_variant(const TcPlan& plan, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& sm,
                                 const TcParams& prm, const PrefixPieces& pre, cudaStream_t stream) {
  auto kern = decode_tc_kernel<CACHE, D, MAXW, MINB>;
  auto merge = decode_merge_kernel<D, 1>;
  auto merge_all = decode_merge_all_kernel<D, 1>;
  auto merge_wide = decode_merge_kernel<D, kMergeLanes>;
  auto merge_all_wide = decode_merge_all_kernel<D, kMergeLanes>;
  static int configured_bytes = 0;  // max dynamic smem already granted to this instantiation
  if ((int)plan.smem_bytes > configured_bytes) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan.smem_bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    if (configured_bytes == 0) {
      // the whole shared memory of an SM for the step's kernels (see prefer_max_smem)
      e = prefer_max_smem(kern);
      if (e == cudaSuccess) e = prefer_max_smem(merge);
      if (e == cudaSuccess) e = prefer_max_smem(merge_all);
      if (e == cudaSuccess) e = prefer_max_smem(merge_wide);
      if (e == cudaSuccess) e = prefer_max_smem(merge_all_wide);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
    }
    configured_bytes = (int)plan.smem_bytes;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(plan.num_ctas);
  cfg.blockDim = dim3((plan.NCW + 1) * 32);
  cfg.dynamicSmemBytes = plan.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = plan.overlap_prologue ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, sm, prm);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode_tc_kernel launch");

  // The merge of split units, allowed to become resident while the decode
  // kernel runs; it waits for the decode kernel's completion on the device.
  MergeParams mp;
  mp.out = prm.out;
  mp.lse_out = prm.lse_out;
  mp.part_o = prm.part_o;
  mp.part_lse = prm.part_lse;
  mp.desc = prm.desc;
  mp.HG = plan.HG;
  mp.QH = plan.HPC * plan.G;
  mp.n_q = prm.n_q;
  mp.num_ctas = plan.num_ctas;
  mp.act_bf16 = prm.act_bf16;
  mp.merge_all = prm.merge_all;
  mp.unit_o = prm.unit_o;
  mp.unit_lse = prm.unit_lse;
  mp.pre_o = pre.o;
  mp.pre_lse = pre.lse;
  mp.pre_rows = pre.rows;
  mp.pre_splits = pre.splits;
  mp.G = plan.G;
  mp.HPC = plan.HPC;
  // Pieces a unit is expected to have, with every sequence at the longest
  // length: about num_ctas / units + 1 (plus the prefix's splits).  Past
  // kMergeBatch, kMergeLanes lanes share each (query head, 4 dims), if the
  // threads that takes still fit the GPU at once (few, long units).
  const int pieces_est = (plan.num_ctas + plan.units - 1) / std::max(1, plan.units) + 1 + (prm.merge_all ? pre.splits : 0);
  const long long wide_threads = (long long)plan.units * mp.QH * (D / 4) * kMergeLanes;
  const int lanes = pieces_est > kMergeBatch && wide_threads <= 1024LL * device_sm_count() ? kMergeLanes : 1;
  const int threads = mp.QH * (D / 4) * lanes;
  cudaLaunchConfig_t mcfg = {};
  // up to 512 threads a CTA, as many CTAs per unit as the threads take; at
  // most 64 registers a thread, so that 1024 threads of merge CTAs fit an SM
  mcfg.blockDim = dim3((unsigned)std::min(512, (threads + 31) / 32 * 32));
  mcfg.gridDim = dim3(plan.units, (unsigned)((threads + (int)mcfg.blockDim.x - 1) / (int)mcfg.blockDim.x));
  mcfg.dynamicSmemBytes = 0;
  mcfg.stream = stream;
  cudaLaunchAttribute mattr[1];
  mattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  mattr[0].val.programmaticStreamSerializationAllowed = 1;
  mcfg.attrs = mattr;
  mcfg.numAttrs = 1;
  if (lanes == 1)
    e = prm.merge_all ? cudaLaunchKernelEx(&mcfg, merge_all, mp) : cudaLaunchKernelEx(&mcfg, merge, mp);
  else
    e = prm.merge_all ? cudaLaunchKernelEx(&mcfg, merge_all_wide, mp) : cudaLaunchKernelEx(&mcfg, merge_wide, mp);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode_merge_kernel launch");
  return PKV_OK;
}

// Up to 8 consumer warps use the variant whose launch bound leaves ~220
// registers per thread; wider CTAs take the 16-warp variant.  Quantised
// caches, bound by dequantisation work, run 3 CTAs of up to 4 consumer warps
// per SM (launch bound: at most 136 registers a thread) for more warps in
// flight: 15 warps per SM instead of 12 (INT4 -13 %, INT8 and E4M3 -5 %).
template <int CACHE, int D>
static pkv_status launch_one(const TcPlan& plan, const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& sm,
                             const TcParams& prm, const PrefixPieces& pre, cudaStream_t stream) {
  if constexpr (tc_narrow(CACHE)) {
    if (plan.NCW <= 4) return launch_variant<CACHE, D, 4, kQuantCtasPerSm>(plan, km, vm, sm, prm, pre, stream);
  }
  if (plan.NCW <= 8) return launch_variant<CACHE, D, 8>(plan, km, vm, sm, prm, pre, stream);
  return launch_variant<CACHE, D, kMaxConsumerWarps>(plan, km, vm, sm, prm, pre, stream);
}

pkv_status launch_tc(const DecodeShape& s, const TcPlan& plan, const TcArgs& a, cudaStream_t stream) {
  const int elem = plan.cache_kind == TC_BF16 ? 2 : 1;
  const bool int4 = plan.cache_kind == TC_INT4, kivi = plan.cache_kind == TC_KIVI;
  const int row_bytes = int4 ? s.n_kv * s.head_dim / 2 : kivi ? s.n_kv * s.head_dim / 4 : s.n_kv * s.head_dim * elem;
  const int chunk_bytes = int4 ? s.head_dim / 2 : kivi ? s.head_dim / 4 : 128;
  const int64_t rows = a.num_blocks * kBlockSize;
  CUtensorMap km, vm, sm;
  pkv_status st = make_pool_map(&km, a.key_cache, elem, chunk_bytes, row_bytes, rows);
  if (st != PKV_OK) return st;
  st = make_pool_map(&vm, a.value_cache, elem, chunk_bytes, row_bytes, rows);
  if (st != PKV_OK) return st;
  if (kivi) {
    st = make_kivi_scale_map(&sm, a.k_scale, a.num_blocks, s.n_kv, plan.HPC);
    if (st != PKV_OK) return st;
  } else {
    sm = km;  // unused
  }
  const long long wait_limit = a.wait_limit > 0 ? a.wait_limit : kWaitLimitCycles;
  PrefixPieces pieces;
  const bool shared_prefix = a.skip_blocks > 0 && a.prefix_ws;
  if (shared_prefix) {
    // The shared prefix's pass first; the decode over each sequence's own
    // blocks, queued with programmatic serialisation, runs beside it (or after
    // it, prefix_serial), and the merge combines both sides' pieces.
    st = launch_prefix(s, km, vm, a, wait_limit, &pieces, stream);
    if (st != PKV_OK) return st;
  }

  TcParams prm;
  prm.out = a.out;
  prm.query = a.query;
  prm.k_scale = const_cast<float*>(a.k_scale);
  prm.v_scale = const_cast<float*>(a.v_scale);
  prm.new_key = a.new_key;
  prm.new_value = a.new_value;
  prm.key_cache = const_cast<void*>(a.key_cache);
  prm.value_cache = const_cast<void*>(a.value_cache);
  prm.block_tables = a.block_tables;
  prm.context_lens = a.context_lens;
  prm.lse_out = a.lse_out;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  prm.desc = reinterpret_cast<int2*>(ws + plan.ws_desc);
  prm.part_o = reinterpret_cast<float*>(ws + plan.ws_part_o);
  prm.part_lse = reinterpret_cast<float*>(ws + plan.ws_part_lse);
  prm.err = a.device_error;
  prm.num_blocks = a.num_blocks;
  prm.max_blocks_per_seq = a.max_blocks_per_seq;
  prm.max_context_len = a.max_context_len;
  prm.cap_len = (int)std::min<int64_t>(a.max_context_len, (int64_t)a.max_blocks_per_seq * kBlockSize);
  prm.num_seqs = s.num_seqs;
  prm.n_q = s.n_q;
  prm.n_kv = s.n_kv;
  prm.window = a.window;
  prm.sinks = a.sinks;
  prm.pages = a.pages;
  prm.k_pages = a.k_pages;
  prm.skip_blocks = a.skip_blocks;
  prm.merge_all = shared_prefix ? 1 : 0;
  prm.unit_o = pieces.unit_o;
  prm.unit_lse = pieces.unit_lse;
  prm.late_wait = shared_prefix && !a.prefix_serial ? 1 : 0;
  prm.wait_limit = wait_limit;
  prm.pre_o = a.prefix.o;
  prm.pre_lse = a.prefix.lse;
  prm.pre_rows = a.prefix.rows;
  prm.whole_blocks = kivi ? 1 : 0;
  prm.G = plan.G;
  prm.QC = plan.QC;
  prm.HPC = plan.HPC;
  prm.HG = plan.HG;
  prm.NCW = plan.NCW;
  prm.stages = plan.stages;
  prm.units = plan.units;
  prm.scale_log2 = (float)((double)a.sm_scale * 1.4426950408889634);
  prm.act_bf16 = s.act == PKV_BF16;
  prm.stage_bytes = plan.stage_bytes;
  prm.tx_bytes = plan.tx_bytes;

  if (plan.cache_kind == TC_BF16) {
    if (s.head_dim == 64) return launch_one<TC_BF16, 64>(plan, km, vm, sm, prm, pieces, stream);
    return launch_one<TC_BF16, 128>(plan, km, vm, sm, prm, pieces, stream);
  }
  if (plan.cache_kind == TC_INT8) return launch_one<TC_INT8, 128>(plan, km, vm, sm, prm, pieces, stream);
  if (plan.cache_kind == TC_INT4) return launch_one<TC_INT4, 128>(plan, km, vm, sm, prm, pieces, stream);
  if (plan.cache_kind == TC_E5M2) return launch_one<TC_E5M2, 128>(plan, km, vm, sm, prm, pieces, stream);
  if (plan.cache_kind == TC_KIVI) return launch_one<TC_KIVI, 128>(plan, km, vm, sm, prm, pieces, stream);
  return launch_one<TC_FP8, 128>(plan, km, vm, sm, prm, pieces, stream);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

pkv_status plan_tc(const DecodeShape& s, const pkv_decode_tuning* tuning, TcPlan* plan) {
  TcPlan pl{};
  pl.cache_kind = s.cache == PKV_BF16        ? TC_BF16
                  : s.cache == PKV_INT8      ? TC_INT8
                  : s.cache == PKV_INT4      ? TC_INT4
                  : s.cache == PKV_FP8_E5M2 ? TC_E5M2
                  : s.cache == PKV_KIVI2    ? TC_KIVI
                                             : TC_FP8;
  const int elem = pl.cache_kind == TC_BF16 ? 2 : 1;
  const bool kivi = pl.cache_kind == TC_KIVI;
  pl.chunks = (pl.cache_kind == TC_INT4 || kivi) ? 1 : s.head_dim * elem / 128;
  const size_t tile_bytes = pl.cache_kind == TC_INT4 ? (size_t)s.head_dim / 2 * 16
                            : kivi                   ? (size_t)s.head_dim / 4 * 16
                                                     : (size_t)pl.chunks * 2048;
  pl.G = s.n_q / s.n_kv;
  pl.QC = (pl.G + 7) / 8;
  const int want_hpc = tuning ? tuning->heads_per_cta : 0;
  const size_t scale_bytes = tc_row_scaled(pl.cache_kind) ? 2 * 64 * (size_t)s.n_kv : 0;
  if (want_hpc > 0) {
    if (s.n_kv % want_hpc != 0 || want_hpc * pl.QC > kMaxConsumerWarps) return PKV_ERR_INVALID_ARG;
    pl.HPC = want_hpc;
  } else {
    // Two consumer warps per CTA (2 KV heads when the group fits one warp) and
    // four CTAs per SM measured best for bf16; the quantised caches, whose
    // dequantisation is heavy on the ALUs, do best with four consumer warps per
    // CTA and three CTAs per SM (narrow launch bound, more warps in flight).
    const int warps = tc_narrow(pl.cache_kind) ? 4 : 2;
    pl.HPC = 1;
    for (int h = std::min(s.n_kv, warps); h >= 1; --h) {
      if (s.n_kv % h == 0 && h * pl.QC <= warps) {
        pl.HPC = h;
        break;
      }
    }
  }
  if (pl.HPC * pl.QC > kMaxConsumerWarps) return PKV_ERR_UNSUPPORTED;
  pl.HG = s.n_kv / pl.HPC;
  pl.NCW = pl.HPC * pl.QC;
  pl.units = s.num_seqs * pl.HG;
  // KIVI: the K scales (head_dim floats) and V scales (16 floats) of the CTA's heads
  const size_t kivi_scales = kivi ? (size_t)pl.HPC * s.head_dim * 4 + 64 * (size_t)pl.HPC : 0;
  pl.tx_bytes = (uint32_t)(2 * (size_t)pl.HPC * tile_bytes + scale_bytes + kivi_scales);
  pl.stage_bytes = (uint32_t)align_up(pl.tx_bytes, 1024);

  const int sms = device_sm_count();
  const int optin = device_smem_optin();
  if (sms <= 0 || optin <= 0) return PKV_ERR_CUDA;
  const size_t fixed = align_up(2 * 8 * kMaxStages + 16 + 32 * 4 + ((size_t)pl.units + 1) * 4, 16) + 1024;
  const int want_stages = tuning ? tuning->stages : 0;
  int stages = want_stages;
  if (stages <= 0) {
    // Deepest ring that still lets 4 CTAs share an SM, so the SM keeps its
    // whole shared memory (~190 KB) of K/V in flight; fewer CTAs per SM only
    // when even 2 stages do not fit.
    stages = 2;
    const int target_per_sm = (tc_narrow(pl.cache_kind) && pl.NCW <= 4) ? kQuantCtasPerSm : kTargetCtasPerSm;
    for (int per = target_per_sm; per >= 1; --per) {
      const size_t budget = (size_t)kSmemPerSm / per - 1024;
      if (budget < fixed) continue;
      const int fit = (int)std::min<size_t>(kMaxStages, (budget - fixed) / pl.stage_bytes);
      if (fit >= 2) {
        stages = fit;
        break;
      }
    }
  }
  if (stages < 2 || stages > kMaxStages) return want_stages > 0 ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED;
  pl.stages = stages;
  pl.smem_bytes = (size_t)stages * pl.stage_bytes + fixed;
  if (pl.smem_bytes > (size_t)optin) return want_stages > 0 ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED;
  // CTAs resident per SM from shared memory alone (1 KB reserved per CTA).
  const int per_sm = std::max(1, std::min((tc_narrow(pl.cache_kind) && pl.NCW <= 4) ? kQuantCtasPerSm
                                                                                    : kTargetCtasPerSm,
                                          (int)(kSmemPerSm / (pl.smem_bytes + 1024))));
  const int want_ctas = tuning ? tuning->num_ctas : 0;
  pl.overlap_prologue = tuning && (tuning->flags & PKV_TUNE_OVERLAP_PROLOGUE);
  pl.num_ctas = want_ctas > 0 ? want_ctas : sms * per_sm;
  if (pl.num_ctas > kMaxCtas) return want_ctas > 0 ? PKV_ERR_INVALID_ARG : PKV_ERR_UNSUPPORTED;
  const size_t QH = (size_t)pl.HPC * pl.G;
  // Pieces (two slots per CTA), their lse, one merge descriptor per unit.
  // Every byte read is written earlier in the same call: no zeroing needed.
  pl.ws_part_o = 0;
  pl.ws_part_lse = align_up(pl.ws_part_o + (size_t)pl.num_ctas * 2 * QH * s.head_dim * 4, 256);
  pl.ws_desc = align_up(pl.ws_part_lse + (size_t)pl.num_ctas * 2 * QH * 4, 256);
  pl.ws_total = align_up(pl.ws_desc + (size_t)pl.units * 8, 256);
  *plan = pl;
  return PKV_OK;
}

}  // namespace pkv
