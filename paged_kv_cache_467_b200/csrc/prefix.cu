// Shared-prefix pass of decode attention on the fifth-generation tensor cores.
//
// When every sequence of a batch starts with the same physical blocks (a
// common system prompt: "Chapter 18 - KV-Cache Optimization Strategies",
// Prefix Caching; "KV Cache Engineering for LLM Serving", section 11), the
// attention over those blocks is a dense product: per KV head, the
// R = num_seqs * G query rows against the prefix's tokens.  This pass computes
// it once per KV head for all rows together, so each K/V tile of the prefix is
// read by ceil(R / 128) CTAs instead of by every sequence.
//
// CTA = one KV head, 128 query rows (the MMA's M), one split of the prefix,
// six warps with fixed roles:
//  * a TMA warp streams K and V of 64 tokens (four 16-token blocks) per chunk
//    through a three-stage ring, in the pool's own row layout (K is the K-major
//    B operand of S = Q K^T, V the MN-major B operand of O += P V); its lanes
//    read the split's block-table entries once, up front, and it starts while
//    the softmax warps still load the queries;
//  * an MMA warp issues the tcgen05.mma instructions from one thread: S of a
//    chunk into one of two tensor-memory buffers while the softmax warps still
//    read the other, and P V of the chunk before into the O accumulator
//    [128 x D] (fp32, tensor memory), each committed to mbarriers;
//  * four softmax warps own one query row (one TMEM lane) per thread: a row's
//    64 scores come in by tcgen05.ld, its running max and sum are kept in
//    base 2 (the max moved only past 2^8 of slack, its O row then rescaled in
//    tensor memory), and its bf16 probabilities go to one of two P tiles
//    (the K-major A operand of P V).
//  * Q [128 x D] bf16 sits in shared memory, K-major with the 128-byte swizzle.
// The split's result per row, normalised o and base-2 lse, is one piece of the
// final merge, next to the pieces of the sequence's own blocks.
// The CTAs that hold KV head 0 also check the prefix contract: every
// sequence's first prefix_blocks table entries equal row 0's, and every
// context is longer than the prefix.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "pkv_device.cuh"
#include "tcgen05.cuh"

namespace pkv {

constexpr int kPfxRows = 128;   // query rows per CTA (MMA M, TMEM lanes)
constexpr int kPfxTok = 64;     // tokens per chunk (N of Q K^T, K of P V)
constexpr int kPfxBlocks = kPfxTok / kBlockSize;
constexpr int kPfxStages = 3;
constexpr int kPfxSoftmaxThreads = 128;  // warps 0-3: one query row each
constexpr int kPfxMmaWarp = 4, kPfxTmaWarp = 5;
constexpr int kPfxThreads = 192;
constexpr uint32_t kPfxTmemCols = 256;  // S buffers at columns [0, 64) and [64, 128), O at [128, 128 + D)
constexpr uint32_t kPfxOCol = 128;

template <int D>
struct PfxLayout {
  static constexpr int kDBlk = D / 64;                    // 128-byte column blocks of a bf16 row
  static constexpr uint32_t kQ = kPfxRows * D * 2;        // [dblk][128 rows][128 B]
  static constexpr uint32_t kKV = kPfxTok * D * 2;        // [dblk][64 tokens][128 B]
  static constexpr uint32_t kStage = 2 * kKV;             // K then V
  static constexpr uint32_t kP = kPfxRows * kPfxTok * 2;  // one P tile [128 rows][128 B]
  static constexpr uint32_t kOffStage = kQ;
  static constexpr uint32_t kOffP = kOffStage + kPfxStages * kStage;  // two P tiles
  static constexpr uint32_t kOffBar = kOffP + 2 * kP;
  static constexpr uint32_t kBytes = kOffBar + 256;
  static constexpr uint32_t kSmem = kBytes + 1024;        // slack for 1024-byte alignment
};

struct PrefixParams {
  const __nv_bfloat16* query;    // [num_seqs, n_q, D]
  const int32_t* block_tables;   // the prefix is the first prefix_blocks entries of row 0
  const int32_t* context_lens;
  int* err;
  float* part_o;    // [n_kv][splits][rows][D]
  float* part_lse;  // [n_kv][splits][rows], base 2
  long long num_blocks;
  long long wait_limit;
  int rows, num_seqs, n_q, n_kv, G, prefix_blocks, max_blocks_per_seq;
  int splits, chunks_per_split;
  float scale_log2;
};

// Every sequence shares row 0's first prefix_blocks entries and is longer than
// the prefix; violations set PKV_DEVERR_PREFIX / PKV_DEVERR_CONTEXT_LEN.  The
// CTAs of KV head 0 share the check: this CTA's tile of sequences over its
// split's blocks.
__device__ void check_prefix_contract(const PrefixParams& p, int tile, int b0, int nblk) {
  const int s_first = tile * kPfxRows / p.G;
  const int s_last = min(p.num_seqs - 1, (tile * kPfxRows + kPfxRows - 1) / p.G);
  const int nseq = s_last - s_first + 1;
  bool bad_prefix = false, bad_len = false;
  for (int idx = threadIdx.x; idx < nseq * nblk; idx += blockDim.x) {
    const int s = s_first + idx / nblk, b = b0 + idx % nblk;
    if (s > 0 && __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + b) != __ldg(p.block_tables + b))
      bad_prefix = true;
  }
  if (b0 == 0) {
    for (int s = s_first + (int)threadIdx.x; s <= s_last; s += blockDim.x)
      if (__ldg(p.context_lens + s) <= p.prefix_blocks * kBlockSize) bad_len = true;
  }
  if (bad_prefix) flag_error(p.err, DEVERR_PREFIX);
  if (bad_len) flag_error(p.err, DEVERR_CONTEXT_LEN);
}

template <int D>
__global__ void __launch_bounds__(kPfxThreads, 1)
    prefix_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     const PrefixParams p) {
  using Ly = PfxLayout<D>;
  constexpr int KS = D / 16;  // k-steps of Q K^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_tile = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::kOffBar);  // [stages] K/V chunk landed
  uint64_t* empty = full + kPfxStages;                                // [stages] P V of the chunk done
  uint64_t* s_full = empty + kPfxStages;                              // [2] S buffer written
  uint64_t* s_free = s_full + 2;                                      // [2] S buffer read out
  uint64_t* p_full = s_free + 2;                                      // [2] P tile written (O rescaled)
  uint64_t* p_free = p_full + 2;                                      // [2] P V done with the P tile
  uint64_t* o_done = p_free + 2;                                      // one phase per P V
  uint64_t* bar_done = o_done + 1;                                    // every MMA of the CTA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, kv = blockIdx.y, split = blockIdx.z;
  const int b0 = split * p.chunks_per_split * kPfxBlocks;
  const int b1 = min(b0 + p.chunks_per_split * kPfxBlocks, p.prefix_blocks);
  const int nblk = max(0, b1 - b0);
  const int nchunks = (nblk + kPfxBlocks - 1) / kPfxBlocks;

  // The previous kernel on the stream may still run: wait for it before
  // reading anything, then let the next kernel be scheduled.
  grid_wait_prerequisites();
  grid_launch_dependents();

  if (tid == 0) {
    for (int k = 0; k < kPfxStages; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&s_free[k], kPfxSoftmaxThreads);
      mbar_init(&p_full[k], kPfxSoftmaxThreads);
      mbar_init(&p_free[k], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPfxMmaWarp) {
    tmem_alloc(tmem_slot, kPfxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();  // barriers initialised, TMEM allocated
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem + kPfxOCol;

  // ---- softmax warps: this thread's query row into the K-major swizzled Q
  // tile (16-byte piece j of row r at column block j / 8, position (j % 8) ^ (r % 8))
  const int row = tile * kPfxRows + tid;
  const bool row_ok = tid < kPfxSoftmaxThreads && row < p.rows;
  if (tid < kPfxSoftmaxThreads) {
    const int s = row_ok ? row / p.G : 0, h = row_ok ? row % p.G : 0;
    const uint4* src = reinterpret_cast<const uint4*>(p.query + ((size_t)s * p.n_q + kv * p.G + h) * D);
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint4 v = row_ok ? __ldg(src + j) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t off = (j >> 3) * (kPfxRows * 128) + tid * 128 + (((j & 7) ^ (tid & 7)) << 4);
      *reinterpret_cast<uint4*>(q_tile + off) = v;
    }
    fence_proxy_async_smem();
  }
  // the Q tile is complete once the softmax warps and the MMA warp meet here
  // (the TMA warp does not wait for it)
  if (warp != kPfxTmaWarp) named_barrier(1, kPfxSoftmaxThreads + 32);

  if (warp == kPfxTmaWarp) {
    // ---------------------------------------------------------- TMA warp
    // lane i holds the physical block of the split's blocks b0 + i, b0 + 32 + i, ...
    constexpr int kMaxHeld = 4;  // up to 128 blocks per split held in registers
    int held[kMaxHeld];
#pragma unroll
    for (int r = 0; r < kMaxHeld; ++r) {
      const int b = b0 + r * 32 + lane;
      held[r] = -1;
      if (b < b1) {
        held[r] = __ldg(p.block_tables + b);
        if (held[r] < 0 || (long long)held[r] >= p.num_blocks) {
          flag_error(p.err, DEVERR_BLOCK_RANGE);
          held[r] = -1;
        }
      }
    }
    int issued = 0;
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
    }
    for (; issued < nchunks; ++issued) {
      // the chunk's four physical blocks (-1: past the split or outside the pool)
      int phys4[kPfxBlocks];
#pragma unroll
      for (int i = 0; i < kPfxBlocks; ++i) {
        const int j = issued * kPfxBlocks + i;  // block index inside the split
        int v = -1;
#pragma unroll
        for (int r = 0; r < kMaxHeld; ++r) v = (j >> 5) == r ? held[r] : v;
        phys4[i] = __shfl_sync(0xffffffffu, v, j & 31);
        if (j >= kMaxHeld * 32 && b0 + j < b1) {  // a split longer than the lanes hold: read it here
          phys4[i] = __ldg(p.block_tables + b0 + j);
          if (phys4[i] < 0 || (long long)phys4[i] >= p.num_blocks) {
            if (lane == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
            phys4[i] = -1;
          }
        }
      }
      if (lane == 0) {
        const int k = issued, stage = k % kPfxStages;
        // the stage's previous chunk (k - stages) must have gone through P V
        if (k >= kPfxStages && !mbar_wait(&empty[stage], ((k / kPfxStages) - 1) & 1, p.wait_limit))
          atomicExch(abort_flag, 1);
        uint8_t* kst = smem + Ly::kOffStage + stage * Ly::kStage;
        uint8_t* vst = kst + Ly::kKV;
        if (!*abort_flag) {
          mbar_arrive_expect_tx(&full[stage], Ly::kStage);
#pragma unroll
          for (int i = 0; i < kPfxBlocks; ++i) {
            // blocks past the split, and table entries outside the pool, read as zeros (TMA fill)
#pragma unroll
            for (int db = 0; db < Ly::kDBlk; ++db) {
              const uint32_t off = db * (kPfxTok * 128) + i * (kBlockSize * 128);
              tma_load_3d(kst + off, &kmap, 0, kv * Ly::kDBlk + db, phys4[i] * kBlockSize, &full[stage]);
              tma_load_3d(vst + off, &vmap, 0, kv * Ly::kDBlk + db, phys4[i] * kBlockSize, &full[stage]);
            }
          }
        }
      }
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
    }
    // never leave with copies in flight: the last stages issued have landed
    if (lane == 0) {
      for (int k = max(0, issued - kPfxStages); k < issued; ++k)
        mbar_wait(&full[k % kPfxStages], (k / kPfxStages) & 1);
    }
  } else if (warp == kPfxMmaWarp) {
    // ---------------------------------------------------------- MMA warp
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kPfxRows, kPfxTok, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kPfxRows, D, false, true);
      const uint32_t q_addr = smem_addr(q_tile);
      auto issue_pv = [&](int c) {  // O += P(c) V(c), then free the stage and the P tile
        const uint32_t v_addr = smem_addr(smem + Ly::kOffStage + (c % kPfxStages) * Ly::kStage + Ly::kKV);
        const uint32_t pt = smem_addr(smem + Ly::kOffP + (c & 1) * Ly::kP);
#pragma unroll
        for (int kt = 0; kt < kPfxTok / 16; ++kt) {
          const uint64_t a = umma_desc_sw128(pt + kt * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(v_addr + kt * 2048, kPfxTok * 128, 1024);
          umma_bf16(t_o, a, b, idesc_pv, (c > 0 || kt > 0) ? 1u : 0u);
        }
        umma_commit(&empty[c % kPfxStages]);
        umma_commit(&p_free[c & 1]);
        umma_commit(o_done);
      };
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        ok = mbar_wait(&full[c % kPfxStages], (c / kPfxStages) & 1, p.wait_limit);
        if (ok && c >= 2) ok = mbar_wait(&s_free[c & 1], ((c - 2) >> 1) & 1, p.wait_limit);
        if (!ok) break;
        tc_fence_after_sync();
        // S(c) = Q K(c)^T into S buffer c % 2
        const uint32_t k_addr = smem_addr(smem + Ly::kOffStage + (c % kPfxStages) * Ly::kStage);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint64_t a = umma_desc_sw128(q_addr + (ks >> 2) * (kPfxRows * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(k_addr + (ks >> 2) * (kPfxTok * 128) + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem + (c & 1) * kPfxTok, a, b, idesc_qk, ks > 0);
        }
        umma_commit(&s_full[c & 1]);
        // P V of the chunk before, once its probabilities are written
        if (c >= 1) {
          ok = mbar_wait(&p_full[(c - 1) & 1], ((c - 1) >> 1) & 1, p.wait_limit);
          if (!ok) break;
          tc_fence_after_sync();
          issue_pv(c - 1);
        }
      }
      if (ok && nchunks > 0) {
        ok = mbar_wait(&p_full[(nchunks - 1) & 1], ((nchunks - 1) >> 1) & 1, p.wait_limit);
        if (ok) {
          tc_fence_after_sync();
          issue_pv(nchunks - 1);
        }
      }
      if (!ok) atomicExch(abort_flag, 1);
      // every MMA issued has completed before the CTA moves on
      umma_commit(bar_done);
      mbar_wait(bar_done, 0);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes
    float m = -INFINITY, l = 0.f;                             // running max (log2 units) and sum
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      if (!mbar_wait(&s_full[c & 1], (c >> 1) & 1, p.wait_limit)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      // ---- this row's 64 scores (raw Q K^T); tokens past the split do not count
      uint32_t sr[2][32];
      tmem_ld32(tmem + (c & 1) * kPfxTok + lane_base, sr[0]);
      tmem_ld32(tmem + (c & 1) * kPfxTok + lane_base + 32, sr[1]);
      tmem_wait_ld();
      tc_fence_before_sync();
      mbar_arrive(&s_free[c & 1]);
      const int valid = min(kPfxTok, (nblk - c * kPfxBlocks) * kBlockSize);
      if (valid < kPfxTok) {
#pragma unroll
        for (int j = 0; j < kPfxTok; ++j)
          if (j >= valid) sr[j >> 5][j & 31] = __float_as_uint(-INFINITY);
      }
      // row max over eight independent chains
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = __uint_as_float(sr[0][e]);
#pragma unroll
      for (int j = 8; j < kPfxTok; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(sr[j >> 5][j & 31]));
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx *= p.scale_log2;
      // lazy running max: moved only when a score passes it by more than 2^8;
      // the O row is rescaled once the P V before has completed
      const bool need = c > 0 && mx > m + 8.f;
      if (__any_sync(0xffffffffu, need)) {
        if (!mbar_wait(o_done, (c - 1) & 1, p.wait_limit)) ok = false;
        tc_fence_after_sync();
        const float alpha = need ? ex2_approx(m - mx) : 1.f;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t orow[32];
          tmem_ld32(t_o + lane_base + cb * 32, orow);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) orow[j] = __float_as_uint(__uint_as_float(orow[j]) * alpha);
          tmem_st32(t_o + lane_base + cb * 32, orow);
        }
        tmem_wait_st();
        if (need) {
          l *= alpha;
          m = mx;
        }
      }
      if (c == 0) m = mx;
      // ---- probabilities in bf16 into P tile c % 2 (row tid, K-major, 128-byte swizzle),
      // once the P V two chunks back is done with it
      if (c >= 2 && !mbar_wait(&p_free[c & 1], ((c - 2) >> 1) & 1, p.wait_limit)) ok = false;
      fence_proxy_async_smem();  // the tensor core's reads of this P tile come before these stores
      uint8_t* pt = smem + Ly::kOffP + (c & 1) * Ly::kP;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};  // row sum over four independent chains
#pragma unroll
      for (int j8 = 0; j8 < kPfxTok / 8; ++j8) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = j8 * 8 + 2 * e;
          const float p0 = ex2_approx(fmaf(__uint_as_float(sr[j >> 5][j & 31]), p.scale_log2, -m));
          const float p1 = ex2_approx(fmaf(__uint_as_float(sr[(j + 1) >> 5][(j + 1) & 31]), p.scale_log2, -m));
          ls4[e] += p0 + p1;
          w[e] = pack_bf16(p0, p1);
        }
        *reinterpret_cast<uint4*>(pt + tid * 128 + ((j8 ^ (tid & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(&p_full[c & 1]);
      if (!ok) break;
    }
    // ---- the last P V done: normalised partial o and base-2 lse of this row
    // and split (every lane takes part in the warp-wide loads; rows past the
    // batch store nothing)
    if (ok && nchunks > 0 && !mbar_wait(o_done, (nchunks - 1) & 1, p.wait_limit)) ok = false;
    if (!__all_sync(0xffffffffu, ok)) {
      atomicExch(abort_flag, 1);
    } else {
      tc_fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float4* dst =
          reinterpret_cast<float4*>(p.part_o + (((size_t)kv * p.splits + split) * p.rows + (row_ok ? row : 0)) * D);
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t orow[32];
        tmem_ld32(t_o + lane_base + cb * 32, orow);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[cb * 8 + j] = make_float4(__uint_as_float(orow[4 * j]) * inv, __uint_as_float(orow[4 * j + 1]) * inv,
                                          __uint_as_float(orow[4 * j + 2]) * inv,
                                          __uint_as_float(orow[4 * j + 3]) * inv);
        }
      }
      if (row_ok) p.part_lse[((size_t)kv * p.splits + split) * p.rows + row] = nchunks > 0 ? m + log2f(l) : -INFINITY;
    }
  }

  if (kv == 0) check_prefix_contract(p, tile, b0, nblk);
  tc_fence_before_sync();
  __syncthreads();  // nothing in flight, every TMEM read done
  if (tid == 0 && *abort_flag) flag_error(p.err, DEVERR_TIMEOUT);
  if (warp == kPfxMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kPfxTmemCols);
  }
}

// Splits of the prefix: about one CTA per SM over the (row tile, KV head)
// pairs, each split a whole number of 64-token chunks.
static void prefix_grid(int rows, int n_kv, int prefix_blocks, int want_splits, int* splits, int* chunks_per_split) {
  const int tiles = (rows + kPfxRows - 1) / kPfxRows;
  const int chunks = (prefix_blocks + kPfxBlocks - 1) / kPfxBlocks;
  int sp = want_splits > 0 ? want_splits : std::max(1, std::max(1, device_sm_count()) / std::max(1, tiles * n_kv));
  sp = std::max(1, std::min({sp, chunks, kMaxPrefixSplits}));
  *chunks_per_split = (chunks + sp - 1) / sp;
  *splits = (chunks + *chunks_per_split - 1) / *chunks_per_split;
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t prefix_workspace_bytes(int num_seqs, int n_q, int n_kv, int head_dim, int prefix_blocks, int want_splits) {
  const int rows = num_seqs * (n_q / n_kv);
  int splits = 1, cps = 1;
  prefix_grid(rows, n_kv, prefix_blocks, want_splits, &splits, &cps);
  const size_t part_o = (size_t)n_kv * rows * splits * head_dim * 4;
  const size_t part_l = (size_t)n_kv * rows * splits * 4;
  const size_t unit_o = (size_t)num_seqs * n_q * head_dim * 4;
  const size_t unit_l = (size_t)num_seqs * n_q * 4;
  return align256(part_o) + align256(part_l) + align256(unit_o) + align256(unit_l);
}

// One instantiation per head_dim, each granted its own shared-memory size once.
template <int D>
static pkv_status run_prefix_kernel(dim3 grid, const CUtensorMap& km, const CUtensorMap& vm, const PrefixParams& p,
                                    cudaStream_t stream) {
  constexpr uint32_t smem = PfxLayout<D>::kSmem;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(prefix_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefix)");
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kPfxThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, prefix_tc_kernel<D>, km, vm, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "prefix_tc_kernel launch");
  return PKV_OK;
}

pkv_status launch_prefix(const DecodeShape& s, const CUtensorMap& km, const CUtensorMap& vm, const TcArgs& a,
                         long long wait_limit, PrefixPieces* pieces, cudaStream_t stream) {
  PrefixParams p;
  p.query = static_cast<const __nv_bfloat16*>(a.query);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.err = a.device_error;
  p.num_seqs = s.num_seqs;
  p.n_q = s.n_q;
  p.n_kv = s.n_kv;
  p.G = s.n_q / s.n_kv;
  p.rows = s.num_seqs * p.G;
  p.prefix_blocks = a.skip_blocks;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.num_blocks = a.num_blocks;
  p.wait_limit = wait_limit;
  p.scale_log2 = (float)((double)a.sm_scale * 1.4426950408889634);
  prefix_grid(p.rows, s.n_kv, a.skip_blocks, a.prefix_splits, &p.splits, &p.chunks_per_split);
  uint8_t* ws = static_cast<uint8_t*>(a.prefix_ws);
  const size_t part_o = align256((size_t)s.n_kv * p.rows * p.splits * s.head_dim * 4);
  const size_t part_l = align256((size_t)s.n_kv * p.rows * p.splits * 4);
  const size_t unit_o = align256((size_t)s.num_seqs * s.n_q * s.head_dim * 4);
  p.part_o = reinterpret_cast<float*>(ws);
  p.part_lse = reinterpret_cast<float*>(ws + part_o);
  pieces->o = p.part_o;
  pieces->lse = p.part_lse;
  pieces->splits = p.splits;
  pieces->rows = p.rows;
  pieces->unit_o = reinterpret_cast<float*>(ws + part_o + part_l);
  pieces->unit_lse = reinterpret_cast<float*>(ws + part_o + part_l + unit_o);

  const int tiles = (p.rows + kPfxRows - 1) / kPfxRows;
  const dim3 grid(tiles, s.n_kv, p.splits);
  if (s.head_dim == 128) return run_prefix_kernel<128>(grid, km, vm, p, stream);
  if (s.head_dim == 64) return run_prefix_kernel<64>(grid, km, vm, p, stream);
  return PKV_ERR_UNSUPPORTED;
}

}  // namespace pkv
