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
// seven warps with fixed roles:
//  * two loader warps stream K and V of 64 tokens (four 16-token blocks) per
//    chunk, each through its own three-stage ring, in the pool's own row
//    layout (K is the K-major B operand of S = Q K^T, V the MN-major B operand
//    of O += P V).  K's stage is free again once S of its chunk is done, V's
//    once P V is: K runs ahead of the softmax and V ahead of P V.  Their lanes
//    read the split's block-table entries once, up front;
//  * an MMA warp issues the tcgen05.mma instructions from one thread: S of a
//    chunk into one of two tensor-memory buffers while the softmax warps still
//    read the other, and P V of the chunk before into the O accumulator
//    [128 x D] (fp32, tensor memory), each committed to mbarriers;
//  * four softmax warps own one query row (one TMEM lane) per thread: a row's
//    64 scores come in by tcgen05.ld, its running max and sum are kept in
//    base 2 (the max moved only past 2^8 of slack, its O row then rescaled in
//    tensor memory), and its bf16 probabilities go to one of two P tiles
//    (the K-major A operand of P V).  At the end they stage the normalised O
//    rows in shared memory (128-byte swizzle), then store them row by row.
//  * Q [128 x D] bf16 sits in shared memory, K-major with the 128-byte swizzle.
// The split's result per row, normalised o and base-2 lse, is one piece of the
// final merge, next to the pieces of the sequence's own blocks.
// The CTAs also check the prefix contract, each a share of it: every
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
constexpr int kPfxStages = 3;   // per ring (K, V)
constexpr int kPfxSoftmaxThreads = 128;  // warps 0-3: one query row each
constexpr int kPfxMmaWarp = 4, kPfxKWarp = 5, kPfxVWarp = 6;
constexpr int kPfxThreads = 224;
constexpr uint32_t kPfxTmemCols = 256;  // S buffers at columns [0, 64) and [64, 128), O at [128, 128 + D)
constexpr uint32_t kPfxOCol = 128;

template <int D>
struct PfxLayout {
  static constexpr int kDBlk = D / 64;                    // 128-byte column blocks of a bf16 row
  static constexpr uint32_t kQ = kPfxRows * D * 2;        // [dblk][128 rows][128 B]
  static constexpr uint32_t kKV = kPfxTok * D * 2;        // one stage: [dblk][64 tokens][128 B]
  static constexpr uint32_t kP = kPfxRows * kPfxTok * 2;  // one P tile [128 rows][128 B]
  static constexpr uint32_t kOffK = kQ;                   // K ring, then V ring
  static constexpr uint32_t kOffV = kOffK + kPfxStages * kKV;
  static constexpr uint32_t kOffP = kOffV + kPfxStages * kKV;  // two P tiles
  static constexpr uint32_t kOffBar = kOffP + 2 * kP;
  static constexpr uint32_t kOffTbl = kOffBar + 256;  // each loader warp's copy of the split's block numbers
  static constexpr uint32_t kBytes = kOffTbl + 2 * 128 * 4;
  static constexpr uint32_t kSmem = kBytes + 1024;        // slack for 1024-byte alignment
  // the O rows staged for the row stores, fp32 [D / 32][128 rows][128 B],
  // over the two rings (every load has landed and been read by then)
  static constexpr uint32_t kOffO = kOffK;
  static_assert(kPfxRows * D * 4 <= 2 * kPfxStages * kKV, "O staging fits the rings");
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
// the prefix; violations set PKV_DEVERR_PREFIX / PKV_DEVERR_CONTEXT_LEN.  One
// warp of each CTA checks the sequences s of its row tile with s % n_kv == kv
// over its split's blocks (the splits starting at block 0: their lengths), so
// the CTAs of all KV heads share the work.
__device__ void check_prefix_contract(const PrefixParams& p, int tile, int kv, int b0, int nblk, int lane) {
  const int s_first = tile * kPfxRows / p.G;
  const int s_last = min(p.num_seqs - 1, (tile * kPfxRows + kPfxRows - 1) / p.G);
  int s0 = s_first + ((kv - s_first % p.n_kv) + p.n_kv) % p.n_kv;  // first s >= s_first with s % n_kv == kv
  const int nseq = s0 > s_last ? 0 : (s_last - s0) / p.n_kv + 1;
  bool bad_prefix = false, bad_len = false;
  for (int idx = lane; idx < nseq * nblk; idx += 32) {
    const int s = s0 + (idx / nblk) * p.n_kv, b = b0 + idx % nblk;
    if (s > 0 && __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + b) != __ldg(p.block_tables + b))
      bad_prefix = true;
  }
  if (b0 == 0) {
    for (int i = lane; i < nseq; i += 32)
      if (__ldg(p.context_lens + s0 + i * p.n_kv) <= p.prefix_blocks * kBlockSize) bad_len = true;
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
  uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + Ly::kOffBar);  // [stages] K chunk landed
  uint64_t* empty_k = full_k + kPfxStages;                               // [stages] S of the chunk done
  uint64_t* full_v = empty_k + kPfxStages;                               // [stages] V chunk landed
  uint64_t* empty_v = full_v + kPfxStages;                               // [stages] P V of the chunk done
  uint64_t* s_full = empty_v + kPfxStages;                               // [2] S buffer written
  uint64_t* s_free = s_full + 2;                                         // [2] S buffer read out
  uint64_t* p_full = s_free + 2;                                         // [2] P tile written (O rescaled)
  uint64_t* p_free = p_full + 2;                                         // [2] P V done with the P tile
  uint64_t* o_done = p_free + 2;                                         // one phase per P V
  uint64_t* bar_done = o_done + 1;                                       // every MMA of the CTA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);  // some wait gave up
  int* soft_abort = abort_flag + 1;  // a softmax warp gave up (written by those warps only)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x, kv = blockIdx.y, split = blockIdx.z;
  const int b0 = split * p.chunks_per_split * kPfxBlocks;
  const int b1 = min(b0 + p.chunks_per_split * kPfxBlocks, p.prefix_blocks);
  const int nblk = max(0, b1 - b0);
  const int nchunks = (nblk + kPfxBlocks - 1) / kPfxBlocks;
  const bool loader = warp == kPfxKWarp || warp == kPfxVWarp;

  // The previous kernel on the stream may still run: wait for it before
  // reading anything, then let the next kernel be scheduled.
  grid_wait_prerequisites();
  grid_launch_dependents();

  // Loader lanes: the physical blocks of the split's blocks b0 + i, b0 + 32 + i, ...
  // (read first, so that their latency overlaps the set-up below)
  constexpr int kMaxHeld = 4;  // up to 128 blocks per split kept in shared memory
  int held[kMaxHeld];
#pragma unroll
  for (int r = 0; r < kMaxHeld; ++r) {
    const int b = b0 + r * 32 + lane;
    held[r] = (loader && b < b1) ? __ldg(p.block_tables + b) : -1;
  }

  if (tid == 0) {
    for (int k = 0; k < kPfxStages; ++k) {
      mbar_init(&full_k[k], 1);
      mbar_init(&empty_k[k], 1);
      mbar_init(&full_v[k], 1);
      mbar_init(&empty_v[k], 1);
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
    *soft_abort = 0;
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
  // (the loader warps do not wait for it)
  if (!loader) named_barrier(1, kPfxSoftmaxThreads + 32);

  if (loader) {
    // ---------------------------------------------------------- loader warps (K, V)
    const bool is_k = warp == kPfxKWarp;
    uint64_t* fullb = is_k ? full_k : full_v;
    uint64_t* emptyb = is_k ? empty_k : empty_v;
    const CUtensorMap* map = is_k ? &kmap : &vmap;
    uint8_t* ring = smem + (is_k ? Ly::kOffK : Ly::kOffV);
    // the split's physical blocks into this warp's table in shared memory
    // (-1: past the split, or outside the pool: read as zeros, flagged)
    int* tbl = reinterpret_cast<int*>(smem + Ly::kOffTbl) + (is_k ? 0 : kMaxHeld * 32);
#pragma unroll
    for (int r = 0; r < kMaxHeld; ++r) {
      const bool in_split = b0 + r * 32 + lane < b1;
      int v = held[r];
      if (in_split && (v < 0 || (long long)v >= p.num_blocks)) {
        if (is_k) flag_error(p.err, DEVERR_BLOCK_RANGE);
        v = -1;
      }
      tbl[r * 32 + lane] = v;
    }
    __syncwarp();
    if (lane == 0) prefetch_tensormap(map);
    int issued = 0;
    for (; issued < nchunks; ++issued) {
      // the chunk's four physical blocks
      int phys4[kPfxBlocks];
#pragma unroll
      for (int i = 0; i < kPfxBlocks; ++i) {
        const int j = issued * kPfxBlocks + i;  // block index inside the split
        if (j < kMaxHeld * 32) {
          phys4[i] = tbl[j];
        } else {  // a split longer than the table: read it here
          phys4[i] = b0 + j < b1 ? __ldg(p.block_tables + b0 + j) : -1;
          if (b0 + j < b1 && (phys4[i] < 0 || (long long)phys4[i] >= p.num_blocks)) {
            if (lane == 0 && is_k) flag_error(p.err, DEVERR_BLOCK_RANGE);
            phys4[i] = -1;
          }
        }
      }
      if (lane == 0) {
        const int k = issued, stage = k % kPfxStages;
        // the stage's previous chunk (k - stages) must have been read by its MMA
        if (k >= kPfxStages && !mbar_wait(&emptyb[stage], ((k / kPfxStages) - 1) & 1, p.wait_limit))
          atomicExch(abort_flag, 1);
        uint8_t* dst = ring + stage * Ly::kKV;
        if (!*abort_flag) {
          mbar_arrive_expect_tx(&fullb[stage], Ly::kKV);
#pragma unroll
          for (int i = 0; i < kPfxBlocks; ++i) {
            // blocks past the split, and table entries outside the pool, read as zeros (TMA fill)
#pragma unroll
            for (int db = 0; db < Ly::kDBlk; ++db) {
              const uint32_t off = db * (kPfxTok * 128) + i * (kBlockSize * 128);
              tma_load_3d(dst + off, map, 0, kv * Ly::kDBlk + db, phys4[i] * kBlockSize, &fullb[stage]);
            }
          }
        }
      }
      if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
    }
    // the K warp, done issuing, takes this CTA's share of the contract check
    if (is_k) check_prefix_contract(p, tile, kv, b0, nblk, lane);
    // never leave with copies in flight: the last stages issued have landed
    if (lane == 0) {
      for (int k = max(0, issued - kPfxStages); k < issued; ++k)
        mbar_wait(&fullb[k % kPfxStages], (k / kPfxStages) & 1);
    }
  } else if (warp == kPfxMmaWarp) {
    // ---------------------------------------------------------- MMA warp
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kPfxRows, kPfxTok, false, false);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kPfxRows, D, false, true);
      const uint32_t q_addr = smem_addr(q_tile);
      bool ok = true;
      auto issue_pv = [&](int c) {  // O += P(c) V(c), then free the V stage and the P tile
        ok = mbar_wait(&p_full[c & 1], (c >> 1) & 1, p.wait_limit) &&
             mbar_wait(&full_v[c % kPfxStages], (c / kPfxStages) & 1, p.wait_limit);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t v_addr = smem_addr(smem + Ly::kOffV + (c % kPfxStages) * Ly::kKV);
        const uint32_t pt = smem_addr(smem + Ly::kOffP + (c & 1) * Ly::kP);
#pragma unroll
        for (int kt = 0; kt < kPfxTok / 16; ++kt) {
          const uint64_t a = umma_desc_sw128(pt + kt * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(v_addr + kt * 2048, kPfxTok * 128, 1024);
          umma_bf16(t_o, a, b, idesc_pv, (c > 0 || kt > 0) ? 1u : 0u);
        }
        umma_commit(&empty_v[c % kPfxStages]);
        umma_commit(&p_free[c & 1]);
        umma_commit(o_done);
      };
      for (int c = 0; c < nchunks && ok; ++c) {
        ok = mbar_wait(&full_k[c % kPfxStages], (c / kPfxStages) & 1, p.wait_limit);
        if (ok && c >= 2) ok = mbar_wait(&s_free[c & 1], ((c - 2) >> 1) & 1, p.wait_limit);
        if (!ok) break;
        tc_fence_after_sync();
        // S(c) = Q K(c)^T into S buffer c % 2
        const uint32_t k_addr = smem_addr(smem + Ly::kOffK + (c % kPfxStages) * Ly::kKV);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint64_t a = umma_desc_sw128(q_addr + (ks >> 2) * (kPfxRows * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t b = umma_desc_sw128(k_addr + (ks >> 2) * (kPfxTok * 128) + (ks & 3) * 32, 16, 1024);
          umma_bf16(tmem + (c & 1) * kPfxTok, a, b, idesc_qk, ks > 0);
        }
        umma_commit(&s_full[c & 1]);
        umma_commit(&empty_k[c % kPfxStages]);
        // P V of the chunk before, once its probabilities are written
        if (c >= 1) issue_pv(c - 1);
      }
      if (ok && nchunks > 0) issue_pv(nchunks - 1);
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
    // ---- the last P V done: normalised partial o of the 128 rows through
    // shared memory (fp32, [D / 32][128 rows][128 B], 128-byte swizzle, each
    // thread writes its row conflict-free) to coalesced row stores (rows past
    // the batch are skipped), and the base-2 lse per row
    if (ok && nchunks > 0 && !mbar_wait(o_done, (nchunks - 1) & 1, p.wait_limit)) ok = false;
    if (!__all_sync(0xffffffffu, ok) && lane == 0) {
      atomicExch(abort_flag, 1);
      *soft_abort = 1;
    }
    named_barrier(2, kPfxSoftmaxThreads);  // every softmax warp knows whether one gave up
    if (!*reinterpret_cast<volatile int*>(soft_abort)) {
      tc_fence_after_sync();
      // the staging reuses shared memory the TMA wrote and the tensor core
      // read (async proxy): order those before these generic stores
      fence_proxy_async_smem();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint8_t* ostage = smem + Ly::kOffO;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t orow[32];
        tmem_ld32(t_o + lane_base + cb * 32, orow);
        tmem_wait_ld();
        uint8_t* dst = ostage + cb * (kPfxRows * 128) + tid * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(dst + ((j ^ (tid & 7)) << 4)) =
              make_float4(__uint_as_float(orow[4 * j]) * inv, __uint_as_float(orow[4 * j + 1]) * inv,
                          __uint_as_float(orow[4 * j + 2]) * inv, __uint_as_float(orow[4 * j + 3]) * inv);
      }
      named_barrier(2, kPfxSoftmaxThreads);
      // row by row, a warp per row: lane e holds floats 4e .. 4e+3 (column
      // block e / 8, 16-byte piece e % 8), one coalesced store of the row
      float* o_plane = p.part_o + ((size_t)kv * p.splits + split) * p.rows * D;
      const int nrows = min(kPfxRows, p.rows - tile * kPfxRows);
      for (int r = warp; r < nrows; r += kPfxSoftmaxThreads / 32) {
#pragma unroll
        for (int e = lane; e < D / 4; e += 32) {
          const float4 v = *reinterpret_cast<const float4*>(ostage + (e >> 3) * (kPfxRows * 128) + r * 128 +
                                                            (((e & 7) ^ (r & 7)) << 4));
          reinterpret_cast<float4*>(o_plane + (size_t)(tile * kPfxRows + r) * D)[e] = v;
        }
      }
      if (row_ok)
        p.part_lse[((size_t)kv * p.splits + split) * p.rows + row] = nchunks > 0 ? m + log2f(l) : -INFINITY;
    }
  }

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
    if (e == cudaSuccess) e = prefer_max_smem(prefix_tc_kernel<D>);  // decode CTAs share the SM
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
