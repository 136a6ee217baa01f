// Shared-prefix pass of decode attention.  When every sequence of a batch
// starts with the same physical blocks (a common system prompt: "Chapter 18 -
// KV-Cache Optimization Strategies", Prefix Caching; "KV Cache Engineering for
// LLM Serving", section 11), the attention over those blocks is computed once
// per KV head for the queries of all sequences together: the scores are a
// dense [S*G x 16] x [16 x d] product per block instead of S separate
// [G x 16] ones, and the prefix is read once per query tile instead of once
// per sequence.  The pass is split along the prefix; each split leaves a
// normalised partial output and its base-2 log-sum-exp per query row, a small
// second launch combines the splits (softmax states merge exactly:
// M = max lse_i, o = sum 2^(lse_i - M) o_i / sum 2^(lse_i - M)), and the
// decode kernel over each sequence's own blocks starts from that state.
//
// CTA = 4 warps x 16 query rows of one KV head, one split of the prefix.  Q
// fragments stay in registers; K and V blocks come through a ring of TMA
// stages (the decode kernel's pool view: 16 rows x 128-byte chunks, 128-byte
// swizzle); S = Q K^T and O += P V on m16n8k16 BF16 MMAs, P reused from the
// score accumulators.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

constexpr int kPrefixWarps = 4;
constexpr int kPrefixStages = 4;

struct PrefixParams {
  const __nv_bfloat16* query;  // [num_seqs, n_q, D]
  const int32_t* block_tables;  // the prefix is the first prefix_blocks entries of row 0
  int* err;
  float* part_o;    // [n_kv][rows][splits][D]
  float* part_lse;  // [n_kv][rows][splits], base 2
  long long num_blocks;
  int rows, n_q, n_kv, G, prefix_blocks, splits, per_split;
  float scale_log2;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kPrefixWarps * 32) prefix_attn_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                          const __grid_constant__ CUtensorMap vmap,
                                                                          const PrefixParams p) {
  constexpr int kChunks = D * 2 / 128;
  constexpr int kTile = kChunks * 2048;  // one head's 16-row tile of K (or V)
  constexpr int KS = D / 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kPrefixStages];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int kv = blockIdx.y, split = blockIdx.z;
  const int b0 = split * p.per_split, b1 = min(b0 + p.per_split, p.prefix_blocks);
  const int nblk = max(0, b1 - b0);

  grid_launch_dependents();
  if (tid == 0) {
    for (int k = 0; k < kPrefixStages; ++k) mbar_init(&full[k], 1);
    fence_barrier_init();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  __syncthreads();
  grid_wait_prerequisites();

  auto issue = [&](int j) {  // block b0 + j into stage j % kPrefixStages
    const int stage = j % kPrefixStages;
    int phys = __ldg(p.block_tables + b0 + j);
    if (phys < 0 || (long long)phys >= p.num_blocks) {
      flag_error(p.err, DEVERR_BLOCK_RANGE);
      phys = -1;  // row -16: the TMA zero-fills the box
    }
    uint8_t* st = smem + (size_t)stage * 2 * kTile;
    mbar_arrive_expect_tx(&full[stage], 2 * kTile);
#pragma unroll
    for (int ch = 0; ch < kChunks; ++ch) {
      tma_load_3d(st + ch * 2048, &kmap, 0, kv * kChunks + ch, phys * kBlockSize, &full[stage]);
      tma_load_3d(st + kTile + ch * 2048, &vmap, 0, kv * kChunks + ch, phys * kBlockSize, &full[stage]);
    }
  };
  if (tid == 0)
    for (int j = 0; j < min(nblk, kPrefixStages); ++j) issue(j);

  // ---- this warp's 16 query rows as A fragments (rows past the batch are 0)
  const int row0 = blockIdx.x * (kPrefixWarps * 16) + warp * 16;
  uint32_t qa[KS][4];
  {
    const int ra = row0 + g, rb = row0 + g + 8;
    const bool oka = ra < p.rows, okb = rb < p.rows;
    const uint32_t* qa_row = reinterpret_cast<const uint32_t*>(
        p.query + ((size_t)(oka ? ra / p.G : 0) * p.n_q + kv * p.G + (oka ? ra % p.G : 0)) * D);
    const uint32_t* qb_row = reinterpret_cast<const uint32_t*>(
        p.query + ((size_t)(okb ? rb / p.G : 0) * p.n_q + kv * p.G + (okb ? rb % p.G : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = oka ? __ldg(qa_row + ks * 8 + c) : 0u;
      qa[ks][1] = okb ? __ldg(qb_row + ks * 8 + c) : 0u;
      qa[ks][2] = oka ? __ldg(qa_row + ks * 8 + 4 + c) : 0u;
      qa[ks][3] = okb ? __ldg(qb_row + ks * 8 + 4 + c) : 0u;
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;  // rows g and g + 8

  // ldmatrix row addresses: K (non-transposed) and V (transposed), tokens 0..15
  const int mi = lane >> 3, r8 = lane & 7;
  const int k_tok = r8 + (mi >> 1) * 8, k_half = mi & 1;  // matrices (tok 0-7 | 8-15) x (d 0-7 | 8-15)
  const int v_tok = r8 + (mi & 1) * 8, v_dt = mi >> 1;    // matrices (tok 0-7 | 8-15) x (d-tile dt | dt + 1)

  bool ok = true;
  int j = 0;
  for (; j < nblk; ++j) {
    const int stage = j % kPrefixStages;
    ok = mbar_wait(&full[stage], (j / kPrefixStages) & 1);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    const uint32_t kt = smem_addr(smem + (size_t)stage * 2 * kTile);
    const uint32_t vt = kt + kTile;

    // ---- S = Q K^T: [16 rows x 16 tokens] as two n8 tiles
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int piece = (ks & 3) * 2 + k_half;
      uint32_t b[4];
      ldmatrix_x4(b, kt + (ks >> 2) * 2048 + k_tok * 128 + ((piece ^ (k_tok & 7)) << 4));
      mma_bf16(s0, qa[ks], b[0], b[1]);
      mma_bf16(s1, qa[ks], b[2], b[3]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s0[e] *= p.scale_log2;
      s1[e] *= p.scale_log2;
    }
    // ---- online softmax over the block, rows g (s*[0], s*[1]) and g + 8 (s*[2], s*[3])
    float mx_a = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
    float mx_b = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
    mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
    mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
    // lazy rescale: the reference max moves (and the accumulators are
    // rescaled) only when a score exceeds it by more than 2^8, so P <= 2^8
    if (__any_sync(0xffffffffu, mx_a > m_a + 8.f || mx_b > m_b + 8.f)) {
      const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
      const float al_a = ex2f(m_a - mn_a), al_b = ex2f(m_b - mn_b);
      m_a = mn_a;
      m_b = mn_b;
      l_a *= al_a;
      l_b *= al_b;
#pragma unroll
      for (int dt = 0; dt < D / 8; ++dt) {
        o[dt][0] *= al_a;
        o[dt][1] *= al_a;
        o[dt][2] *= al_b;
        o[dt][3] *= al_b;
      }
    }
    float pa[4] = {ex2f(s0[0] - m_a), ex2f(s0[1] - m_a), ex2f(s1[0] - m_a), ex2f(s1[1] - m_a)};
    float pb[4] = {ex2f(s0[2] - m_b), ex2f(s0[3] - m_b), ex2f(s1[2] - m_b), ex2f(s1[3] - m_b)};
    l_a += (pa[0] + pa[1] + pa[2] + pa[3]);
    l_b += (pb[0] + pb[1] + pb[2] + pb[3]);
    // P as the A operand: (row g, tokens 2c, 2c+1), (row g+8, ...), (row g, 2c+8, 2c+9), (row g+8, ...)
    uint32_t pf[4] = {pack_bf16(pa[0], pa[1]), pack_bf16(pb[0], pb[1]), pack_bf16(pa[2], pa[3]),
                      pack_bf16(pb[2], pb[3])};
    // ---- O += P V: d-tiles of 8, two per transposed ldmatrix
#pragma unroll
    for (int dt = 0; dt < D / 8; dt += 2) {
      const int d_tile = dt + v_dt;  // the 8 dims (16 bytes) of this lane's matrix
      uint32_t b[4];
      ldmatrix_x4_trans(b, vt + (d_tile >> 3) * 2048 + v_tok * 128 + (((d_tile & 7) ^ (v_tok & 7)) << 4));
      mma_bf16(o[dt], pf, b[0], b[1]);
      mma_bf16(o[dt + 1], pf, b[2], b[3]);
    }
    __syncthreads();  // every warp is done with this stage
    if (tid == 0 && j + kPrefixStages < nblk) issue(j + kPrefixStages);
  }
  if (!ok) {
    if (tid == 0) {
      flag_error(p.err, DEVERR_TIMEOUT);
      // blocks j .. j + stages - 1 were issued and not consumed: let them land
      // before the CTA exits (each wait bounded)
      for (int i = j; i < min(nblk, j + kPrefixStages); ++i)
        mbar_wait(&full[i % kPrefixStages], (i / kPrefixStages) & 1);
    }
    return;
  }

  // ---- normalise and store this split's partial state
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const int ra = row0 + g, rb = row0 + g + 8;
  const float ia = l_a > 0.f ? 1.f / l_a : 0.f, ib = l_b > 0.f ? 1.f / l_b : 0.f;
  const size_t base = (size_t)kv * p.rows;
#pragma unroll
  for (int dt = 0; dt < D / 8; ++dt) {
    const int d = dt * 8 + 2 * c;
    if (ra < p.rows)
      *reinterpret_cast<float2*>(p.part_o + ((base + ra) * p.splits + split) * D + d) =
          make_float2(o[dt][0] * ia, o[dt][1] * ia);
    if (rb < p.rows)
      *reinterpret_cast<float2*>(p.part_o + ((base + rb) * p.splits + split) * D + d) =
          make_float2(o[dt][2] * ib, o[dt][3] * ib);
  }
  if (c == 0) {
    if (ra < p.rows) p.part_lse[(base + ra) * p.splits + split] = nblk > 0 ? m_a + log2f(l_a) : -INFINITY;
    if (rb < p.rows) p.part_lse[(base + rb) * p.splits + split] = nblk > 0 ? m_b + log2f(l_b) : -INFINITY;
  }
}

// Splits of the prefix so that about four CTAs run on every SM (the pass is
// latency-bound: more resident warps hide more of each block's MMA and
// softmax chain), each split at least 4 blocks long.
static void prefix_grid(int rows, int n_kv, int prefix_blocks, int* splits, int* per_split) {
  const int tiles = (rows + kPrefixWarps * 16 - 1) / (kPrefixWarps * 16);
  const int want = std::max(1, (4 * std::max(1, device_sm_count())) / std::max(1, tiles * n_kv));
  int sp = std::max(1, std::min(want, prefix_blocks / 4));
  sp = std::min(sp, kMaxPrefixSplits);
  *per_split = (prefix_blocks + sp - 1) / sp;
  *splits = (prefix_blocks + *per_split - 1) / *per_split;
}

// The splits' states combined per (KV head, query row): one CTA of 256 threads
// per 8 rows, a thread per (row, 4 dims), the splits' loads independent.
struct CombineParams {
  const float* part_o;
  const float* part_lse;
  float* o;    // [n_kv * rows][D]
  float* lse;  // [n_kv * rows]
  int total_rows, splits;
};

template <int D>
__global__ void __launch_bounds__(256) prefix_combine_kernel(const CombineParams p) {
  grid_launch_dependents();
  grid_wait_prerequisites();
  constexpr int V = D / 4;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int r = idx / V, v = idx - r * V;
  if (r >= p.total_rows) return;
  const float* lse = p.part_lse + (size_t)r * p.splits;
  float M = -INFINITY;
#pragma unroll 8
  for (int k = 0; k < p.splits; ++k) M = fmaxf(M, __ldcg(lse + k));
  float wsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int k = 0; k < p.splits; ++k) {
    const float w = ex2f(__ldcg(lse + k) - M);
    const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + ((size_t)r * p.splits + k) * D) + v);
    wsum += w;
    acc.x += w * o.x;
    acc.y += w * o.y;
    acc.z += w * o.z;
    acc.w += w * o.w;
  }
  const float inv = 1.f / wsum;
  reinterpret_cast<float4*>(p.o + (size_t)r * D)[v] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (v == 0) p.lse[r] = M + log2f(wsum);
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t prefix_workspace_bytes(int num_seqs, int n_q, int n_kv, int head_dim, int prefix_blocks) {
  const int rows = num_seqs * (n_q / n_kv);
  int splits = 1, per = 1;
  prefix_grid(rows, n_kv, prefix_blocks, &splits, &per);
  const size_t part_o = (size_t)n_kv * rows * splits * head_dim * 4;
  const size_t part_l = (size_t)n_kv * rows * splits * 4;
  const size_t o = (size_t)n_kv * rows * head_dim * 4;
  const size_t l = (size_t)n_kv * rows * 4;
  return align256(part_o) + align256(part_l) + align256(o) + align256(l);
}

pkv_status launch_prefix(const DecodeShape& s, const CUtensorMap& km, const CUtensorMap& vm, const void* query,
                         const int32_t* block_tables, int64_t num_blocks, int prefix_blocks, float sm_scale,
                         void* prefix_ws, int32_t* device_error, PrefixState* state, cudaStream_t stream) {
  PrefixParams p;
  p.query = static_cast<const __nv_bfloat16*>(query);
  p.block_tables = block_tables;
  p.err = device_error;
  p.n_q = s.n_q;
  p.n_kv = s.n_kv;
  p.G = s.n_q / s.n_kv;
  p.rows = s.num_seqs * p.G;
  p.prefix_blocks = prefix_blocks;
  p.num_blocks = num_blocks;
  p.scale_log2 = (float)((double)sm_scale * 1.4426950408889634);
  prefix_grid(p.rows, s.n_kv, prefix_blocks, &p.splits, &p.per_split);
  uint8_t* ws = static_cast<uint8_t*>(prefix_ws);
  const size_t part_o = align256((size_t)s.n_kv * p.rows * p.splits * s.head_dim * 4);
  const size_t part_l = align256((size_t)s.n_kv * p.rows * p.splits * 4);
  const size_t comb_o = align256((size_t)s.n_kv * p.rows * s.head_dim * 4);
  p.part_o = reinterpret_cast<float*>(ws);
  p.part_lse = reinterpret_cast<float*>(ws + part_o);
  CombineParams cp;
  cp.part_o = p.part_o;
  cp.part_lse = p.part_lse;
  cp.o = reinterpret_cast<float*>(ws + part_o + part_l);
  cp.lse = reinterpret_cast<float*>(ws + part_o + part_l + comb_o);
  cp.total_rows = s.n_kv * p.rows;
  cp.splits = p.splits;
  state->o = cp.o;
  state->lse = cp.lse;
  state->splits = 1;
  state->rows = p.rows;

  const int tiles = (p.rows + kPrefixWarps * 16 - 1) / (kPrefixWarps * 16);
  const int tile_bytes = s.head_dim * 2 * 16;
  const size_t smem = (size_t)kPrefixStages * 2 * tile_bytes + 1024;
  auto run = [&](auto kern) -> pkv_status {
    static int configured = 0;
    if ((int)smem > configured) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefix)");
      configured = (int)smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles, s.n_kv, p.splits);
    cfg.blockDim = dim3(kPrefixWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefix_attn_kernel launch");
    return PKV_OK;
  };
  auto combine = [&](auto kern) -> pkv_status {
    const long long threads = (long long)cp.total_rows * (s.head_dim / 4);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, cp);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefix_combine_kernel launch");
    return PKV_OK;
  };
  pkv_status st = PKV_ERR_UNSUPPORTED;
  if (s.head_dim == 128) {
    st = run(prefix_attn_kernel<128>);
    if (st == PKV_OK) st = combine(prefix_combine_kernel<128>);
  } else if (s.head_dim == 64) {
    st = run(prefix_attn_kernel<64>);
    if (st == PKV_OK) st = combine(prefix_combine_kernel<64>);
  }
  return st;
}

}  // namespace pkv
