// Host-side declarations shared by the .cu files of libpkv (not installed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

constexpr int kBlockSize = 16;
constexpr int kMaxStages = 8;
constexpr int kMaxConsumerWarps = 16;
constexpr int kMaxCtas = 4096;          // upper bound of persistent CTAs per launch
constexpr int kTargetCtasPerSm = 4;
constexpr int kQuantCtasPerSm = 3;  // quantised caches: CTAs of up to 4 consumer warps
constexpr size_t kSmemPerSm = 233472;  // 228 KB of shared memory per SM

// Cache kinds of the tensor-core decode kernel.
enum TcCache : int { TC_BF16 = 0, TC_INT8 = 1, TC_FP8 = 2, TC_E5M2 = 3, TC_INT4 = 4, TC_KIVI = 5 };
__host__ __device__ constexpr bool tc_fp8(int c) { return c == TC_FP8 || c == TC_E5M2; }          // one scale per KV head
__host__ __device__ constexpr bool tc_row_scaled(int c) { return c == TC_INT8 || c == TC_INT4; }  // one scale per (token, head)
// V scaled per (token, head): the row-scaled formats and the 2-bit KIVI cache,
// whose K scales are per (block, head, channel)
__host__ __device__ constexpr bool tc_v_row_scaled(int c) { return tc_row_scaled(c) || c == TC_KIVI; }
// Caches whose decode is bound by the work of unpacking codes (every format but
// BF16): 3 CTAs of up to 4 consumer warps per SM under a narrow register
// bound, for more warps in flight.  BF16 takes 4 CTAs of 2 warps.
__host__ __device__ constexpr bool tc_narrow(int c) { return c != TC_BF16; }

struct DecodeShape {
  int num_seqs, n_q, n_kv, head_dim, block_size;
  pkv_dtype act, cache;
};

// Launch plan of the tensor-core decode kernel; a pure function of the shape,
// the device's SM count / shared-memory limit and the tuning overrides.
struct TcPlan {
  int cache_kind;   // TcCache
  int G, QC, HPC, HG, NCW;
  int chunks;       // 128-byte row chunks per KV head row (head_dim * elem / 128)
  int stages;
  int num_ctas;
  bool overlap_prologue;  // programmatic dependent launch (PKV_TUNE_OVERLAP_PROLOGUE)
  int units;        // num_seqs * HG
  uint32_t stage_bytes, tx_bytes;
  size_t smem_bytes;
  size_t ws_part_o, ws_part_lse, ws_desc, ws_total;  // byte offsets / total
};

pkv_status plan_tc(const DecodeShape& s, const pkv_decode_tuning* tuning, TcPlan* plan);

// The decode and merge kernels ask for the largest shared-memory carveout.
// An SM's split between L1 and shared memory is fixed while CTAs run on it,
// and the default picks the smallest split that fits a kernel's own CTA, which
// would keep the CTAs of a kernel running beside it off that SM.
template <typename Kernel>
inline cudaError_t prefer_max_smem(Kernel kern) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
}

// Start state of a decode unit (kivi.cu's residual pass): per (KV head,
// query row = s * G + head in group) the normalised output and its base-2 lse,
// which the decode over the quantised blocks starts from.
struct PrefixState {
  const float* o = nullptr;    // [n_kv][rows][head_dim]
  const float* lse = nullptr;  // [n_kv][rows]
  int splits = 0;
  int rows = 0;
};

// Shared-prefix pass (prefix.cu): per (KV head, query row = s * G + head in
// group, split of the prefix) the normalised output over the split's tokens
// and its base-2 lse.  The merge launch combines these pieces with the pieces
// of each sequence's own blocks; a decode unit that one CTA finished whole
// leaves its piece in unit_o / unit_lse.
constexpr int kMaxPrefixSplits = 64;
struct PrefixPieces {
  const float* o = nullptr;    // [n_kv][splits][rows][head_dim]
  const float* lse = nullptr;  // [n_kv][splits][rows]
  int splits = 0;
  int rows = 0;
  float* unit_o = nullptr;     // [num_seqs * n_q][head_dim]
  float* unit_lse = nullptr;   // [num_seqs * n_q]
};

struct TcArgs {
  void* out;
  const void* query;
  const void* key_cache;
  const void* value_cache;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_tables;
  int max_blocks_per_seq;
  const int32_t* context_lens;
  int max_context_len;
  int64_t num_blocks;
  float sm_scale;
  float* lse_out;
  void* workspace;
  int32_t* device_error;
  // fused decode step only: new rows [num_seqs, n_kv, head_dim] appended as token
  // L-1 of each sequence before the attention (the caches are then written)
  const void* new_key = nullptr;
  const void* new_value = nullptr;
  // sliding window with sinks: attend to [0, sinks) and [L - window, L); 0 = all
  int window = 0;
  int sinks = 0;
  // Quest decode only: [num_seqs, n_kv, k_pages] logical pages to read
  const int32_t* pages = nullptr;
  int k_pages = 0;
  // shared-prefix decode only: the first skip_blocks logical blocks of every
  // sequence were attended by the prefix pass, whose state each unit starts from
  int skip_blocks = 0;
  PrefixState prefix;
  void* prefix_ws = nullptr;  // scratch of the prefix pass (prefix_workspace_bytes)
  int prefix_splits = 0;      // splits of the prefix pass (0 = automatic)
  bool prefix_serial = false; // the decode waits for the prefix pass instead of running beside it
  long long wait_limit = 0;   // SM cycles a bounded wait of the decode kernels spends (0 = default)
};

pkv_status launch_tc(const DecodeShape& s, const TcPlan& plan, const TcArgs& a, cudaStream_t stream);

// 2-bit KIVI cache (kivi.cu).  The residual pass appends the new rows (if
// any) to the BF16 residual of each sequence, quantises a residual that became
// a full block into the pool, and leaves per (KV head, row = s * G + head in
// group) the normalised output and base-2 lse over the residual rows, which the
// decode over the quantised full blocks starts from.
struct KiviArgs {
  const void* query;
  const void* new_key;    // [num_seqs, n_kv, 128] bf16 or null
  const void* new_value;
  void* residual_k;       // [num_seqs, 16, n_kv, 128] bf16
  void* residual_v;
  void* key_cache;        // [num_blocks, n_kv, 16, 32] bytes
  void* value_cache;
  float* k_scale;         // [num_blocks, n_kv, 128]
  float* v_scale;         // [num_blocks, n_kv, 16]
  const int32_t* block_tables;
  int max_blocks_per_seq;
  const int32_t* context_lens;
  int cap_len;
  int64_t num_blocks;
  int num_seqs, n_q, n_kv;
  float sm_scale;
  int32_t* device_error;
};
size_t kivi_state_bytes(int num_seqs, int n_q);
pkv_status launch_kivi_residual(const KiviArgs& a, void* state_ws, PrefixState* state, cudaStream_t stream);
pkv_status launch_kivi_quantize_blocks(const void* key_rows, const void* value_rows, const int32_t* dst_blocks,
                                       int64_t n, void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                                       int n_kv, int64_t num_blocks, int32_t* device_error, cudaStream_t stream);

size_t prefix_workspace_bytes(int num_seqs, int n_q, int n_kv, int head_dim, int prefix_blocks, int want_splits);
pkv_status make_pool_map(CUtensorMap* map, const void* base, int elem, int chunk_bytes, int row_bytes, int64_t rows);
pkv_status launch_prefix(const DecodeShape& s, const CUtensorMap& km, const CUtensorMap& vm, const TcArgs& a,
                         long long wait_limit, PrefixPieces* pieces, cudaStream_t stream);

pkv_status launch_decode_f32(const DecodeShape& s, const TcArgs& a, cudaStream_t stream);

pkv_status launch_cache_write(const void* key, const void* value, void* key_cache, void* value_cache, float* k_scale,
                              float* v_scale, const int64_t* slot_mapping, int64_t num_tokens, int n_kv, int head_dim,
                              int block_size, int64_t num_blocks, pkv_dtype act, pkv_dtype cache, int32_t* device_error,
                              cudaStream_t stream);

pkv_status launch_move_blocks(const void* const src[4], void* const dst[4], const size_t bytes_per_block[4], int npools,
                              const int64_t* pairs, int64_t num_pairs, int64_t src_blocks, int64_t dst_blocks,
                              int32_t* device_error, cudaStream_t stream);

pkv_status launch_quest_summaries(const void* key_cache, void* page_min, void* page_max, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* context_lens, int num_seqs, int n_kv,
                                  int head_dim, int64_t num_blocks, pkv_dtype cache, int last_page_only,
                                  int32_t* device_error, cudaStream_t stream);
pkv_status launch_quest_select(const void* query, const void* page_min, const void* page_max,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int64_t num_blocks,
                               pkv_dtype act, pkv_dtype cache, int k_pages, int32_t* selected, float* scores,
                               int32_t* device_error, cudaStream_t stream);

// Records the CUDA error text for pkv_last_cuda_error() and returns PKV_ERR_CUDA.
pkv_status cuda_fail(cudaError_t e, const char* where);
pkv_status driver_fail(int code, const char* where);
// Sets the text pkv_last_cuda_error() returns for this thread.
void note_error(const char* fmt, ...);

int device_sm_count();
int device_smem_optin();

}  // namespace pkv
