// C ABI of libpkv: argument validation, launch planning and status codes.
// Every check here runs on the host before anything is enqueued.
#include <cuda_runtime.h>

#include <algorithm>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "internal.h"

namespace pkv {

static thread_local char g_last_cuda_error[256] = "";

pkv_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", where, cudaGetErrorString(e));
  return PKV_ERR_CUDA;
}

void note_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_cuda_error, sizeof(g_last_cuda_error), fmt, ap);
  va_end(ap);
}

pkv_status driver_fail(int code, const char* where) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: driver error %d", where, code);
  return PKV_ERR_CUDA;
}

int device_sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return v;
}

int device_smem_optin() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return -1;
  return v;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static bool valid_dtype(int d) { return d >= PKV_F32 && d <= PKV_INT4; }
static bool row_scaled(int d) { return d == PKV_INT8 || d == PKV_INT4; }
static bool head_scaled(int d) { return d == PKV_FP8_E4M3 || d == PKV_FP8_E5M2; }

// Shape rules of the decode kernels; PKV_OK when the tensor-core path or the
// F32 path can run it.
static pkv_status check_decode_shape(const DecodeShape& s) {
  if (s.num_seqs < 0 || s.n_q <= 0 || s.n_kv <= 0 || s.head_dim <= 0 || s.block_size <= 0) return PKV_ERR_INVALID_ARG;
  if (!valid_dtype(s.act) || !valid_dtype(s.cache)) return PKV_ERR_INVALID_ARG;
  if (s.act != PKV_F32 && s.act != PKV_BF16) return PKV_ERR_INVALID_ARG;
  if (s.n_q % s.n_kv != 0) return PKV_ERR_INVALID_ARG;
  if (s.block_size != kBlockSize) return PKV_ERR_UNSUPPORTED;
  if (s.n_q / s.n_kv > 64) return PKV_ERR_UNSUPPORTED;
  switch (s.cache) {
    case PKV_F32:
      if (s.act != PKV_F32) return PKV_ERR_UNSUPPORTED;
      if (s.head_dim % 32 != 0 || s.head_dim > 256) return PKV_ERR_UNSUPPORTED;
      return PKV_OK;
    case PKV_BF16:
      if (s.act != PKV_BF16) return PKV_ERR_UNSUPPORTED;
      if (s.head_dim != 64 && s.head_dim != 128) return PKV_ERR_UNSUPPORTED;
      return PKV_OK;
    default:
      if (s.head_dim != 128) return PKV_ERR_UNSUPPORTED;
      return PKV_OK;
  }
}

static size_t workspace_for(const DecodeShape& s, const pkv_decode_tuning* tuning) {
  if (check_decode_shape(s) != PKV_OK) return (size_t)-1;
  if (s.cache == PKV_F32 || s.num_seqs == 0) return 0;
  TcPlan plan;
  if (plan_tc(s, tuning, &plan) != PKV_OK) return (size_t)-1;
  return plan.ws_total;
}

static pkv_status decode_impl(void* out, const void* query, const void* key_cache, const void* value_cache,
                              const float* k_scale, const float* v_scale, const int32_t* block_tables,
                              int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
                              int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks, float sm_scale,
                              pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out, void* workspace,
                              size_t workspace_bytes, int32_t* device_error, const pkv_decode_tuning* tuning,
                              void* stream, const void* new_key = nullptr, const void* new_value = nullptr,
                              int window = 0, int sinks = 0, const int32_t* pages = nullptr, int k_pages = 0,
                              int prefix_blocks = 0) {
  const DecodeShape s{num_seqs, n_q, n_kv, head_dim, block_size, act_dtype, cache_dtype};
  pkv_status st = check_decode_shape(s);
  if (st != PKV_OK) return st;
  if (max_blocks_per_seq < 0 || max_context_len < 0 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (num_blocks * (int64_t)block_size > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  if (num_seqs == 0) return PKV_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_INVALID_ARG;
  const bool quant = row_scaled(cache_dtype) || head_scaled(cache_dtype);
  if (quant && (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale))) return PKV_ERR_INVALID_ARG;
  if (!quant && (k_scale || v_scale)) return PKV_ERR_INVALID_ARG;
  if (max_blocks_per_seq == 0 && max_context_len > 0) return PKV_ERR_INVALID_ARG;
  if (window < 0 || sinks < 0) return PKV_ERR_INVALID_ARG;
  if (pages && (k_pages < 1 || window > 0 || new_key)) return PKV_ERR_INVALID_ARG;
  if (prefix_blocks < 0 || (prefix_blocks > 0 && (pages || window > 0))) return PKV_ERR_INVALID_ARG;
  if (prefix_blocks > 0) {
    if (cache_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (prefix_blocks > max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
  }

  if (tuning && (tuning->reserved != 0 || tuning->prefix_splits < 0 || tuning->wait_limit_cycles < 0))
    return PKV_ERR_INVALID_ARG;
  TcArgs a{out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq, context_lens,
           max_context_len, num_blocks, sm_scale, lse_out, workspace, device_error, new_key, new_value, window,
           sinks, pages, k_pages};
  a.skip_blocks = prefix_blocks;
  if (tuning) {
    a.prefix_splits = tuning->prefix_splits;
    a.prefix_serial = (tuning->flags & PKV_TUNE_PREFIX_SERIAL) != 0;
    a.wait_limit = tuning->wait_limit_cycles;
  }
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  if (cache_dtype == PKV_F32) return launch_decode_f32(s, a, strm);
  // a page list is per KV head: one KV head per CTA
  pkv_decode_tuning one_head = tuning ? *tuning : pkv_decode_tuning{0, 0, 0, 0, 0, 0, 0};
  if (pages) {
    one_head.heads_per_cta = 1;
    tuning = &one_head;
  }
  TcPlan plan;
  st = plan_tc(s, tuning, &plan);
  if (st != PKV_OK) return st;
  size_t need = plan.ws_total;
  if (prefix_blocks > 0) {
    // the prefix pass keeps its partial states after the decode's scratch
    const size_t off = (plan.ws_total + 255) / 256 * 256;
    need = off + prefix_workspace_bytes(num_seqs, n_q, n_kv, head_dim, prefix_blocks, a.prefix_splits);
    if (workspace && workspace_bytes >= need) a.prefix_ws = static_cast<uint8_t*>(workspace) + off;
    plan.overlap_prologue = true;  // the decode is queued behind the prefix pass with programmatic serialisation
  }
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  return launch_tc(s, plan, a, strm);
}

// Address a kernel on the current device may use for p: device (or managed)
// memory of this device as is, page-locked host memory through its mapped
// device address.  Anything else (pageable host memory, another device's
// memory) is rejected, so the kernel never dereferences an unmapped pointer.
static pkv_status device_address(const void* p, const void** out) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of the query
    return PKV_ERR_INVALID_ARG;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  switch (a.type) {
    case cudaMemoryTypeDevice:
      if (a.device != dev) return PKV_ERR_INVALID_ARG;
      *out = p;
      return PKV_OK;
    case cudaMemoryTypeManaged:
      *out = p;
      return PKV_OK;
    case cudaMemoryTypeHost:
      if (!a.devicePointer) return PKV_ERR_INVALID_ARG;
      *out = a.devicePointer;
      return PKV_OK;
    default:
      return PKV_ERR_INVALID_ARG;
  }
}

static pkv_status device_addresses(const void* src[4], void* dst[4], int npools, const int64_t** pairs) {
  for (int i = 0; i < npools; ++i) {
    const void* d = nullptr;
    pkv_status st = device_address(src[i], &src[i]);
    if (st != PKV_OK) return st;
    st = device_address(dst[i], &d);
    if (st != PKV_OK) return st;
    dst[i] = const_cast<void*>(d);
  }
  const void* m = nullptr;
  pkv_status st = device_address(*pairs, &m);
  if (st != PKV_OK) return st;
  *pairs = static_cast<const int64_t*>(m);
  return PKV_OK;
}

// Shared checks of the block movers; fills the pool descriptors.
static pkv_status move_plan(const void* src_k, const void* src_v, const float* src_ks, const float* src_vs,
                            void* dst_k, void* dst_v, float* dst_ks, float* dst_vs, const int64_t* pairs,
                            int64_t num_pairs, int n_kv, int head_dim, int block_size, pkv_dtype cache_dtype,
                            const void* src[4], void* dst[4], size_t bpb[4], int* npools) {
  if (num_pairs < 0 || n_kv <= 0 || head_dim <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
  const bool kivi = cache_dtype == PKV_KIVI2;
  if (!valid_dtype(cache_dtype) && !kivi) return PKV_ERR_INVALID_ARG;
  if (num_pairs > 0 && (!pairs || !src_k || !src_v || !dst_k || !dst_v)) return PKV_ERR_INVALID_ARG;
  const size_t elem = cache_dtype == PKV_F32 ? 4 : (cache_dtype == PKV_BF16 ? 2 : 1);
  const size_t row = cache_dtype == PKV_INT4 ? (size_t)n_kv * head_dim / 2
                     : kivi                  ? (size_t)n_kv * head_dim / 4
                                             : (size_t)n_kv * head_dim * elem;
  if (row % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v)) return PKV_ERR_INVALID_ARG;
  src[0] = src_k;
  src[1] = src_v;
  dst[0] = dst_k;
  dst[1] = dst_v;
  bpb[0] = bpb[1] = row * block_size;
  *npools = 2;
  const bool scaled = row_scaled(cache_dtype) || kivi;
  if (scaled != (src_ks && src_vs && dst_ks && dst_vs)) return PKV_ERR_INVALID_ARG;
  if (scaled) {
    if (!aligned16(src_ks) || !aligned16(src_vs) || !aligned16(dst_ks) || !aligned16(dst_vs)) return PKV_ERR_INVALID_ARG;
    if (((size_t)block_size * n_kv * 4) % 16 != 0) return PKV_ERR_UNSUPPORTED;
    src[2] = src_ks;
    src[3] = src_vs;
    dst[2] = dst_ks;
    dst[3] = dst_vs;
    // KIVI: K scales per (head, channel) of the block, V per (token, head)
    bpb[2] = kivi ? (size_t)n_kv * head_dim * 4 : (size_t)block_size * n_kv * 4;
    bpb[3] = (size_t)block_size * n_kv * 4;
    *npools = 4;
  }
  return PKV_OK;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

pkv_status pkv_kv_cache_write(const void* key, const void* value, void* key_cache, void* value_cache, float* k_scale,
                              float* v_scale, const int64_t* slot_mapping, int64_t num_tokens, int n_kv, int head_dim,
                              int block_size, int64_t num_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                              int32_t* device_error, void* stream) {
  if (num_tokens < 0 || n_kv <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (!valid_dtype(act_dtype) || !valid_dtype(cache_dtype)) return PKV_ERR_INVALID_ARG;
  if (act_dtype != PKV_F32 && act_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
  if (cache_dtype == PKV_F32 && act_dtype != PKV_F32) return PKV_ERR_UNSUPPORTED;
  if (cache_dtype == PKV_BF16 && act_dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PKV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PKV_ERR_INVALID_ARG;
  const bool quant = row_scaled(cache_dtype) || head_scaled(cache_dtype);
  if (quant && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
  if (!quant && (k_scale || v_scale)) return PKV_ERR_INVALID_ARG;
  return launch_cache_write(key, value, key_cache, value_cache, k_scale, v_scale, slot_mapping, num_tokens, n_kv,
                            head_dim, block_size, num_blocks, act_dtype, cache_dtype, device_error,
                            static_cast<cudaStream_t>(stream));
}

size_t pkv_paged_attention_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                          pkv_dtype cache_dtype) {
  const pkv_dtype act = cache_dtype == PKV_F32 ? PKV_F32 : PKV_BF16;
  return workspace_for(DecodeShape{num_seqs, n_q, n_kv, head_dim, block_size, act, cache_dtype}, nullptr);
}

size_t pkv_paged_attention_workspace_size_ex(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                             pkv_dtype cache_dtype, const pkv_decode_tuning* tuning) {
  const pkv_dtype act = cache_dtype == PKV_F32 ? PKV_F32 : PKV_BF16;
  return workspace_for(DecodeShape{num_seqs, n_q, n_kv, head_dim, block_size, act, cache_dtype}, tuning);
}

pkv_status pkv_paged_attention_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                                      const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                      int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                      float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                      void* workspace, size_t workspace_bytes, int32_t* device_error, void* stream) {
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, nullptr, stream);
}

pkv_status pkv_paged_attention_decode_ex(void* out, const void* query, const void* key_cache, const void* value_cache,
                                         const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                         int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                         int64_t num_blocks, float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                         float* lse_out, void* workspace, size_t workspace_bytes, int32_t* device_error,
                                         const pkv_decode_tuning* tuning, void* stream) {
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, tuning, stream);
}

pkv_status pkv_paged_attention_decode_window(void* out, const void* query, const void* key_cache,
                                             const void* value_cache, const float* k_scale, const float* v_scale,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                             int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                             float sm_scale, int window, int sinks, pkv_dtype act_dtype,
                                             pkv_dtype cache_dtype, float* lse_out, void* workspace,
                                             size_t workspace_bytes, int32_t* device_error, void* stream) {
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, nullptr, stream,
                     nullptr, nullptr, window, sinks);
}

pkv_status pkv_quest_page_summaries(const void* key_cache, void* page_min, void* page_max,
                                    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                                    int num_seqs, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    pkv_dtype cache_dtype, int last_page_only, int32_t* device_error, void* stream) {
  if (num_seqs < 0 || n_kv <= 0 || head_dim <= 0 || max_blocks_per_seq < 0 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (block_size != kBlockSize) return PKV_ERR_UNSUPPORTED;
  if (cache_dtype != PKV_BF16 && cache_dtype != PKV_F32) return PKV_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (num_seqs == 0 || max_blocks_per_seq == 0) return PKV_OK;
  if (!key_cache || !page_min || !page_max || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
  return launch_quest_summaries(key_cache, page_min, page_max, block_tables, max_blocks_per_seq, context_lens,
                                num_seqs, n_kv, head_dim, num_blocks, cache_dtype, last_page_only, device_error,
                                static_cast<cudaStream_t>(stream));
}

pkv_status pkv_quest_select(const void* query, const void* page_min, const void* page_max,
                            const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                            int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                            int64_t num_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype, int k_pages,
                            int32_t* selected, float* scores, int32_t* device_error, void* stream) {
  if (num_seqs < 0 || n_q <= 0 || n_kv <= 0 || n_q % n_kv || k_pages < 1 || max_context_len < 0 || num_blocks < 0)
    return PKV_ERR_INVALID_ARG;
  if (act_dtype != PKV_BF16 && act_dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  if (block_size != kBlockSize) return PKV_ERR_UNSUPPORTED;
  if (cache_dtype != PKV_BF16 && cache_dtype != PKV_F32) return PKV_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PKV_OK;
  if (!query || !page_min || !page_max || !block_tables || !context_lens || !selected || !scores)
    return PKV_ERR_INVALID_ARG;
  return launch_quest_select(query, page_min, page_max, block_tables, max_blocks_per_seq, context_lens,
                             max_context_len, num_seqs, n_q, n_kv, head_dim, num_blocks, act_dtype, cache_dtype,
                             k_pages, selected, scores, device_error, static_cast<cudaStream_t>(stream));
}

pkv_status pkv_paged_attention_decode_pages(void* out, const void* query, const void* key_cache,
                                            const void* value_cache, const float* k_scale, const float* v_scale,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                            int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                            float sm_scale, const int32_t* pages, int k_pages, pkv_dtype act_dtype,
                                            pkv_dtype cache_dtype, float* lse_out, void* workspace,
                                            size_t workspace_bytes, int32_t* device_error, void* stream) {
  return pkv_paged_attention_decode_pages_ex(out, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                                             max_blocks_per_seq, context_lens, max_context_len, num_seqs, n_q, n_kv,
                                             head_dim, block_size, num_blocks, sm_scale, pages, k_pages, act_dtype,
                                             cache_dtype, lse_out, workspace, workspace_bytes, device_error, nullptr,
                                             stream);
}

pkv_status pkv_paged_attention_decode_pages_ex(void* out, const void* query, const void* key_cache,
                                               const void* value_cache, const float* k_scale, const float* v_scale,
                                               const int32_t* block_tables, int max_blocks_per_seq,
                                               const int32_t* context_lens, int max_context_len, int num_seqs,
                                               int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                               float sm_scale, const int32_t* pages, int k_pages,
                                               pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                               void* workspace, size_t workspace_bytes, int32_t* device_error,
                                               const pkv_decode_tuning* tuning, void* stream) {
  if (num_seqs > 0 && (!pages || k_pages < 1)) return PKV_ERR_INVALID_ARG;
  if (tuning && tuning->heads_per_cta > 1) return PKV_ERR_INVALID_ARG;  // a page list is per KV head
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, tuning, stream,
                     nullptr, nullptr, 0, 0, pages, k_pages);
}

size_t pkv_shared_prefix_workspace_size_ex(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                           int prefix_blocks, const pkv_decode_tuning* tuning) {
  const DecodeShape s{num_seqs, n_q, n_kv, head_dim, block_size, PKV_BF16, PKV_BF16};
  if (prefix_blocks < 1 || check_decode_shape(s) != PKV_OK) return (size_t)-1;
  if (tuning && tuning->prefix_splits < 0) return (size_t)-1;
  if (num_seqs == 0) return 0;
  TcPlan plan;
  if (plan_tc(s, tuning, &plan) != PKV_OK) return (size_t)-1;
  return (plan.ws_total + 255) / 256 * 256 +
         prefix_workspace_bytes(num_seqs, n_q, n_kv, head_dim, prefix_blocks, tuning ? tuning->prefix_splits : 0);
}

size_t pkv_shared_prefix_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                        int prefix_blocks) {
  return pkv_shared_prefix_workspace_size_ex(num_seqs, n_q, n_kv, head_dim, block_size, prefix_blocks, nullptr);
}

pkv_status pkv_paged_attention_decode_shared_prefix_ex(void* out, const void* query, const void* key,
                                                       const void* value, void* key_cache, void* value_cache,
                                                       const int32_t* block_tables, int max_blocks_per_seq,
                                                       const int32_t* context_lens, int max_context_len,
                                                       int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                                                       int64_t num_blocks, float sm_scale, int prefix_blocks,
                                                       pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                                       void* workspace, size_t workspace_bytes,
                                                       int32_t* device_error, const pkv_decode_tuning* tuning,
                                                       void* stream) {
  if (prefix_blocks < 1) return PKV_ERR_INVALID_ARG;
  if ((key == nullptr) != (value == nullptr)) return PKV_ERR_INVALID_ARG;
  if (key && (!aligned16(key) || !aligned16(value))) return PKV_ERR_INVALID_ARG;
  if (max_context_len <= prefix_blocks * block_size && num_seqs > 0) return PKV_ERR_INVALID_ARG;
  return decode_impl(out, query, key_cache, value_cache, nullptr, nullptr, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, tuning, stream, key,
                     value, 0, 0, nullptr, 0, prefix_blocks);
}

pkv_status pkv_paged_attention_decode_shared_prefix(void* out, const void* query, const void* key, const void* value,
                                                    void* key_cache, void* value_cache, const int32_t* block_tables,
                                                    int max_blocks_per_seq, const int32_t* context_lens,
                                                    int max_context_len, int num_seqs, int n_q, int n_kv,
                                                    int head_dim, int block_size, int64_t num_blocks, float sm_scale,
                                                    int prefix_blocks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                                    float* lse_out, void* workspace, size_t workspace_bytes,
                                                    int32_t* device_error, void* stream) {
  return pkv_paged_attention_decode_shared_prefix_ex(out, query, key, value, key_cache, value_cache, block_tables,
                                                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, n_q,
                                                     n_kv, head_dim, block_size, num_blocks, sm_scale, prefix_blocks,
                                                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes,
                                                     device_error, nullptr, stream);
}

pkv_status pkv_paged_decode_step_ex(void* out, const void* query, const void* key, const void* value, void* key_cache,
                                    void* value_cache, float* k_scale, float* v_scale, const int32_t* block_tables,
                                    int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                    int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                    void* workspace, size_t workspace_bytes, int32_t* device_error,
                                    const pkv_decode_tuning* tuning, void* stream) {
  if (num_seqs > 0 && (!key || !value || !aligned16(key) || !aligned16(value))) return PKV_ERR_INVALID_ARG;
  if (head_scaled(cache_dtype) && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, tuning, stream, key,
                     value);
}

pkv_status pkv_paged_decode_step(void* out, const void* query, const void* key, const void* value, void* key_cache,
                                 void* value_cache, float* k_scale, float* v_scale, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* context_lens, int max_context_len,
                                 int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                 float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out,
                                 void* workspace, size_t workspace_bytes, int32_t* device_error, void* stream) {
  return pkv_paged_decode_step_ex(out, query, key, value, key_cache, value_cache, k_scale, v_scale, block_tables,
                                  max_blocks_per_seq, context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim,
                                  block_size, num_blocks, sm_scale, act_dtype, cache_dtype, lse_out, workspace,
                                  workspace_bytes, device_error, nullptr, stream);
}

pkv_status pkv_paged_decode_step_window(void* out, const void* query, const void* key, const void* value,
                                        void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                                        const int32_t* block_tables, int max_blocks_per_seq,
                                        const int32_t* context_lens, int max_context_len, int num_seqs, int n_q,
                                        int n_kv, int head_dim, int block_size, int64_t num_blocks, float sm_scale,
                                        int window, int sinks, pkv_dtype act_dtype, pkv_dtype cache_dtype,
                                        float* lse_out, void* workspace, size_t workspace_bytes,
                                        int32_t* device_error, void* stream) {
  if (num_seqs > 0 && (!key || !value || !aligned16(key) || !aligned16(value))) return PKV_ERR_INVALID_ARG;
  if (head_scaled(cache_dtype) && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
  return decode_impl(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq,
                     context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim, block_size, num_blocks, sm_scale,
                     act_dtype, cache_dtype, lse_out, workspace, workspace_bytes, device_error, nullptr, stream, key,
                     value, window, sinks);
}

// ---------------------------------------------------------------- 2-bit KIVI cache
static pkv_status check_kivi_shape(int num_seqs, int n_q, int n_kv, int head_dim, int block_size, pkv_dtype act) {
  if (num_seqs < 0 || n_q <= 0 || n_kv <= 0 || head_dim <= 0 || block_size <= 0) return PKV_ERR_INVALID_ARG;
  if (n_q % n_kv != 0 || (act != PKV_F32 && act != PKV_BF16)) return PKV_ERR_INVALID_ARG;
  if (act != PKV_BF16 || head_dim != 128 || block_size != kBlockSize) return PKV_ERR_UNSUPPORTED;
  if (n_q / n_kv > 64) return PKV_ERR_UNSUPPORTED;
  return PKV_OK;
}

static pkv_status kivi_plan(int num_seqs, int n_q, int n_kv, TcPlan* plan, size_t* state_off, size_t* total) {
  const DecodeShape s{num_seqs, n_q, n_kv, 128, kBlockSize, PKV_BF16, PKV_KIVI2};
  pkv_status st = plan_tc(s, nullptr, plan);
  if (st != PKV_OK) return st;
  // the residual pass's state after the decode's scratch
  *state_off = (plan->ws_total + 255) / 256 * 256;
  *total = *state_off + kivi_state_bytes(num_seqs, n_q);
  return PKV_OK;
}

size_t pkv_kivi_workspace_size(int num_seqs, int n_q, int n_kv, int head_dim, int block_size) {
  if (check_kivi_shape(num_seqs, n_q, n_kv, head_dim, block_size, PKV_BF16) != PKV_OK) return (size_t)-1;
  if (num_seqs == 0) return 0;
  TcPlan plan;
  size_t off = 0, total = 0;
  if (kivi_plan(num_seqs, n_q, n_kv, &plan, &off, &total) != PKV_OK) return (size_t)-1;
  return total;
}

pkv_status pkv_kivi_quantize_blocks(const void* key_rows, const void* value_rows, const int32_t* dst_blocks,
                                    int64_t num_src_blocks, void* key_cache, void* value_cache, float* k_scale,
                                    float* v_scale, int n_kv, int head_dim, int block_size, int64_t num_blocks,
                                    pkv_dtype act_dtype, int32_t* device_error, void* stream) {
  pkv_status st = check_kivi_shape(1, n_kv, n_kv, head_dim, block_size, act_dtype);
  if (st != PKV_OK) return st;
  if (num_src_blocks < 0 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (num_src_blocks * (int64_t)n_kv > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  if (num_src_blocks == 0) return PKV_OK;
  if (!key_rows || !value_rows || !dst_blocks || !key_cache || !value_cache || !k_scale || !v_scale)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(key_rows) || !aligned16(value_rows)) return PKV_ERR_INVALID_ARG;
  return launch_kivi_quantize_blocks(key_rows, value_rows, dst_blocks, num_src_blocks, key_cache, value_cache,
                                     k_scale, v_scale, n_kv, num_blocks, device_error,
                                     static_cast<cudaStream_t>(stream));
}

pkv_status pkv_kivi_decode(void* out, const void* query, const void* key, const void* value, void* residual_k,
                           void* residual_v, void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                           const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                           int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int block_size,
                           int64_t num_blocks, float sm_scale, pkv_dtype act_dtype, float* lse_out, void* workspace,
                           size_t workspace_bytes, int32_t* device_error, void* stream) {
  pkv_status st = check_kivi_shape(num_seqs, n_q, n_kv, head_dim, block_size, act_dtype);
  if (st != PKV_OK) return st;
  if (max_blocks_per_seq < 0 || max_context_len < 0 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (num_blocks * (int64_t)block_size > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  if (num_blocks * (int64_t)n_kv * 4 > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;  // K-scale rows (int32 TMA coordinate)
  if ((int64_t)num_seqs * n_kv > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !query || !residual_k || !residual_v || !key_cache || !value_cache || !k_scale || !v_scale ||
      !block_tables || !context_lens)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(residual_k) || !aligned16(residual_v) ||
      !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(k_scale) || !aligned16(v_scale))
    return PKV_ERR_INVALID_ARG;
  if ((key == nullptr) != (value == nullptr)) return PKV_ERR_INVALID_ARG;
  if (key && (!aligned16(key) || !aligned16(value))) return PKV_ERR_INVALID_ARG;
  if (max_blocks_per_seq == 0 && max_context_len > 0) return PKV_ERR_INVALID_ARG;
  TcPlan plan;
  size_t state_off = 0, need = 0;
  st = kivi_plan(num_seqs, n_q, n_kv, &plan, &state_off, &need);
  if (st != PKV_OK) return st;
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);

  KiviArgs k{query, key, value, residual_k, residual_v, key_cache, value_cache, k_scale, v_scale, block_tables,
             max_blocks_per_seq, context_lens,
             (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * kBlockSize), num_blocks,
             num_seqs, n_q, n_kv, sm_scale, device_error};
  PrefixState state;
  st = launch_kivi_residual(k, static_cast<uint8_t*>(workspace) + state_off, &state, strm);
  if (st != PKV_OK) return st;

  const DecodeShape s{num_seqs, n_q, n_kv, head_dim, block_size, act_dtype, PKV_KIVI2};
  TcArgs a{out, query, key_cache, value_cache, k_scale, v_scale, block_tables, max_blocks_per_seq, context_lens,
           max_context_len, num_blocks, sm_scale, lse_out, workspace, device_error};
  a.prefix = state;
  plan.overlap_prologue = true;  // the decode's prologue overlaps the residual pass
  return launch_tc(s, plan, a, strm);
}

pkv_status pkv_copy_blocks(void* key_cache, void* value_cache, float* k_scale, float* v_scale,
                           const int64_t* block_mapping, int64_t num_pairs, int n_kv, int head_dim, int block_size,
                           int64_t num_blocks, pkv_dtype cache_dtype, int32_t* device_error, void* stream) {
  const void* src[4];
  void* dst[4];
  size_t bpb[4];
  int npools = 0;
  pkv_status st = move_plan(key_cache, value_cache, k_scale, v_scale, key_cache, value_cache, k_scale, v_scale,
                            block_mapping, num_pairs, n_kv, head_dim, block_size, cache_dtype, src, dst, bpb, &npools);
  if (st != PKV_OK) return st;
  if (num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (num_pairs == 0) return PKV_OK;
  st = device_addresses(src, dst, npools, &block_mapping);
  if (st != PKV_OK) return st;
  return launch_move_blocks(src, dst, bpb, npools, block_mapping, num_pairs, num_blocks, num_blocks, device_error,
                            static_cast<cudaStream_t>(stream));
}

pkv_status pkv_swap_blocks(const void* src_key, const void* src_value, const float* src_k_scale,
                           const float* src_v_scale, int64_t src_num_blocks, void* dst_key, void* dst_value,
                           float* dst_k_scale, float* dst_v_scale, int64_t dst_num_blocks,
                           const int64_t* block_mapping, int64_t num_pairs, int n_kv, int head_dim, int block_size,
                           pkv_dtype cache_dtype, int32_t* device_error, void* stream) {
  const void* src[4];
  void* dst[4];
  size_t bpb[4];
  int npools = 0;
  pkv_status st = move_plan(src_key, src_value, src_k_scale, src_v_scale, dst_key, dst_value, dst_k_scale,
                            dst_v_scale, block_mapping, num_pairs, n_kv, head_dim, block_size, cache_dtype, src, dst,
                            bpb, &npools);
  if (st != PKV_OK) return st;
  if (src_num_blocks < 0 || dst_num_blocks < 0) return PKV_ERR_INVALID_ARG;
  if (num_pairs == 0) return PKV_OK;
  st = device_addresses(src, dst, npools, &block_mapping);
  if (st != PKV_OK) return st;
  return launch_move_blocks(src, dst, bpb, npools, block_mapping, num_pairs, src_num_blocks, dst_num_blocks,
                            device_error, static_cast<cudaStream_t>(stream));
}

const char* pkv_status_string(pkv_status status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* pkv_last_cuda_error(void) { return g_last_cuda_error; }

int pkv_version(void) { return 100; }

}  // extern "C"
