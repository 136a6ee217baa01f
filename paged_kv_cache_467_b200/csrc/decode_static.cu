// Decode attention with a library-owned scratch buffer, for callers that
// cannot allocate device memory themselves.
//
// Some callers have no way to hand the library a workspace: a library loaded
// inside a host runtime that owns every device allocation and exposes no
// allocator to plug-ins, or a serving loop that must never call cudaMalloc
// because cudaMalloc can synchronise the device.  For them,
// pkv_paged_attention_decode_static runs the same decode kernel as
// pkv_paged_attention_decode, with its scratch (partial results of split
// sequences and their merge descriptors) in one fixed array that is part of
// the loaded library.
//
// The array below is kStaticScratchBytes (16 MiB) of device memory that every
// GPU which loads libpkv holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace pkv {

constexpr size_t kStaticScratchBytes = 16u << 20;
constexpr int kMaxDevices = 64;

// Device-side scratch.  Host code must not pass this symbol to a kernel: on the
// host it only names the variable; its device address comes from
// cudaGetSymbolAddress (see static_scratch_address).
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device, looked up once per
// device (cudaGetSymbolAddress) and remembered.  nullptr when the lookup fails.
static void* static_scratch_address(int device, cudaError_t* err) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_static_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[device] = p;
  }
  *err = cudaSuccess;
  return addr[device];
}

}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_paged_attention_decode_static(
    void* out, const void* query, const void* key_cache, const void* value_cache, const float* k_scale,
    const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    int max_context_len, int num_seqs, int n_q, int n_kv, int head_dim, int block_size, int64_t num_blocks,
    float sm_scale, pkv_dtype act_dtype, pkv_dtype cache_dtype, float* lse_out, int32_t* device_error, void* stream) {
  // Scratch this shape needs; the shape checks of the regular entry point run here too.
  const size_t need = pkv_paged_attention_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size, cache_dtype);
  if (need == (size_t)-1) {
    // unsupported shape or no device: the regular entry point reports which
    return pkv_paged_attention_decode(out, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                                      max_blocks_per_seq, context_lens, max_context_len, num_seqs, n_q, n_kv,
                                      head_dim, block_size, num_blocks, sm_scale, act_dtype, cache_dtype, lse_out,
                                      nullptr, 0, device_error, stream);
  }
  if (need > kStaticScratchBytes) {
    note_error("pkv_paged_attention_decode_static: this shape needs %zu bytes of scratch, more than the %zu-byte "
               "static array; use pkv_paged_attention_decode with a caller-owned workspace",
               need, kStaticScratchBytes);
    return PKV_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return PKV_ERR_UNSUPPORTED;
    scratch = static_scratch_address(dev, &e);
    if (!scratch) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    // Whatever the previous call left there is overwritten before it is read.
  }
  return pkv_paged_attention_decode(out, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                                    max_blocks_per_seq, context_lens, max_context_len, num_seqs, n_q, n_kv, head_dim,
                                    block_size, num_blocks, sm_scale, act_dtype, cache_dtype, lse_out, scratch,
                                    scratch ? kStaticScratchBytes : 0, device_error, stream);
}
