// Whole-block movers of a paged cache.
//
//  * pkv_copy_blocks: duplicate physical blocks inside one pool, for
//    copy-on-write of shared blocks ("Chapter 18 - KV-Cache Optimization
//    Strategies", Prefix Caching; KV-cache overview page t13_4, copy-on-write
//    paragraph).
//  * pkv_swap_blocks: move blocks between two pools, e.g. device memory and
//    page-locked host memory, to offload them and bring them back ("KV Cache
//    Engineering for LLM Serving", section 12, Cache Offloading from GPU).
//
// One kernel serves both: CTA (pair, 4 KiB chunk, pool) moves one 16-byte
// vector per thread, so a 32 KiB bf16 block is 8 CTAs per pool and every
// access is a coalesced 16-byte load or store.  Host pools are reached
// directly through unified addressing (page-locked, mapped memory).
#include <cuda_runtime.h>

#include "internal.h"
#include "pkv_device.cuh"

namespace pkv {

constexpr int kMovePools = 4;          // K, V, int8 K scales, int8 V scales
constexpr int kMoveChunkBytes = 4096;  // bytes of a block one CTA moves

struct MoveParams {
  const uint8_t* src[kMovePools];
  uint8_t* dst[kMovePools];
  unsigned long long bytes_per_block[kMovePools];
  const int64_t* pairs;  // [num_pairs, 2] (src block, dst block)
  long long num_pairs;
  long long src_blocks, dst_blocks;
  int chunks;  // ceil(largest bytes_per_block / kMoveChunkBytes)
  int* err;
};

__global__ void __launch_bounds__(256) move_blocks_kernel(const MoveParams p) {
  const long long pc = blockIdx.x;
  const long long pair = pc / p.chunks;
  const int chunk = (int)(pc - pair * p.chunks);
  const int pool = blockIdx.y;
  if (pair >= p.num_pairs) return;
  const long long s = __ldg(p.pairs + 2 * pair), d = __ldg(p.pairs + 2 * pair + 1);
  if (s < 0 || s >= p.src_blocks || d < 0 || d >= p.dst_blocks) {
    if (threadIdx.x == 0 && chunk == 0 && pool == 0) flag_error(p.err, DEVERR_BLOCK_RANGE);
    return;
  }
  const unsigned long long bpb = p.bytes_per_block[pool];
  const unsigned long long off = (unsigned long long)chunk * kMoveChunkBytes + threadIdx.x * 16ull;
  if (off >= bpb) return;
  const uint4 v = *reinterpret_cast<const uint4*>(p.src[pool] + (unsigned long long)s * bpb + off);
  *reinterpret_cast<uint4*>(p.dst[pool] + (unsigned long long)d * bpb + off) = v;
}

pkv_status launch_move_blocks(const void* const src[4], void* const dst[4], const size_t bytes_per_block[4], int npools,
                              const int64_t* pairs, int64_t num_pairs, int64_t src_blocks, int64_t dst_blocks,
                              int32_t* device_error, cudaStream_t stream) {
  MoveParams p = {};
  size_t largest = 0;
  for (int i = 0; i < npools; ++i) {
    p.src[i] = static_cast<const uint8_t*>(src[i]);
    p.dst[i] = static_cast<uint8_t*>(dst[i]);
    p.bytes_per_block[i] = bytes_per_block[i];
    if (bytes_per_block[i] > largest) largest = bytes_per_block[i];
  }
  p.pairs = pairs;
  p.num_pairs = num_pairs;
  p.src_blocks = src_blocks;
  p.dst_blocks = dst_blocks;
  p.chunks = (int)((largest + kMoveChunkBytes - 1) / kMoveChunkBytes);
  p.err = device_error;
  const long long gx = num_pairs * p.chunks;
  if (gx > 0x7FFFFFFFLL) return PKV_ERR_UNSUPPORTED;
  move_blocks_kernel<<<dim3((unsigned)gx, npools), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "move_blocks_kernel launch");
  return PKV_OK;
}

}  // namespace pkv
