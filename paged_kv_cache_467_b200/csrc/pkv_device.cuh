// Device-side building blocks for sm_100a: mbarriers, TMA / bulk copies into
// shared memory, ldmatrix, legacy-path mma.sync, movmatrix and byte unpacking.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace pkv {

// Error bits OR-ed into the caller's device error word (mirrors include/pkv.h).
enum : int {
  DEVERR_SLOT_RANGE = 0x1,
  DEVERR_BLOCK_RANGE = 0x2,
  DEVERR_CONTEXT_LEN = 0x4,
  DEVERR_TIMEOUT = 0x8,
  DEVERR_PREFIX = 0x10,
};

// A bounded wait gives up after this many SM clock cycles (about 1 s at 2 GHz).
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ void flag_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      "  .reg .pred p;\n"
      "  mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "  selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false if the wait ran
// out (after `limit` SM clock cycles).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}

// ------------------------------------------------------------ bulk copies
// Tiled TMA load of one box of a rank-3 tensor map into shared memory,
// completing on an mbarrier.  Out-of-range boxes are zero-filled by the TMA unit.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// Tiled TMA load of one box of a rank-2 tensor map (same completion rules).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// Contiguous bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Orders this thread's earlier generic-proxy global stores before later
// async-proxy (TMA) accesses that are ordered after it.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Programmatic dependent launch: let the next grid on the stream be scheduled,
// and wait until the previous grid has completed and its writes are visible.
// Both are no-ops for a grid launched without the programmatic attribute.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait_prerequisites() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 16-byte global -> shared copy through the async copy unit; src_bytes 0
// zero-fills the destination and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------ fragments
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// D(16x8, f32) += A(16x16) * B(16x8), bf16 or f16 operands.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8, s32) += A(16x32) * B(32x8), 8-bit integer operands: A signed
// (mma_s8s8) or unsigned (mma_u8s8), B signed.
__device__ __forceinline__ void mma_s8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(16x8, f32) += A(16x32) * B(32x8), FP8 operands: A E4M3 (a_e5m2 = false)
// or E5M2 codes, B E4M3.
template <bool A_E5M2>
__device__ __forceinline__ void mma_fp8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (A_E5M2) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e5m2.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Four int8 values packed into a word, element 0 in the low byte.
__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) | ((uint32_t)d << 24);
}

// Transpose an 8x8 matrix of 16-bit values held in the ldmatrix fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two signed int8 codes (bytes 0 and 1 of `sel`-arranged word w, already XOR-ed
// with 0x80) -> f16x2 holding the exact integers.  The byte u = code + 128 is
// placed in the low mantissa byte of 0x6400 (= 1024.0), giving 1024 + u, and
// 1152 = 1024 + 128 is subtracted; integers below 2048 are exact in f16.
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t biased_word, uint32_t sel) {
  const uint32_t h = prmt(biased_word, 0x64646464u, sel);
  __half2 v = *reinterpret_cast<const __half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half(0x6480)));  // 0x6480 = 1152.0
  return *reinterpret_cast<uint32_t*>(&v);
}

// The two E4M3 pairs of w (bytes 0-1 and bytes 2-3) -> two f16x2 words holding
// the codes' values exactly (the hardware conversion; NaN codes give NaN).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n"
      "  .reg .b16 l, h;\n"
      "  mov.b32 {l, h}, %2;\n"
      "  cvt.rn.f16x2.e4m3x2 %0, l;\n"
      "  cvt.rn.f16x2.e4m3x2 %1, h;\n"
      "}\n"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Two E4M3 bytes held in bits [15:8] and [31:24] of t (other bits ignored) ->
// f16x2 equal to the E4M3 values times 2^-8, exactly.  The E4M3 magnitude bits
// EEEE.MMM moved to f16 bits [13:7] read as an f16 with exponent field EEEE and
// mantissa MMM0000000: the exponent biases differ by 8 (15 vs 7), subnormals
// included, so the f16 value is the E4M3 value scaled by 2^-8.
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2_div256(uint32_t t) {
  return ((t >> 1) & 0x3F803F80u) | (t & 0x80008000u);
}

// Two 4-bit codes held as offset-binary nibbles (code + 8) at bits [3:0] and
// [19:16] of t (other bits ignored) -> f16x2 of the codes, exactly: the nibble
// n ORed into the mantissa of 1024.0 (0x6400) reads as 1024 + n, and
// subtracting 1032 leaves n - 8.
__device__ __forceinline__ uint32_t i4x2_to_f16x2(uint32_t t) {
  const uint32_t h = (t & 0x000F000Fu) | 0x64006400u;
  __half2 v = *reinterpret_cast<const __half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half(0x6408)));  // 0x6408 = 1032.0
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two 2-bit two's-complement codes at bits [1:0] and [17:16] of t (other bits
// ignored) -> f16x2 of the codes, exactly.  XOR with 2 turns a code c into
// c + 2 in [0, 3]; ORed into the mantissa of 1024.0 it reads as 1026 + c, and
// subtracting 1026 leaves c.  One LOP3 and one HSUB2.
__device__ __forceinline__ uint32_t i2x2_to_f16x2(uint32_t t) {
  const uint32_t h = (t & 0x00030003u) ^ 0x64026402u;
  __half2 v = *reinterpret_cast<const __half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half(0x6402)));  // 0x6402 = 1026.0
  return *reinterpret_cast<uint32_t*>(&v);
}

// The two 2-bit two's-complement codes at bits [2s, 2s+1] and [16+2s, 17+2s]
// of t (other bits ignored) -> f16x2 of the codes times 4^s, exactly: XOR with
// 2 << 2s turns a code c in place into (c + 2) << 2s, which ORed into the
// mantissa of 1024.0 reads as 1024 + (c + 2) 4^s; subtracting 1024 + 2 * 4^s
// leaves c * 4^s.  One LOP3 and one HSUB2, no shift (s is a constant once the
// caller's loop is unrolled).
__device__ __forceinline__ uint32_t i2x2_at_to_f16x2(uint32_t t, int s) {
  const uint32_t mask = 0x00030003u << (2 * s);
  const uint32_t flip = 0x64006400u | (0x00020002u << (2 * s));
  const unsigned short base = (unsigned short)(0x6400 + (2 << (2 * s)));  // f16 of 1024 + 2 * 4^s
  const uint32_t h = (t & mask) ^ flip;
  __half2 v = *reinterpret_cast<const __half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half(base)));
  return *reinterpret_cast<uint32_t*>(&v);
}

// The two two's-complement 4-bit codes in the low (HI = false) or high
// (HI = true) nibbles of bytes 0 and 2 of t -> f16x2 of the codes (low) or of
// 16 times the codes (high), exactly: XOR with 8 << shift makes the nibble
// n = code + 8 in place, which ORed into the mantissa of 1024.0 reads as
// 1024 + n (or 1024 + 16 n); subtracting 1032 (or 1152) leaves the code (or
// 16 times it).  One LOP3 and one HSUB2, no shift.
template <bool HI>
__device__ __forceinline__ uint32_t i4x2_at_to_f16x2(uint32_t t) {
  constexpr uint32_t mask = HI ? 0x00F000F0u : 0x000F000Fu;
  constexpr uint32_t flip = HI ? 0x64806480u : 0x64086408u;
  constexpr unsigned short base = HI ? 0x6480 : 0x6408;  // f16 of 1152 = 1024 + 16 * 8, of 1032 = 1024 + 8
  const uint32_t h = (t & mask) ^ flip;
  __half2 v = *reinterpret_cast<const __half2*>(&h);
  v = __hsub2(v, __half2half2(__ushort_as_half(base)));
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// 2^x on the special-function unit (flush-to-zero, approximate).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace pkv
