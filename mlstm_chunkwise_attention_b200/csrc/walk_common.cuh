// Pieces shared by the chunk walkers (tc_fwd_walk.cu, tc_bwd_walk.cu): one CTA per
// head walks its chunks with the state (or its gradient) in TMEM; chunk tiles are
// 128 rows x 128 bf16, stored as two 128-byte-swizzled 64-column blocks.
#pragma once

#include <stdint.h>

#include "tc_common.cuh"

namespace mlstm {
namespace walk {

constexpr int TILE = 32768;  // one 128 x 128 bf16 tile

// Byte offset of (row, col) in a tile: the layout TMA writes with a 64-element,
// 128-byte-swizzled box, and the K- or MN-major operand layout of tcgen05.mma.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return (uint32_t)((col >> 6) * 16384 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                    (col & 7) * 2);
}

// AND of v over the NT threads of the row warps (named barrier 1).
template <int NT>
__device__ __forceinline__ bool rows_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(NT)
      : "memory");
  return r != 0;
}

// Wait until every bulk store group of this thread but the newest has read its source.
__device__ __forceinline__ void bulk_wait_read_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Two consecutive 32-bit TMEM columns of this thread's lane (32x32b.x2), waited on.
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, float& a, float& b) {
  uint32_t r0, r1;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r0), "=r"(r1)
      : "r"(taddr)
      : "memory");
  a = __uint_as_float(r0);
  b = __uint_as_float(r1);
}

// Element t (0..127) of row r (0 or 1) of a 16 x 128 K-major bf16 operand tile (the B
// operand of an N = 16 product): two 2 KB blocks of 64 K-elements, rows of 128 bytes.
__device__ __forceinline__ uint32_t n16_off(int r, int t) {
  return (uint32_t)((t >> 6) * 2048 + r * 128 + ((((t & 63) >> 3) ^ r) << 4) + (t & 7) * 2);
}

// A pair of fp32 values as hi = bf16(x) and lo = bf16(x - hi), each a packed bf16x2 word
// (first value in the low half); hi + lo keeps about 16 mantissa bits.  One packed
// conversion per plane; the hi halves are widened back by a shift and a mask.
__device__ __forceinline__ void split_hi_lo(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = tc::pack_bf16(x0, x1);
  const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
  lo = tc::pack_bf16(x0 - h0, x1 - h1);
}

// w = f x over 32 fp32 values held as raw bits, two lanes per f32x2 multiply.
__device__ __forceinline__ void scale32(const uint32_t (&x)[32], float f, uint32_t (&w)[32]) {
  const uint64_t f2 = tc::f2_make(f, f);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float2 y =
        tc::f2_split(tc::f2_mul(tc::f2_make(__uint_as_float(x[e]), __uint_as_float(x[e + 1])), f2));
    w[e] = __float_as_uint(y.x);
    w[e + 1] = __float_as_uint(y.y);
  }
}

// The two bf16 values of a packed word as fp32.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace walk
}  // namespace mlstm
