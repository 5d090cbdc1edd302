// nf4_dequant.cuh -- NF4 dequantisation of one 64-element block row segment, shared by the
// GEMM mainloop and the dequant export kernel.
//
// deq(code) = bf16(fp32(level[code] * absmax)): each level is multiplied by the block's
// absmax in fp32 (round to nearest) and rounded once more to bf16 (round to nearest even).
// All 64 elements of a block share the absmax, so the 16 possible bf16 results are built
// once per block into a register table and every element becomes a table lookup done with
// byte permutes: the table is split into a low-byte plane and a high-byte plane (16 bytes,
// i.e. 4 registers, each); `prmt` picks bytes by a 3-bit index out of 8, so a 4-bit code
// takes two picks (levels 0-7 and 8-15) and a third `prmt` chooses by the code's top bit.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace qlora {

// The fp32 codebook (16 ascending levels) and its 15 fp32 midpoints, passed by value in
// kernel parameters (constant bank).
struct Codebook {
  float level[16];
  float mid[15];
};

struct Nf4Lut {
  uint32_t lo[4];  // byte i of lo[j] = low byte of bf16 table entry 4j+i
  uint32_t hi[4];  // byte i of hi[j] = high byte of bf16 table entry 4j+i
};

__device__ __forceinline__ void nf4_build_lut(const Codebook& cb, float absmax, Nf4Lut& t) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    p[j] = pack_bf16x2(__fmul_rn(cb.level[2 * j], absmax), __fmul_rn(cb.level[2 * j + 1], absmax));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.lo[i] = prmt(p[2 * i], p[2 * i + 1], 0x6420u);
    t.hi[i] = prmt(p[2 * i], p[2 * i + 1], 0x7531u);
  }
}

// Four codes held in the low 16 bits of `sel3` (3-bit indices, bit 3 cleared) and `msel`
// (top-bit chooser nibbles i + 4*bit3) -> their 4 low bytes and 4 high bytes.
__device__ __forceinline__ void nf4_pick4(const Nf4Lut& t, uint32_t sel3, uint32_t msel,
                                          uint32_t& lo, uint32_t& hi) {
  const uint32_t la = prmt(t.lo[0], t.lo[1], sel3);
  const uint32_t lb = prmt(t.lo[2], t.lo[3], sel3);
  const uint32_t ha = prmt(t.hi[0], t.hi[1], sel3);
  const uint32_t hb = prmt(t.hi[2], t.hi[3], sel3);
  lo = prmt(la, lb, msel);
  hi = prmt(ha, hb, msel);
}

// One 32-bit word of packed codes (4 bytes = 8 elements; element 2j in the high nibble of
// byte j) -> 8 bf16 values in element order, as 4 bf16x2 words.
//
// Nibble i of the word holds element i^1, so each pick returns bytes for elements
// (1, 0, 3, 2); the final permutes put them back in order and interleave low/high bytes.
__device__ __forceinline__ uint4 nf4_lookup8(const Nf4Lut& t, uint32_t w) {
  const uint32_t sel3 = w & 0x77777777u;
  const uint32_t msel = ((w >> 1) & 0x44444444u) | 0x32103210u;
  uint32_t l0, h0, l1, h1;
  nf4_pick4(t, sel3, msel, l0, h0);
  nf4_pick4(t, sel3 >> 16, msel >> 16, l1, h1);
  uint4 o;
  o.x = prmt(l0, h0, 0x4051u);
  o.y = prmt(l0, h0, 0x6273u);
  o.z = prmt(l1, h1, 0x4051u);
  o.w = prmt(l1, h1, 0x6273u);
  return o;
}

// Effective absmax of block `blk`: fp32 absmax, or fp32(q8 * scale[blk / 256]) when the
// absmax is double-quantised.
__device__ __forceinline__ float nf4_block_absmax(const float* __restrict__ absmax,
                                                  const uint8_t* __restrict__ q8,
                                                  const float* __restrict__ scale, int dq,
                                                  long long blk) {
  if (!dq) return __ldg(absmax + blk);
  const float s = __ldg(scale + (blk >> 8));
  return __fmul_rn(static_cast<float>(__ldg(q8 + blk)), s);
}

}  // namespace qlora
