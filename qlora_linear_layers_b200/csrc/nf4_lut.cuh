// NF4 -> bf16 expansion in registers, shared by the tensor-core GEMMs.
//
// A converter thread owns one weight row and one NF4 block (64 weights) per
// step.  It builds the block's 16-entry bf16 table RNbf16(RN32(q[i] * a^)) --
// the exact values nf4_dequantize writes -- as two byte planes, then expands
// packed codes with prmt (21 integer ops per 8 weights).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace qnf4 {

// 16-entry bf16 table for one block, held as byte planes: L[i] holds the low
// bytes of entries 4i..4i+3, H[i] the high bytes.
struct Lut { uint32_t L[4], H[4]; };

__device__ __forceinline__ Lut build_lut(float a, const float* q) {
  uint32_t P[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    P[i] = pack_bf16x2(__fmul_rn(q[2 * i], a), __fmul_rn(q[2 * i + 1], a));
  Lut l;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    l.L[i] = prmt(P[2 * i], P[2 * i + 1], 0x6420);
    l.H[i] = prmt(P[2 * i], P[2 * i + 1], 0x7531);
  }
  return l;
}

// Expand one 32-bit word of packed codes (8 weights, byte j = element 2j in
// the high nibble, 2j+1 in the low nibble) into 4 bf16x2 words ordered by K.
__device__ __forceinline__ void lookup8(uint32_t w, const Lut& l, uint32_t* out) {
  const uint32_t s7 = w & 0x77777777u;                       // entry index within a plane half
  const uint32_t t = ((w >> 1) & 0x44444444u) | 0x32103210u; // pick half 0-7 or 8-15 per byte
  {
    const uint32_t xl = prmt(l.L[0], l.L[1], s7), yl = prmt(l.L[2], l.L[3], s7);
    const uint32_t xh = prmt(l.H[0], l.H[1], s7), yh = prmt(l.H[2], l.H[3], s7);
    const uint32_t lo = prmt(xl, yl, t), hi = prmt(xh, yh, t);
    out[0] = prmt(lo, hi, 0x4051);
    out[1] = prmt(lo, hi, 0x6273);
  }
  {
    const uint32_t s7h = s7 >> 16, th = t >> 16;
    const uint32_t xl = prmt(l.L[0], l.L[1], s7h), yl = prmt(l.L[2], l.L[3], s7h);
    const uint32_t xh = prmt(l.H[0], l.H[1], s7h), yh = prmt(l.H[2], l.H[3], s7h);
    const uint32_t lo = prmt(xl, yl, th), hi = prmt(xh, yh, th);
    out[2] = prmt(lo, hi, 0x4051);
    out[3] = prmt(lo, hi, 0x6273);
  }
}

}  // namespace qnf4
