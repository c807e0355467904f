// nf4_decode.cuh — double dequantisation of NF4 codes to bfloat16 in registers.
//
// "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
// §The QLoRA layer, end to end: doubleDequant first recovers the block
// constant from its 8-bit code with the group's float32 scale, then scales the
// looked-up NF4 level.  Here:
//     c2_hat = fmaf(E4M3(e_b), S_g, mu)
//     w_hat  = bf16_rn(float32(level[code] * c2_hat))
// Each thread owns one 64-element block at a time: it evaluates the 16
// possible w_hat of its block once (16 multiplies, 8 packed conversions) and
// then expands codes with byte permutes only: the low and the high bytes of the
// 16 bfloat16 values live in 4 + 4 registers; two permutes select among codes
// 0-7 and 8-15, a third merges on the code's top bit.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace qlora {

struct Nf4Levels {
  float q[16];
};

// OCP E4M3FN byte -> float32 (exact; via the hardware fp8 -> f16x2 conversion).
__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  const uint16_t two = static_cast<uint16_t>(byte | (byte << 8));
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
  const uint16_t h = static_cast<uint16_t>(h2 & 0xFFFFu);
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

__device__ __forceinline__ float reconstruct_c2(uint32_t e_byte, float s_g, float mu) {
  return __fmaf_rn(e4m3_to_f32(e_byte), s_g, mu);
}

// Byte-plane lookup table of the 16 w_hat values of one block.
struct BlockLut {
  uint32_t lo[4];  // lo[t] byte i = low  byte of w_hat(level 4t+i)
  uint32_t hi[4];  // hi[t] byte i = high byte of w_hat(level 4t+i)
};

__device__ __forceinline__ BlockLut make_lut(float c2h, const Nf4Levels &lv) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(__fmul_rn(lv.q[2 * j], c2h), __fmul_rn(lv.q[2 * j + 1], c2h));
  BlockLut t;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    t.lo[j] = prmt(p[2 * j], p[2 * j + 1], 0x6420u);
    t.hi[j] = prmt(p[2 * j], p[2 * j + 1], 0x7531u);
  }
  return t;
}

// Four codes in the low 16 bits of (s7, sm) -> two bf16x2 words.
// Nibble order of a packed word: bits 0-3 element 1, 4-7 element 0, 8-11 element 3,
// 12-15 element 2 (even element in the high nibble of each byte).
__device__ __forceinline__ void decode4(uint32_t s7, uint32_t sm, const BlockLut &t, uint32_t &o01,
                                        uint32_t &o23) {
  const uint32_t la = prmt(t.lo[0], t.lo[1], s7);
  const uint32_t lb = prmt(t.lo[2], t.lo[3], s7);
  const uint32_t ha = prmt(t.hi[0], t.hi[1], s7);
  const uint32_t hb = prmt(t.hi[2], t.hi[3], s7);
  const uint32_t l = prmt(la, lb, sm);
  const uint32_t h = prmt(ha, hb, sm);
  o01 = prmt(l, h, 0x4051u);  // (element 0 low half, element 1 high half)
  o23 = prmt(l, h, 0x6273u);
}

// One 32-bit word of packed codes (8 elements, one byte per element pair) -> 4 bf16x2 words.
__device__ __forceinline__ void decode8(uint32_t w, const BlockLut &t, uint32_t (&o)[4]) {
  const uint32_t s7 = w & 0x77777777u;                              // code & 7 per nibble
  const uint32_t sm = ((w >> 1) & 0x44444444u) | 0x32103210u;      // byte j from table a or b
  decode4(s7, sm, t, o[0], o[1]);
  decode4(s7 >> 16, sm >> 16, t, o[2], o[3]);
}

// Same result; the three right shifts are done as high-half multiplies by the
// run-time constants k16 = 2^16 and k1 = 2^31, which issue on the FMA pipe and
// leave the integer/permute (ALU) pipe — the dequantiser's bottleneck — to the
// byte permutes.
__device__ __forceinline__ void decode8(uint32_t w, const BlockLut &t, uint32_t (&o)[4], uint32_t k16,
                                        uint32_t k1) {
  const uint32_t s7 = w & 0x77777777u;
  const uint32_t sm = (__umulhi(w, k1) & 0x44444444u) | 0x32103210u;
  decode4(s7, sm, t, o[0], o[1]);
  decode4(__umulhi(s7, k16), __umulhi(sm, k16), t, o[2], o[3]);
}

}  // namespace qlora
