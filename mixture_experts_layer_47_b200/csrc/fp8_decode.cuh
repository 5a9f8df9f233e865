// fp8_decode.cuh -- E4M3 weight codes with a power-of-two block scale, decoded to bf16.
//
// Written into bits 4-10 of a bf16 (exponent field bits 7-10, mantissa bits 4-6) with its
// sign in bit 15, a code's bits read as a bf16 equal the code's value times 2^-120 -- for
// normal codes (exponent e >= 1: 2^(e-127) (1 + m/8) against 2^(e-7) (1 + m/8)), for
// subnormal ones (bf16 subnormal 2^-126 m/8 against 2^-6 m/8) and for zero.  One bf16
// multiply by 2^(120 + s - 127) then gives code * 2^(s - 127) exactly (a product with at
// most 4 significant bits) for scale bytes s <= 134, where that factor is a finite bf16,
// and results at or above bf16's smallest subnormal.  The integer and bf16 pipes do the
// work; the conversion pipe is not used.
#pragma once
#include <cstdint>

namespace moe {

// PRMT selectors placing code bytes (0,1) or (2,3) of a word into bits 8-15 and 24-31 of
// the result (the other bytes taken from the zero operand).
constexpr uint32_t kSel01 = 0x1404u;
constexpr uint32_t kSel23 = 0x3424u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(a), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Two codes (in bits 8-15 and 24-31 of x8) to a bf16 pair times mult2.
__device__ __forceinline__ uint32_t decode_pair(uint32_t x8, uint32_t mult2) {
  const uint32_t mag = (x8 >> 4) & 0x07F007F0u;       // magnitude bits -> bits 4-10, 20-26
  const uint32_t v = mag | (x8 & 0x80008000u);        // sign bits stay at 15 and 31
  return bf16x2_mul(v, mult2);
}

// Four codes (one word, code i in byte i) to the bf16 pairs (code 0, code 1) and (code 2,
// code 3) times mult2, with the bits of decode_pair built a word at a time: a byte plane L
// of the pairs' low bytes (magnitude bits 0-3 at bits 4-7) and H of their high bytes (sign
// at bit 7, magnitude bits 4-6 at bits 0-2), then one PRMT per pair interleaves them.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t mult2, uint32_t& p01,
                                            uint32_t& p23) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;
  const uint32_t hi = ((w >> 4) & 0x07070707u) | (w & 0x80808080u);
  uint32_t a, b;
  asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(a) : "r"(lo), "r"(hi));
  asm("prmt.b32 %0, %1, %2, 0x7362;" : "=r"(b) : "r"(lo), "r"(hi));
  p01 = bf16x2_mul(a, mult2);
  p23 = bf16x2_mul(b, mult2);
}

// bf16 pair (2^(s - 7), 2^(s - 7)) for scale byte s.
__device__ __forceinline__ uint32_t scale_pair(uint32_t s) {
  const uint32_t e = (s + 120u) << 7;
  return e | (e << 16);
}

}  // namespace moe
