// tcf4_device.cuh -- device helpers: bit-sliced XOR-Trellis decode of 32-weight blocks.
//
// The decoder ("XOR-Trellis: Hadamard-free FP4 LLM quantization" news page, bullet
// "XOR-Trellis FP4 decoder") keys each weight on a 16-bit sliding state. With the new 2-bit
// symbol entering at bits 14-15, the state of weight i holds symbols i-7..i, symbol i-7+m at bits
// 2m (low bit) and 2m+1 (high bit). Each masked parity is therefore an XOR of the low/high bit
// planes of the block delayed by a fixed number of symbols:
//
//   p0 = parity(s & 0x1089) = L<<7 ^ H<<6 ^ H<<4 ^ L<<1
//   p1 = parity(s & 0x2112) = H<<7 ^ L<<5 ^ L<<3 ^ H<<1
//   q0 = parity(s & 0x0A24) = L<<6 ^ H<<5 ^ H<<3 ^ H<<2
//   q1 = parity(s & 0x2441) = L<<7 ^ L<<4 ^ L<<2 ^ H<<1
//
// where L, H are the 32-bit planes of the block (bit i = symbol i) and "X<<d" delays by d
// symbols (bits shifted in come from the previous block of the segment, zero at its start).
// With p = p0 + 2 p1, q = q0 + 2 q1, entry e = b ^ q and P3's zero read as -0, the E2M1 code of
// palette entry P_p[e] has the bit planes
//
//   neg = ~(H ^ q1)            (entries 0 and 1 of every palette are the negative ones)
//   n0  = p0 ^ neg,  n1 = p1 ^ neg,  n2 = L ^ q0 ^ neg,  n3 = neg.
//
// So a whole 32-weight block decodes with 11 to 14 shifts and 9 three-input XORs, independent of
// any table. The identity is checked bit-exactly against the oracle by the GPU parity tests and
// over all 65,536 states by a CPU test.
#pragma once
#include <cstdint>

namespace tcf4 {

// Bit planes of the E2M1 codes of one 32-weight block: bit i of n_c is bit c of weight i's code.
struct Planes {
  uint32_t n0, n1, n2, n3;
};

// x delayed by d symbols: bit i <- bit i-d, with the top bits of px (previous block) shifted in.
template <int D>
__device__ __forceinline__ uint32_t dly(uint32_t x, uint32_t px) {
  return __funnelshift_l(px, x, D);
}

// Three-input logic op with an immediate truth table over (a, b, c) = (0xF0, 0xCC, 0xAA). The XOR
// sums below are written with it: left to the compiler, not every three-input XOR became one
// instruction (2.4 M of 31 M instructions of the gate_up GEMV). Tables used: a ^ b = 0x3C,
// ~(a ^ b) = 0xC3, a ^ b ^ c = 0x96, ~(a ^ b ^ c) = 0x69.
template <uint32_t LUT>
__device__ __forceinline__ uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
  return d;
}

// Decode one block. (L, H) are its planes; (pL, pH) the previous block's planes in the same
// segment (zero at a segment start). 14 funnel shifts and 9 three-input XORs.
__device__ __forceinline__ Planes decode_block(uint32_t L, uint32_t H, uint32_t pL, uint32_t pH) {
  const uint32_t L1 = dly<1>(L, pL), L2 = dly<2>(L, pL), L3 = dly<3>(L, pL), L4 = dly<4>(L, pL);
  const uint32_t L5 = dly<5>(L, pL), L6 = dly<6>(L, pL), L7 = dly<7>(L, pL);
  const uint32_t H1 = dly<1>(H, pH), H2 = dly<2>(H, pH), H3 = dly<3>(H, pH), H4 = dly<4>(H, pH);
  const uint32_t H5 = dly<5>(H, pH), H6 = dly<6>(H, pH), H7 = dly<7>(H, pH);
  const uint32_t neg = lop3<0x69>(H, lop3<0x96>(L7, L4, L2), H1);  // ~(H ^ q1)
  Planes r;
  r.n0 = lop3<0x96>(neg, lop3<0x96>(L7, H6, H4), L1);              // p0 ^ neg
  r.n1 = lop3<0x96>(neg, lop3<0x96>(H7, L5, L3), H1);              // p1 ^ neg
  r.n2 = lop3<0x96>(lop3<0x96>(neg, L, L6), lop3<0x3C>(H5, H3, 0u), H2);  // e0 ^ neg, e0 = L ^ q0
  r.n3 = neg;
  return r;
}

// Segment-start form (no carry from a previous block). Delays are then plain shifts, which
// distribute over XOR, so shared sums are shifted once: with F = L ^ L2, U = L ^ L6, G = H ^ H2,
//   L2 ^ L4 = F << 2,  L3 ^ L5 = F << 3,  L1 ^ L7 = U << 1,  H4 ^ H6 = G << 4,  H3 ^ H5 = G << 3,
// X = H ^ F2 ^ L7 is shared by q1 (X ^ H1) and n1 (H1 cancels), and t = U ^ (G << 3) by n2 and,
// shifted once more, n0 (U1 ^ G4 = t << 1): 10 shifts and 9 XORs instead of 14 and 10.
// decode_block0 with n3 returned inverted (n3 = ~H ^ q1, returned as H ^ q1), for the transpose
// that absorbs the inversion.
__device__ __forceinline__ Planes decode_block0_i3(uint32_t L, uint32_t H) {
  const uint32_t F = lop3<0x3C>(L, L << 2, 0u), U = lop3<0x3C>(L, L << 6, 0u), H2 = H << 2;
  const uint32_t t = lop3<0x3C>(U, lop3<0x3C>(H, H2, 0u) << 3, 0u);
  const uint32_t X = lop3<0x96>(H, F << 2, L << 7);
  const uint32_t q1h = lop3<0x3C>(X, H << 1, 0u);  // H ^ q1
  Planes r;
  r.n3 = q1h;
  r.n0 = lop3<0xC3>(q1h, t << 1, 0u);
  r.n1 = lop3<0x69>(X, F << 3, H << 7);
  r.n2 = lop3<0x69>(q1h, t, H2);
  return r;
}

__device__ __forceinline__ Planes decode_block0(uint32_t L, uint32_t H) {
  Planes r = decode_block0_i3(L, H);
  r.n3 = ~r.n3;
  return r;
}

// Exchange the bits of a selected by (M << S) with the bits of b selected by M, as two bit selects
// (two shifts and two three-input logic ops; with operands (x, y, mask), lop3 LUT 0xE4 is
// "mask ? x : y"; the masks are immediates).
template <int S, uint32_t M>
__device__ __forceinline__ void delta_swap(uint32_t &a, uint32_t &b) {
  uint32_t na, nb;
  const uint32_t a_sh = a >> S, b_sh = b << S;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(nb) : "r"(a_sh), "r"(b), "n"(M));
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(na) : "r"(b_sh), "r"(a), "n"(M << S));
  a = na;
  b = nb;
}

// The same exchange for b given inverted (bi = ~b): the selects read ~bi (LUTs 0xB1 for
// "mask ? x : ~y" and 0x4E for "mask ? ~x : y"), so the inversion costs no instruction.
template <int S, uint32_t M>
__device__ __forceinline__ void delta_swap_inv_b(uint32_t &a, uint32_t &b, uint32_t bi) {
  uint32_t na, nb;
  const uint32_t a_sh = a >> S, bi_sh = bi << S;
  asm("lop3.b32 %0, %1, %2, %3, 0xB1;" : "=r"(nb) : "r"(a_sh), "r"(bi), "n"(M));
  asm("lop3.b32 %0, %1, %2, %3, 0x4E;" : "=r"(na) : "r"(bi_sh), "r"(a), "n"(M << S));
  a = na;
  b = nb;
}

// Planes -> four nibble words in "interleaved" order: word j, nibble v holds the code of weight
// 4v + j (j = 0..3). Four delta swaps.
__device__ __forceinline__ void planes_to_nibbles_interleaved(const Planes &p, uint32_t &w0, uint32_t &w1,
                                                              uint32_t &w2, uint32_t &w3) {
  uint32_t a = p.n0, b = p.n1, c = p.n2, d = p.n3;
  delta_swap<1, 0x55555555u>(a, b);  // a: (n0,n1) of even weights; b: of odd weights
  delta_swap<1, 0x55555555u>(c, d);  // c: (n2,n3) of even weights; d: of odd weights
  delta_swap<2, 0x33333333u>(a, c);  // a: nibbles of weights 4v; c: of 4v+2
  delta_swap<2, 0x33333333u>(b, d);  // b: nibbles of weights 4v+1; d: of 4v+3
  w0 = a;
  w1 = b;
  w2 = c;
  w3 = d;
}

// The same from planes whose n3 is given inverted (n3i = ~n3, as the segment-start decoder
// produces it).
__device__ __forceinline__ void planes_to_nibbles_interleaved_i3(const Planes &p, uint32_t &w0, uint32_t &w1,
                                                                 uint32_t &w2, uint32_t &w3) {
  uint32_t a = p.n0, b = p.n1, c = p.n2, d;
  delta_swap<1, 0x55555555u>(a, b);
  delta_swap_inv_b<1, 0x55555555u>(c, d, p.n3);
  delta_swap<2, 0x33333333u>(a, c);
  delta_swap<2, 0x33333333u>(b, d);
  w0 = a;
  w1 = b;
  w2 = c;
  w3 = d;
}

// Planes -> four nibble words in natural MXFP4 order: word q holds weights 8q..8q+7, byte u of
// the block holds weight 2u (low nibble) and 2u+1 (high nibble).
__device__ __forceinline__ void planes_to_nibbles_natural(const Planes &p, uint32_t &o0, uint32_t &o1,
                                                          uint32_t &o2, uint32_t &o3) {
  uint32_t A, B, C, D;
  planes_to_nibbles_interleaved(p, A, B, C, D);
  // A: weight 4v at nibble v; B: 4v+1; C: 4v+2; D: 4v+3. Exchange A's odd nibbles with B's even
  // nibbles (and C with D): afterwards byte w of A = (8w, 8w+1), B = (8w+4, 8w+5),
  // C = (8w+2, 8w+3), D = (8w+6, 8w+7).
  delta_swap<4, 0x0F0F0F0Fu>(A, B);
  delta_swap<4, 0x0F0F0F0Fu>(C, D);
  // 4x4 byte transpose of (A, C, B, D): output word q = [A.q, C.q, B.q, D.q].
  const uint32_t u0 = __byte_perm(A, C, 0x5140), u1 = __byte_perm(A, C, 0x7362);
  const uint32_t v0 = __byte_perm(B, D, 0x5140), v1 = __byte_perm(B, D, 0x7362);
  o0 = __byte_perm(u0, v0, 0x5410);
  o1 = __byte_perm(u0, v0, 0x7632);
  o2 = __byte_perm(u1, v1, 0x5410);
  o3 = __byte_perm(u1, v1, 0x7632);
}

// UE8M0 byte -> float scale 2^(E-127) (E = 0 gives the subnormal 2^-127, E = 255 gives NaN).
__device__ __forceinline__ float ue8m0_to_float(uint32_t E) {
  return E == 0u ? __uint_as_float(0x00400000u) : (E == 255u ? __uint_as_float(0x7FC00000u)
                                                              : __uint_as_float(E << 23));
}

// E5M3 block scale -> float, exact. The XOR-Trellis news page pairs E2M1 elements with E5M3 block
// scales (its paragraph on the grouping format) and gives no encoding; read as: no sign, exponent
// bits 7..3 with bias 15, mantissa bits 2..0, exponent 0 subnormal (m * 2^-17), exponent 31 NaN.
// A normal byte b is the float with exponent field (b >> 3) + 112 and mantissa bits (b & 7) << 20.
__device__ __forceinline__ float e5m3_to_float(uint32_t b) {
  if (b >= 0xF8u) return __uint_as_float(0x7FC00000u);
  if (b < 8u) return (float)b * __uint_as_float(110u << 23);  // m * 2^-17
  return __uint_as_float((b << 20) + (112u << 23));
}

// Eight E2M1 codes (a word, byte u = codes 2u and 2u+1, low nibble first) -> four half2
// (exact: every E2M1 value is a binary16 value).
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t &h0, uint32_t &h1, uint32_t &h2,
                                                  uint32_t &h3) {
  asm("{\n\t.reg .b8 a0, a1, a2, a3;\n\t"
      "mov.b32 {a0, a1, a2, a3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, a0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, a1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, a2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, a3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}

}  // namespace tcf4
