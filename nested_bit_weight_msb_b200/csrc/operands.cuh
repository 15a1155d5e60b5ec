// Register-level construction of fp16 MMA operands from MATQ-PL1 plane words, shared by the
// decode (mma.sync) and prefill (tcgen05) paths.
//
// A lane's words of one (row tile, chunk) hold 128 weights.  For block W (inputs 32W..32W+31)
// the builder returns the A-operand registers of the two 16x16 MMA tiles of that block,
// A[j][rho] = register rho of tile j in the m16n8k16 A-fragment order.  Every fp16 half is
// 1024 + sigma * v exactly, where v is the prefix p (r <= 4) or p * 2^(8-r) (r = 6, 8) and
// sigma is a power of two fixed by the register:
//   r = 2:    sigma = 1, 4, 16, 64 for rho = 0, 1, 2, 3
//   r = 3, 4: sigma = 1, 1, 16, 16
//   r = 6, 8: sigma = 1
// (a mask-and-or against the fp16 bit pattern of 1024 places the field in the mantissa).
#pragma once
#include "common.cuh"

namespace matq {

constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves

// Plane words of one (row tile, chunk) for one lane.
struct LaneWords {
  uint32_t p0[8], p1[4], p2[4], p3[8], p4[8];
};

template <int R>
__device__ __forceinline__ void load_lane_words(const uint8_t* __restrict__ planes, const PlaneGeom& g, size_t t,
                                                int lane, LaneWords& L) {
  {
    const uint8_t* b = planes + g.off[0] + t * 1024 + lane * 16;
    uint4 a = ldg_stream(b), c = ldg_stream(b + 512);
    L.p0[0] = a.x; L.p0[1] = a.y; L.p0[2] = a.z; L.p0[3] = a.w;
    L.p0[4] = c.x; L.p0[5] = c.y; L.p0[6] = c.z; L.p0[7] = c.w;
  }
  if constexpr (R >= 3) {
    uint4 a = ldg_stream(planes + g.off[1] + t * 512 + lane * 16);
    L.p1[0] = a.x; L.p1[1] = a.y; L.p1[2] = a.z; L.p1[3] = a.w;
  }
  if constexpr (R >= 4) {
    uint4 a = ldg_stream(planes + g.off[2] + t * 512 + lane * 16);
    L.p2[0] = a.x; L.p2[1] = a.y; L.p2[2] = a.z; L.p2[3] = a.w;
  }
  if constexpr (R >= 6) {
    const uint8_t* b = planes + g.off[3] + t * 1024 + lane * 16;
    uint4 a = ldg_stream(b), c = ldg_stream(b + 512);
    L.p3[0] = a.x; L.p3[1] = a.y; L.p3[2] = a.z; L.p3[3] = a.w;
    L.p3[4] = c.x; L.p3[5] = c.y; L.p3[6] = c.z; L.p3[7] = c.w;
  }
  if constexpr (R >= 8) {
    const uint8_t* b = planes + g.off[4] + t * 1024 + lane * 16;
    uint4 a = ldg_stream(b), c = ldg_stream(b + 512);
    L.p4[0] = a.x; L.p4[1] = a.y; L.p4[2] = a.z; L.p4[3] = a.w;
    L.p4[4] = c.x; L.p4[5] = c.y; L.p4[6] = c.z; L.p4[7] = c.w;
  }
}

// Build the A-operand registers of the two 16x16 MMA tiles of block W (inputs 32W..32W+31):
// A[j][rho] is register rho of tile j.  Values are 1024 + sigma * p (fp16, exact).
template <int R, int W>
__device__ __forceinline__ void build_operands(const LaneWords& L, uint32_t (&A)[2][4]) {
  constexpr int a = W & 1;
  if constexpr (R == 2) {
    // fields rho (+8 in the high half) sit at bits 2*rho: sigma = 4^rho
    uint32_t x = L.p0[W];
    A[0][0] = and_or(x, 0x00030003u, kMagic);
    A[0][1] = and_or(x, 0x000C000Cu, kMagic);
    A[0][2] = and_or(x, 0x00300030u, kMagic);
    A[0][3] = and_or(x, 0x00C000C0u, kMagic);
    x >>= 8;
    A[1][0] = and_or(x, 0x00030003u, kMagic);
    A[1][1] = and_or(x, 0x000C000Cu, kMagic);
    A[1][2] = and_or(x, 0x00300030u, kMagic);
    A[1][3] = and_or(x, 0x00C000C0u, kMagic);
  } else if constexpr (R == 3 || R == 4) {
    // nibble form: nibble n of word C_c holds field 2n + c; sigma = 1 (nibbles 0, 2) or 16 (1, 3)
    constexpr uint32_t kField = (R == 3) ? 0x00070007u : 0x000F000Fu;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t C;
      const uint32_t w0 = L.p0[W];
      const uint32_t w1 = L.p1[W >> 1];
      if constexpr (R == 3) {
        const uint32_t s0 = (c == 0) ? (w0 << 1) : (w0 >> 1);
        const uint32_t s1 = w1 >> (2 * a + c);
        C = bitsel(s0, s1, 0x66666666u);
      } else {
        const uint32_t w2 = L.p2[W >> 1];
        const uint32_t s0 = (c == 0) ? (w0 << 2) : w0;
        const int sh1 = 1 - 2 * a - c;
        const uint32_t s1 = sh1 >= 0 ? (w1 << sh1) : (w1 >> (-sh1));
        const uint32_t s2 = w2 >> (2 * a + c);
        C = bitsel(bitsel(s0, s1, 0xCCCCCCCCu), s2, 0xEEEEEEEEu);
      }
      A[0][c] = and_or(C, kField, kMagic);
      A[0][2 + c] = and_or(C, kField << 4, kMagic);
      C >>= 8;
      A[1][c] = and_or(C, kField, kMagic);
      A[1][2 + c] = and_or(C, kField << 4, kMagic);
    }
  } else {
    // byte form: byte k of word C_c holds field 4k + c as the code with its low 8-r bits
    // cleared; prmt pairs bytes (0,2) and (1,3) with the 0x64 exponent byte.
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int o1 = 4 * (c >> 1) + 2 * a + (c & 1);  // bit of field (4k+c) in 1-bit words, minus 8k
      const uint32_t s0 = L.p0[W] << (6 - 2 * c);
      const int sh1 = 5 - o1, sh2 = 4 - o1;
      const uint32_t w1 = L.p1[W >> 1], w2 = L.p2[W >> 1];
      const uint32_t s1 = sh1 >= 0 ? (w1 << sh1) : (w1 >> (-sh1));
      const uint32_t s2 = sh2 >= 0 ? (w2 << sh2) : (w2 >> (-sh2));
      const int sh3 = 2 - 2 * c;
      const uint32_t s3 = sh3 >= 0 ? (L.p3[W] << sh3) : (L.p3[W] >> (-sh3));
      uint32_t C = bitsel(s0, s1, 0xC0C0C0C0u);
      C = bitsel(C, s2, 0xE0E0E0E0u);
      C = bitsel(C, s3, 0xF0F0F0F0u);
      if constexpr (R == 8) {
        const uint32_t s4 = L.p4[W] >> (2 * c);
        C = bitsel(C, s4, 0xFCFCFCFCu);
      } else {
        C &= 0xFCFCFCFCu;
      }
      A[0][c] = prmt(C, 0x64646464u, 0x4240u);
      A[1][c] = prmt(C, 0x64646464u, 0x4341u);
    }
  }
}

// ---- bf16 operands (decode path) ------------------------------------------------------------
// Every bf16 half is 128 + alpha * v exactly: a mask-and-or against the bf16 bit pattern of 128
// (exponent 7, seven mantissa bits of step 1) places a field of at most 7 bits in the mantissa.
// alpha depends only on the register's row half h = rho & 1, never on its input half, so the
// activations enter the B operand unscaled (raw bf16).  Fields wider than 4 bits never occur:
// widths 6 and 8 are served as a high part (code bits 7..4) plus a low part (bits 3..2 or 3..0),
// one MMA each.
//
// Plane words of one lane for half a chunk (blocks 4*hc .. 4*hc + 3, 128 inputs): 2-bit planes
// one word per block, 1-bit planes one word per block pair.
struct HalfWords {
  uint32_t p0[4], p1[2], p2[2], p3[4], p4[4];
};

constexpr uint32_t kMagicBf16 = 0x43004300u;  // bf16 128.0 in both halves

// Kinds of operand a width's MMAs take (decode path):
//   kOpP0    2-bit value from plane 0 (bits 7..6): width 2, alpha_h = 4^h
//   kOpNib3  3-bit value from planes 0, 1 (bits 7..5): width 3, alpha = 1
//   kOpNib4  4-bit value from planes 0, 1, 2 (bits 7..4): width 4 and the high part of 6, 8
//   kOpP3    2-bit value from plane 3 (bits 3..2): low part of width 6, alpha_h = 4^h
//   kOpNibLo 4-bit value from planes 3, 4 (bits 3..0): low part of width 8, alpha = 1
enum { kOpP0 = 0, kOpNib3 = 1, kOpNib4 = 2, kOpP3 = 3, kOpNibLo = 4 };

// alpha of row half h for an operand kind
__host__ __device__ constexpr int op_alpha(int kind, int h) {
  return (kind == kOpP0 || kind == kOpP3) ? (h ? 4 : 1) : 1;
}

// 2-bit plane word x of one block: field f at bits [2f, 2f + 2); register (j, h, kh) has its low
// half's field at bit 8j + 2h + 4kh and its high half's 16 bits above.
__device__ __forceinline__ void bf16_from_2bit(uint32_t x, uint32_t (&A)[2][4]) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
      const uint32_t s = x >> (8 * j + 4 * kh);
      A[j][2 * kh] = and_or(s, 0x00030003u, kMagicBf16);
      A[j][2 * kh + 1] = and_or(s, 0x000C000Cu, kMagicBf16);
    }
}
// Nibble words C_h (h = 0, 1): nibble n of C_h holds field 2n + h, so register (j, h, kh) has its
// low half at bit 8j + 4kh of C_h and its high half 16 bits above.
template <uint32_t kField>
__device__ __forceinline__ void bf16_from_nibbles(const uint32_t (&C)[2], uint32_t (&A)[2][4]) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) A[j][h + 2 * kh] = and_or(C[h] >> (8 * j + 4 * kh), kField, kMagicBf16);
}

// Operands of block 4*hc + WB (WB in 0..3) of the given kind, from the half-chunk's words.
template <int KIND, int WB>
__device__ __forceinline__ void build_bf16(const HalfWords& H, uint32_t (&A)[2][4]) {
  constexpr int a = WB & 1;  // which block of its 1-bit word
  if constexpr (KIND == kOpP0) {
    bf16_from_2bit(H.p0[WB], A);
  } else if constexpr (KIND == kOpP3) {
    bf16_from_2bit(H.p3[WB], A);
  } else if constexpr (KIND == kOpNib3 || KIND == kOpNib4) {
    uint32_t C[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint32_t w0 = H.p0[WB];
      const uint32_t w1 = H.p1[WB >> 1];
      if constexpr (KIND == kOpNib3) {
        // bits 2..1 of a nibble from plane 0, bit 0 from plane 1
        const uint32_t s0 = (c == 0) ? (w0 << 1) : (w0 >> 1);
        const uint32_t s1 = w1 >> (2 * a + c);
        C[c] = bitsel(s0, s1, 0x66666666u);
      } else {
        // bits 3..2 from plane 0, bit 1 from plane 1, bit 0 from plane 2
        const uint32_t w2 = H.p2[WB >> 1];
        const uint32_t s0 = (c == 0) ? (w0 << 2) : w0;
        const int sh1 = 1 - 2 * a - c;
        const uint32_t s1 = sh1 >= 0 ? (w1 << sh1) : (w1 >> (-sh1));
        const uint32_t s2 = w2 >> (2 * a + c);
        C[c] = bitsel(bitsel(s0, s1, 0xCCCCCCCCu), s2, 0xEEEEEEEEu);
      }
    }
    bf16_from_nibbles<(KIND == kOpNib3) ? 0x00070007u : 0x000F000Fu>(C, A);
  } else {
    // bits 3..2 from plane 3, bits 1..0 from plane 4 (both 2-bit planes, field f at bit 2f)
    uint32_t C[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) C[c] = bitsel(H.p3[WB] << (2 - 2 * c), H.p4[WB] >> (2 * c), 0xCCCCCCCCu);
    bf16_from_nibbles<0x000F000Fu>(C, A);
  }
}

// Operands of block W0 + wb (wb a runtime value in 0..3, resolved by an unrolled switch).
template <int R, int W0>
__device__ __forceinline__ void build_slice_operands(const LaneWords& L, int wb, uint32_t (&A)[2][4]) {
  switch (wb) {
    case 0: build_operands<R, W0>(L, A); break;
    case 1: if constexpr (W0 + 1 < 8) build_operands<R, W0 + 1>(L, A); break;
    case 2: if constexpr (W0 + 2 < 8) build_operands<R, W0 + 2>(L, A); break;
    default: if constexpr (W0 + 3 < 8) build_operands<R, W0 + 3>(L, A); break;
  }
}

}  // namespace matq
