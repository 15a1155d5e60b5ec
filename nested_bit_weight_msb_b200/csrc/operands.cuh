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
