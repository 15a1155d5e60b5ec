// Shared definitions of libmatq's CUDA sources: the MATQ-PL1 plane layout (documented
// in include/matq.h) and small inline-PTX helpers for sm_100a.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace matq {

// ---- plane layout ---------------------------------------------------------------------
// Code bits per plane, most significant plane first: {7:6}, {5}, {4}, {3:2}, {1:0}.
constexpr int kPlanes = 5;
__host__ __device__ constexpr int plane_bits(int p) { return (p == 1 || p == 2) ? 1 : 2; }
// Lowest code bit held by each plane.
__host__ __device__ constexpr int plane_lsb(int p) {
  return p == 0 ? 6 : p == 1 ? 5 : p == 2 ? 4 : p == 3 ? 2 : 0;
}
// Planes read by width r (r in {2,3,4,6,8}); 0 for any other r.
__host__ __device__ constexpr int planes_for_width(int r) {
  return r == 2 ? 1 : r == 3 ? 2 : r == 4 ? 3 : r == 6 ? 4 : r == 8 ? 5 : 0;
}
__host__ __device__ constexpr bool valid_width(int r) { return planes_for_width(r) != 0; }

constexpr int kTileRows = 16;     // rows per row tile
constexpr int kChunk = 256;       // inputs per K-chunk
constexpr int kTileBytesPerBit = 512;  // bytes of one (row tile, chunk) per plane bit

struct PlaneGeom {
  int N, K, RT, KC;
  // byte offset of each plane from the start of the pack
  unsigned long long off[kPlanes];
};

__host__ __device__ inline unsigned long long plane_bytes(int RT, int KC, int p) {
  return (unsigned long long)RT * KC * plane_bits(p) * kTileBytesPerBit;
}

inline PlaneGeom make_geom(int N, int K) {
  PlaneGeom g;
  g.N = N;
  g.K = K;
  g.RT = (N + kTileRows - 1) / kTileRows;
  g.KC = K / kChunk;
  unsigned long long o = 0;
  for (int p = 0; p < kPlanes; ++p) {
    g.off[p] = o;
    o += plane_bytes(g.RT, g.KC, p);
  }
  return g;
}

// Field (block w, f) of lane (gid, tg) -> (row within tile, k within chunk).
__host__ __device__ inline void field_coords(int gid, int tg, int w, int f, int& row, int& k) {
  const int u = f & 7, hi = f >> 3, j = u >> 2, rho = u & 3;
  row = gid + 8 * (rho & 1);
  k = 32 * w + 16 * j + 2 * tg + 8 * (rho >> 1) + hi;
}
// Bit position of field f of block 2v+a inside lane word v of a 1-bit plane.
__host__ __device__ inline int onebit_pos(int a, int f) { return 4 * (f >> 1) + 2 * a + (f & 1); }

// ---- PTX helpers ------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// d = (a & b) | c (LOP3 truth table (0xF0 & 0xCC) | 0xAA = 0xEA).
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// d = (a & m) | (b & ~m), a bit select.  With the LOP3 operand codes a=0xF0, b=0xCC,
// c=m=0xAA the truth table is (0xAA & 0xF0) | (0x55 & 0xCC) = 0xE4.
__device__ __forceinline__ uint32_t bitsel(uint32_t a, uint32_t b, uint32_t m) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// Shift left by a signed compile-time amount (negative = logical right).
template <int S>
__device__ __forceinline__ uint32_t shl(uint32_t x) {
  if constexpr (S >= 0) return x << S; else return x >> (-S);
}

// mma.sync m16n8k16, fp16 x fp16 -> fp32, D = A*B + C.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

}  // namespace matq
