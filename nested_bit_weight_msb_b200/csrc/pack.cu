// One-time repack of 8-bit parent codes into the MATQ-PL1 true-prefix plane layout, and
// the inverse (prefix extraction) used for verification and export.
//
// The split of the code into most-significant-first bit planes, so that a width-r model
// reads exactly r bits per weight, follows "MatGPTQ: Efficient and Accurate Inference over
// Nested Quantized Models" §4 (bit-plane buffers {1-2, 3, 4, 5-6, 7-8} from the MSB, weights
// permuted offline into the tensor-core operand order).  The order inside each plane is
// this library's own and is documented in include/matq.h.
//
// Both kernels are HBM-bound streaming kernels: one warp per (16-row tile, 256-input chunk);
// the code tile goes through shared memory so that global reads and writes are coalesced.
#include "common.cuh"
#include "internal.h"

namespace matq {

constexpr int kPackWarps = 4;
constexpr int kPitch = kChunk + 16;  // padded smem row pitch: rows land 4 banks apart

// Load one 16 x 256 code tile (rows >= N as zeros) into smem with 16-byte loads.
__device__ __forceinline__ void load_code_tile(const uint8_t* __restrict__ codes, int N, int K, int rt,
                                               int kc, uint8_t* tile, int lane) {
  // 16 rows x 16 vectors of 16 bytes = 256 vectors; 8 per lane
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int v = lane + 32 * i;
    const int row = v >> 4, col = (v & 15) * 16;
    const int grow = rt * kTileRows + row;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (grow < N) val = *reinterpret_cast<const uint4*>(codes + (size_t)grow * K + (size_t)kc * kChunk + col);
    *reinterpret_cast<uint4*>(tile + row * kPitch + col) = val;
  }
}

__global__ void __launch_bounds__(32 * kPackWarps)
pack_kernel(const uint8_t* __restrict__ codes, PlaneGeom g, int nplanes, uint8_t* __restrict__ planes) {
  __shared__ __align__(16) uint8_t smem[kPackWarps][kTileRows * kPitch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tile_id = (long long)blockIdx.x * kPackWarps + warp;
  if (tile_id >= (long long)g.RT * g.KC) return;
  const int rt = (int)(tile_id / g.KC), kc = (int)(tile_id % g.KC);
  uint8_t* tile = smem[warp];
  load_code_tile(codes, g.N, g.K, rt, kc, tile, lane);
  __syncwarp();

  const int gid = lane >> 2, tg = lane & 3;
  // 2-bit planes: 8 words per lane; 1-bit planes: 4 words per lane.
  // The fields f0, f0 + 4, f0 + 8, f0 + 12 of a block (f0 = 0..3) lie 8 bits apart in every
  // plane word (bits 2f of 2-bit words, 4*(f >> 1) + 2a + (f & 1) of 1-bit words), and their
  // codes are bytes k0, k0 + 16, k0 + 1, k0 + 17 of one row (k0 = 32w + 2tg + 8*(f0 >> 1),
  // row gid + 8*(f0 & 1)).  One byte permute gathers the four codes into X; each plane then
  // takes a shift, a mask and an or for four weights at once.
  uint32_t w0[8] = {0}, w3[8] = {0}, w4[8] = {0}, w1[4] = {0}, w2[4] = {0};
#pragma unroll
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int f0 = 0; f0 < 4; ++f0) {
      const uint8_t* rp = tile + (gid + 8 * (f0 & 1)) * kPitch + 32 * w + 2 * tg + 8 * (f0 >> 1);
      const uint32_t p0 = *reinterpret_cast<const uint16_t*>(rp);
      const uint32_t p1 = *reinterpret_cast<const uint16_t*>(rp + 16);
      const uint32_t X = __byte_perm(p0, p1, 0x5140);  // bytes: k0, k0 + 16, k0 + 1, k0 + 17
      const int s2 = 2 * f0;
      w0[w] |= ((X >> 6) & 0x03030303u) << s2;
      w3[w] |= ((X >> 2) & 0x03030303u) << s2;
      w4[w] |= (X & 0x03030303u) << s2;
      const int s1 = 4 * (f0 >> 1) + 2 * (w & 1) + (f0 & 1);
      w1[w >> 1] |= ((X >> 5) & 0x01010101u) << s1;
      w2[w >> 1] |= ((X >> 4) & 0x01010101u) << s1;
    }
  }
  const size_t t = (size_t)rt * g.KC + kc;
  // plane 0 (2 bits): two 512-byte halves, 16 bytes per lane in each
  {
    uint8_t* base = planes + g.off[0] + t * 1024;
    *reinterpret_cast<uint4*>(base + lane * 16) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(base + 512 + lane * 16) = make_uint4(w0[4], w0[5], w0[6], w0[7]);
  }
  if (nplanes > 1) {
    uint8_t* base = planes + g.off[1] + t * 512;
    *reinterpret_cast<uint4*>(base + lane * 16) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  }
  if (nplanes > 2) {
    uint8_t* base = planes + g.off[2] + t * 512;
    *reinterpret_cast<uint4*>(base + lane * 16) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  }
  if (nplanes > 3) {
    uint8_t* base = planes + g.off[3] + t * 1024;
    *reinterpret_cast<uint4*>(base + lane * 16) = make_uint4(w3[0], w3[1], w3[2], w3[3]);
    *reinterpret_cast<uint4*>(base + 512 + lane * 16) = make_uint4(w3[4], w3[5], w3[6], w3[7]);
  }
  if (nplanes > 4) {
    uint8_t* base = planes + g.off[4] + t * 1024;
    *reinterpret_cast<uint4*>(base + lane * 16) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    *reinterpret_cast<uint4*>(base + 512 + lane * 16) = make_uint4(w4[4], w4[5], w4[6], w4[7]);
  }
}

// Inverse: read the planes of width r and write p = q >> (8 - r) as bytes.
__global__ void __launch_bounds__(32 * kPackWarps)
slice_kernel(const uint8_t* __restrict__ planes, PlaneGeom g, int r, uint8_t* __restrict__ out) {
  __shared__ __align__(16) uint8_t smem[kPackWarps][kTileRows * kPitch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tile_id = (long long)blockIdx.x * kPackWarps + warp;
  if (tile_id >= (long long)g.RT * g.KC) return;
  const int rt = (int)(tile_id / g.KC), kc = (int)(tile_id % g.KC);
  const int np = planes_for_width(r);
  const size_t t = (size_t)rt * g.KC + kc;
  uint32_t w0[8], w3[8] = {0}, w4[8] = {0}, w1[4] = {0}, w2[4] = {0};
  {
    const uint8_t* base = planes + g.off[0] + t * 1024;
    uint4 a = *reinterpret_cast<const uint4*>(base + lane * 16);
    uint4 b = *reinterpret_cast<const uint4*>(base + 512 + lane * 16);
    w0[0] = a.x; w0[1] = a.y; w0[2] = a.z; w0[3] = a.w; w0[4] = b.x; w0[5] = b.y; w0[6] = b.z; w0[7] = b.w;
  }
  if (np > 1) {
    uint4 a = *reinterpret_cast<const uint4*>(planes + g.off[1] + t * 512 + lane * 16);
    w1[0] = a.x; w1[1] = a.y; w1[2] = a.z; w1[3] = a.w;
  }
  if (np > 2) {
    uint4 a = *reinterpret_cast<const uint4*>(planes + g.off[2] + t * 512 + lane * 16);
    w2[0] = a.x; w2[1] = a.y; w2[2] = a.z; w2[3] = a.w;
  }
  if (np > 3) {
    const uint8_t* base = planes + g.off[3] + t * 1024;
    uint4 a = *reinterpret_cast<const uint4*>(base + lane * 16);
    uint4 b = *reinterpret_cast<const uint4*>(base + 512 + lane * 16);
    w3[0] = a.x; w3[1] = a.y; w3[2] = a.z; w3[3] = a.w; w3[4] = b.x; w3[5] = b.y; w3[6] = b.z; w3[7] = b.w;
  }
  if (np > 4) {
    const uint8_t* base = planes + g.off[4] + t * 1024;
    uint4 a = *reinterpret_cast<const uint4*>(base + lane * 16);
    uint4 b = *reinterpret_cast<const uint4*>(base + 512 + lane * 16);
    w4[0] = a.x; w4[1] = a.y; w4[2] = a.z; w4[3] = a.w; w4[4] = b.x; w4[5] = b.y; w4[6] = b.z; w4[7] = b.w;
  }
  uint8_t* tile = smem[warp];
  const int gid = lane >> 2, tg = lane & 3;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int f = 0; f < 16; ++f) {
      int row, k;
      field_coords(gid, tg, w, f, row, k);
      const int pos = onebit_pos(w & 1, f);
      uint32_t q = ((w0[w] >> (2 * f)) & 3u) << 6;
      q |= ((w1[w >> 1] >> pos) & 1u) << 5;
      q |= ((w2[w >> 1] >> pos) & 1u) << 4;
      q |= ((w3[w] >> (2 * f)) & 3u) << 2;
      q |= (w4[w] >> (2 * f)) & 3u;
      tile[row * kPitch + k] = (uint8_t)(q >> (8 - r));
    }
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int v = lane + 32 * i;
    const int row = v >> 4, col = (v & 15) * 16;
    const int grow = rt * kTileRows + row;
    if (grow < g.N)
      *reinterpret_cast<uint4*>(out + (size_t)grow * g.K + (size_t)kc * kChunk + col) =
          *reinterpret_cast<const uint4*>(tile + row * kPitch + col);
  }
}

cudaError_t launch_pack(const uint8_t* codes, const PlaneGeom& g, int r_keep, void* planes, cudaStream_t s) {
  const long long tiles = (long long)g.RT * g.KC;
  const unsigned blocks = (unsigned)((tiles + kPackWarps - 1) / kPackWarps);
  pack_kernel<<<blocks, 32 * kPackWarps, 0, s>>>(codes, g, planes_for_width(r_keep), (uint8_t*)planes);
  return cudaGetLastError();
}

cudaError_t launch_slice(const void* planes, const PlaneGeom& g, int r, uint8_t* out, cudaStream_t s) {
  const long long tiles = (long long)g.RT * g.KC;
  const unsigned blocks = (unsigned)((tiles + kPackWarps - 1) / kPackWarps);
  slice_kernel<<<blocks, 32 * kPackWarps, 0, s>>>((const uint8_t*)planes, g, r, out);
  return cudaGetLastError();
}

}  // namespace matq
