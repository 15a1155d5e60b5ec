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

// Build the plane words of one 16 x 256 code tile held in smem and store the first `nplanes`
// planes of tile t.
__device__ __forceinline__ void store_tile_planes(const uint8_t* tile, const PlaneGeom& g, size_t t, int nplanes,
                                                  uint8_t* __restrict__ planes, int lane) {
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

// Read the first `np` planes of tile t and write each weight's code (bits of planes not read
// are zero), passed through op(q), into the smem tile.
template <typename Op>
__device__ __forceinline__ void load_tile_codes(const uint8_t* __restrict__ planes, const PlaneGeom& g, size_t t,
                                                int np, uint8_t* tile, int lane, Op op) {
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
      tile[row * kPitch + k] = (uint8_t)op(q);
    }
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
  store_tile_planes(tile, g, (size_t)rt * g.KC + kc, nplanes, planes, lane);
}

// Inverse: read the planes of width r and write p = q >> (8 - r) as bytes.
__global__ void __launch_bounds__(32 * kPackWarps)
slice_kernel(const uint8_t* __restrict__ planes, PlaneGeom g, int r, uint8_t* __restrict__ out) {
  __shared__ __align__(16) uint8_t smem[kPackWarps][kTileRows * kPitch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tile_id = (long long)blockIdx.x * kPackWarps + warp;
  if (tile_id >= (long long)g.RT * g.KC) return;
  const int rt = (int)(tile_id / g.KC), kc = (int)(tile_id % g.KC);
  uint8_t* tile = smem[warp];
  const int sh = 8 - r;
  load_tile_codes(planes, g, (size_t)rt * g.KC + kc, planes_for_width(r), tile, lane,
                  [sh](uint32_t q) { return q >> sh; });
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

// ---- rounded slicing (strict and Extra-Precision MatQuant) ----------------------------------
// "Matryoshka Quantization | Summary" §3.2 slices a c-bit code by rounding,
// L = floor(q / 2^(8-r) + 1/2), which needs bit 7 - r besides the r-bit prefix; strict MatQuant
// clamps L to 2^r - 1, Extra-Precision MatQuant (§7 Errata) keeps L = 2^r for the weights whose
// codes round up past the last r-bit level.  One warp per (16-row tile, 256-input chunk):
//   phase 0: the clamped level, placed where a code's r-bit prefix sits (L << (8 - r)), is
//            repacked as width-r planes; per (row, chunk) the number of weights with L = 2^r
//            goes to cnt[row * KC + kc];
//   phase 1: with cnt replaced by its exclusive prefix sum, the inputs k of those weights are
//            written to cols, ascending within each row.
// In the smem tile bit 0 of a byte flags L = 2^r (the clamped level leaves the low 8 - r >= 2
// bits of the byte free; width r's planes never read bit 0).
__device__ __forceinline__ uint32_t rounded_level_byte(uint32_t q, int r) {
  if (r == 8) return q;
  const uint32_t L = (q + (1u << (7 - r))) >> (8 - r);  // 0 .. 2^r
  const uint32_t top = 1u << r;
  return L == top ? (((top - 1) << (8 - r)) | 1u) : (L << (8 - r));
}

__global__ void __launch_bounds__(32 * kPackWarps)
round_extract_kernel(const uint8_t* __restrict__ planes, PlaneGeom g, int r, int np_in, int phase,
                     uint8_t* __restrict__ levels, int* __restrict__ cnt, uint16_t* __restrict__ cols,
                     long long cols_cap) {
  __shared__ __align__(16) uint8_t smem[kPackWarps][kTileRows * kPitch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long tile_id = (long long)blockIdx.x * kPackWarps + warp;
  if (tile_id >= (long long)g.RT * g.KC) return;
  const int rt = (int)(tile_id / g.KC), kc = (int)(tile_id % g.KC);
  uint8_t* tile = smem[warp];
  const size_t t = (size_t)rt * g.KC + kc;
  load_tile_codes(planes, g, t, np_in, tile, lane, [r](uint32_t q) { return rounded_level_byte(q, r); });
  __syncwarp();
  if (phase == 0) store_tile_planes(tile, g, t, planes_for_width(r), levels, lane);
  // lane pair (2i, 2i + 1) takes row i of the tile, inputs 0..127 and 128..255 of the chunk
  const int row = lane >> 1, half = lane & 1;
  const int grow = rt * kTileRows + row;
  const uint8_t* src = tile + row * kPitch + half * 128;
  uint32_t flags[4] = {0u, 0u, 0u, 0u};  // bit j of flags[j >> 5]: input half * 128 + j flagged
#pragma unroll
  for (int v = 0; v < 8 && r < 8; ++v) {  // width 8 rounds nothing: its bytes are the codes
    const uint4 b = *reinterpret_cast<const uint4*>(src + v * 16);
    const uint32_t wds[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t m = wds[i] & 0x01010101u;  // bit 0 of each byte
      const uint32_t nib = (m & 1u) | ((m >> 7) & 2u) | ((m >> 14) & 4u) | ((m >> 21) & 8u);
      const int j = v * 16 + i * 4;
      flags[j >> 5] |= nib << (j & 31);
    }
  }
  const int n_mine = __popc(flags[0]) + __popc(flags[1]) + __popc(flags[2]) + __popc(flags[3]);
  const int n_row = n_mine + __shfl_xor_sync(0xffffffffu, n_mine, 1);
  const int n_first = __shfl_sync(0xffffffffu, n_mine, lane & ~1);  // the row's inputs 0..127
  if (grow >= g.N) return;
  const size_t ci = (size_t)grow * g.KC + kc;
  if (phase == 0) {
    if (half == 0) cnt[ci] = n_row;
    return;
  }
  long long off = (long long)cnt[ci] + (half ? n_first : 0);
  const int kbase = kc * kChunk + half * 128;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t f = flags[w];
    while (f) {
      const int j = __ffs(f) - 1;
      f &= f - 1;
      if (off < cols_cap) cols[off] = (uint16_t)(kbase + w * 32 + j);
      ++off;
    }
  }
}

// Exclusive prefix sum of cnt[0 .. n) in place (row-major (row, chunk) order), by one block;
// then row_ptr[i] = cnt[i * KC] for i < N and row_ptr[N] = the total.
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) round_scan_kernel(int* __restrict__ cnt, long long n, int KC, int N,
                                                                  int* __restrict__ row_ptr) {
  __shared__ int wsum[kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long per = (n + kScanThreads - 1) / kScanThreads;
  const long long b = (long long)tid * per;
  const long long e = b + per < n ? b + per : n;
  int sum = 0;
  for (long long i = b; i < e; ++i) sum += cnt[i];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = wsum[lane];
    int iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += u;
    }
    wsum[lane] = iv - v;
  }
  __syncthreads();
  int run = wsum[warp] + incl - sum;
  for (long long i = b; i < e; ++i) {
    const int c = cnt[i];
    cnt[i] = run;
    run += c;
  }
  __syncthreads();
  for (int i = tid; i < N; i += kScanThreads) row_ptr[i] = cnt[(long long)i * KC];
  if (tid == kScanThreads - 1) row_ptr[N] = run;
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

cudaError_t launch_round_extract(const void* planes, const PlaneGeom& g, int r, int r_in, void* levels, int* cnt,
                                 int* row_ptr, uint16_t* cols, long long cols_cap, cudaStream_t s) {
  const long long tiles = (long long)g.RT * g.KC;
  const unsigned blocks = (unsigned)((tiles + kPackWarps - 1) / kPackWarps);
  const int np_in = planes_for_width(r_in);
  round_extract_kernel<<<blocks, 32 * kPackWarps, 0, s>>>((const uint8_t*)planes, g, r, np_in, 0,
                                                          (uint8_t*)levels, cnt, nullptr, 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  round_scan_kernel<<<1, kScanThreads, 0, s>>>(cnt, (long long)g.N * g.KC, g.KC, g.N, row_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess || !cols) return e;
  round_extract_kernel<<<blocks, 32 * kPackWarps, 0, s>>>((const uint8_t*)planes, g, r, np_in, 1, nullptr, cnt,
                                                          cols, cols_cap);
  return cudaGetLastError();
}

}  // namespace matq
