// Prefill path (M > 16): TMA + tcgen05 GEMM over the packed r-bit planes.
//
// y = x . W_hat_r^T with W_hat = s * (q_hat - z), q_hat = p * 2^(8-r) + delta_r ("MatGPTQ:
// Efficient and Accurate Inference over Nested Quantized Models", App. A.1 and §4).  This
// path is a dense contraction, so it runs on the 5th-generation tensor cores:
//
//   * one persistent CTA per SM takes output tiles [128 weight rows x BN tokens] in turn
//     (token tiles fastest, so the CTAs on one weight-row block share its planes in L2);
//   * warp 0 (one thread) streams, with TMA, the raw planes of width r for a 128-row x
//     256-input block (only those planes: exactly r bits per weight cross HBM) and the fp16
//     activation tiles [BN tokens x 64 inputs] (128-byte swizzle, the UMMA K-major layout);
//   * warps 4..11 (one 16-row tile each) turn each 64-input slice of the raw planes into an
//     fp16 weight tile [128 x 64] in shared memory: operand registers are built from the plane
//     words exactly as on the decode path (1024 + sigma*v), the exact code difference
//     q_hat - z is formed in fp16 (exact: a half-integer below 256 in magnitude), and one fp16
//     multiply by the scale gives W_hat with a single rounding.  stmatrix writes the tiles in
//     the swizzled layout; fence.proxy.async hands them to the tensor core;
//   * warp 1 (one thread) issues tcgen05.mma (M = 128 weight rows, N = BN tokens, K = 16)
//     into one of two TMEM accumulators (tiles alternate), releasing ring slots with
//     tcgen05.commit;
//   * warps 12..15 (one TMEM lane quarter each) read a finished accumulator with tcgen05.ld
//     and store y while the next tile accumulates in the other one.
//
// fp16 (not bf16) weight tiles: with bf16 y, bf16-rounded weights exceed the 2e-3 relative
// error budget while fp16 ones stay at the output-rounding level; both formats run at the
// same tensor-core rate.  x is converted bf16 -> fp16 once per call into the workspace, each
// token row first divided by the power of two that keeps its largest value finite in fp16
// (exact); the epilogue multiplies that token's fp32 results back, so every bf16 input range is
// served (values more than 2^30 below the row's largest reach fp16's subnormal range).
//
// Every mbarrier wait is bounded (about a second of clock); on expiry the kernel records an
// error code in the workspace header, every role drains, TMEM is freed, and the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "operands.cuh"
#include "sync.cuh"

namespace matq {

constexpr int kBM = 128;        // weight rows per tile (UMMA M)
constexpr int kSubK = 64;       // inputs per A/B ring slot (one 128-byte swizzle row of fp16)
constexpr int kRawStages = 2;   // raw-plane ring (256 inputs per slot)
constexpr int kAStages = 3;     // fp16 weight-tile ring
constexpr int kBStages = 3;     // activation-tile ring
constexpr int kDeqWarps = 8;                   // dequantising (and epilogue) warps 4 .. 4 + kDeqWarps - 1
constexpr int kWarpsPerTile = kDeqWarps >= 8 ? kDeqWarps / 8 : 1;  // warps sharing a 16-row tile
constexpr int kTilesPerWarp = kDeqWarps >= 8 ? 1 : 8 / kDeqWarps;  // 16-row tiles per warp
constexpr int kEpiWarps = 4;                    // epilogue warps 4 + kDeqWarps .. + 3 (one per TMEM lane quarter)
constexpr int kThreads = 32 * (4 + kDeqWarps + kEpiWarps);
constexpr int kATileBytes = kBM * kSubK * 2;  // 16 KB

// ---- activation conversion -----------------------------------------------------------------
// One block per token row: the row's largest bf16 exponent E gives a power of two 2^e,
// e = max(0, E - 15), so that every x * 2^-e is a finite fp16 (bf16 values below 2^16 convert
// exactly; the scaling is exact).  x16 = fp16(x * 2^-e); xscale[m] = 2^e, multiplied back into
// the token's fp32 results by the epilogue.  Rows whose values all lie below 2^16 keep e = 0.
constexpr int kXprepThreads = 256;
constexpr int kXprepHeld = 8;  // 16-byte vectors a thread keeps in registers (rows of K <= 16384)
__device__ __forceinline__ uint32_t bf16x2_emax(uint32_t w) {
  return max((w >> 7) & 0xFFu, (w >> 23) & 0xFFu);
}
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 in, float down) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint4 o4;
  uint32_t* o = reinterpret_cast<uint32_t*>(&o4);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __uint_as_float(w[i] << 16) * down, b = __uint_as_float(w[i] & 0xFFFF0000u) * down;
    __half2 h = __floats2half2_rn(a, b);
    o[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  return o4;
}
__global__ void __launch_bounds__(kXprepThreads) xprep_prefill_kernel(const uint16_t* __restrict__ x, int K,
                                                                      __half* __restrict__ x16,
                                                                      float* __restrict__ xscale) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * (size_t)K);
  uint4* out = reinterpret_cast<uint4*>(x16 + m * (size_t)K);
  const int nvec = K / 8;
  const bool held = nvec <= kXprepHeld * kXprepThreads;  // the row is read once, kept in registers
  uint4 v[kXprepHeld];
  // largest exponent field of the row (bf16 bits 14..7)
  uint32_t emax = 0;
  if (held) {
#pragma unroll
    for (int u = 0; u < kXprepHeld; ++u) {
      const int i = threadIdx.x + u * kXprepThreads;
      v[u] = i < nvec ? row[i] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kXprepHeld; ++u)
      emax = max(emax, max(max(bf16x2_emax(v[u].x), bf16x2_emax(v[u].y)), max(bf16x2_emax(v[u].z), bf16x2_emax(v[u].w))));
  } else {
    for (int i = threadIdx.x; i < nvec; i += kXprepThreads) {
      const uint4 in = row[i];
      emax = max(emax, max(max(bf16x2_emax(in.x), bf16x2_emax(in.y)), max(bf16x2_emax(in.z), bf16x2_emax(in.w))));
    }
  }
  __shared__ uint32_t red[kXprepThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = emax;
  __syncthreads();
  emax = 0;
#pragma unroll
  for (int i = 0; i < kXprepThreads / 32; ++i) emax = max(emax, red[i]);
  // exponent field 127 + 15 = 142 is the largest that converts without overflow
  const int e = emax > 142u ? (int)emax - 142 : 0;
  const float down = __int_as_float((127 - e) << 23);  // 2^-e (e <= 128 for finite inputs)
  if (threadIdx.x == 0) xscale[m] = __int_as_float((127 + min(e, 127)) << 23);
  if (held) {
#pragma unroll
    for (int u = 0; u < kXprepHeld; ++u) {
      const int i = threadIdx.x + u * kXprepThreads;
      if (i < nvec) out[i] = bf16x8_to_f16x8(v[u], down);
    }
  } else {
    for (int i = threadIdx.x; i < nvec; i += kXprepThreads) out[i] = bf16x8_to_f16x8(row[i], down);
  }
}

// ---- the GEMM kernel -----------------------------------------------------------------------
struct PrefillParams {
  int M, N, K, G, RT;
  int S;        // K splits per (row block, token tile); S > 1: fp32 partial sums into `part`
  float* part;  // [S][M][N] (S > 1), summed and finished by prefill_finish_kernel
  const uint16_t* scales;
  const uint8_t* zeros;
  const float* xscale;  // per token: the power of two its activations were divided by
  float delta;          // added to every level before the zero point: delta_r, or 0 for stored levels
  // Extra-Precision MatQuant: rows' lists (CSR, inputs ascending) of the weights whose rounded
  // level is 2^r, or null.  Their fp16 tile values become s * (256 - z).
  const int* ovf_row_ptr;
  const uint16_t* ovf_cols;
  void* y;
  int y_mode;
  int* err;
};

template <int R>
__host__ __device__ constexpr int raw_stage_bytes() { return 4096 * R; }  // 8 row tiles x r bits x 512 B

template <int R, int BN>
struct PrefillSmem {
  static constexpr int kA = 0;
  static constexpr int kB = kA + kAStages * kATileBytes;
  static constexpr int kRaw = kB + kBStages * BN * 128;
  static constexpr int kBar = kRaw + kRawStages * raw_stage_bytes<R>();
  static constexpr int kNumBars = 2 * kRawStages + 2 * kAStages + 2 * kBStages + 5;
  static constexpr int kTmemSlot = kBar + 8 * kNumBars;
  static constexpr int kTotal = kTmemSlot + 16 + 1024;  // + alignment slack
};

// Byte offset of plane p inside a raw stage: planes are stored back to back, 8 row tiles each.
__device__ __forceinline__ int raw_plane_off(int p) {
  return p == 0 ? 0 : p == 1 ? 8192 : p == 2 ? 12288 : p == 3 ? 16384 : 24576;
}

// Read one lane's plane words of one row tile from a raw stage in shared memory.
template <int R>
__device__ __forceinline__ void lds_lane_words(const uint8_t* raw, int t, int lane, LaneWords& L) {
  {
    const uint8_t* b = raw + raw_plane_off(0) + t * 1024 + lane * 16;
    const uint4 a = *reinterpret_cast<const uint4*>(b), c = *reinterpret_cast<const uint4*>(b + 512);
    L.p0[0] = a.x; L.p0[1] = a.y; L.p0[2] = a.z; L.p0[3] = a.w;
    L.p0[4] = c.x; L.p0[5] = c.y; L.p0[6] = c.z; L.p0[7] = c.w;
  }
  if constexpr (R >= 3) {
    const uint4 a = *reinterpret_cast<const uint4*>(raw + raw_plane_off(1) + t * 512 + lane * 16);
    L.p1[0] = a.x; L.p1[1] = a.y; L.p1[2] = a.z; L.p1[3] = a.w;
  }
  if constexpr (R >= 4) {
    const uint4 a = *reinterpret_cast<const uint4*>(raw + raw_plane_off(2) + t * 512 + lane * 16);
    L.p2[0] = a.x; L.p2[1] = a.y; L.p2[2] = a.z; L.p2[3] = a.w;
  }
  if constexpr (R >= 6) {
    const uint8_t* b = raw + raw_plane_off(3) + t * 1024 + lane * 16;
    const uint4 a = *reinterpret_cast<const uint4*>(b), c = *reinterpret_cast<const uint4*>(b + 512);
    L.p3[0] = a.x; L.p3[1] = a.y; L.p3[2] = a.z; L.p3[3] = a.w;
    L.p3[4] = c.x; L.p3[5] = c.y; L.p3[6] = c.z; L.p3[7] = c.w;
  }
  if constexpr (R >= 8) {
    const uint8_t* b = raw + raw_plane_off(4) + t * 1024 + lane * 16;
    const uint4 a = *reinterpret_cast<const uint4*>(b), c = *reinterpret_cast<const uint4*>(b + 512);
    L.p4[0] = a.x; L.p4[1] = a.y; L.p4[2] = a.z; L.p4[3] = a.w;
    L.p4[4] = c.x; L.p4[5] = c.y; L.p4[6] = c.z; L.p4[7] = c.w;
  }
}

// Multiplier m_rho = 2^(8-r) / sigma_rho turning (A - 1024) into 2^(8-r) * p.
template <int R>
__device__ __forceinline__ float code_mult(int rho) {
  if constexpr (R == 2) return (float)(64 >> (2 * rho));
  else if constexpr (R == 3) return rho < 2 ? 32.f : 2.f;
  else if constexpr (R == 4) return rho < 2 ? 16.f : 1.f;
  else return 1.f;
}

// Dequantise the two MMA tiles of block W for one row tile and store them into the A slot.
// rows: sr[0] / dz[0] for row gid, sr[1] / dz[1] for row gid + 8 (fp16 pairs, both halves equal).
template <int R, int W>
__device__ __forceinline__ void dequant_block(const LaneWords& L, const __half2 (&s2)[2], const __half2 (&dz2)[2],
                                              uint32_t a_slot, int t, int lane) {
  uint32_t A[2][4];
  build_operands<R, W>(L, A);
  const __half2 k1024 = __float2half2_rn(1024.f);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t o[4];
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {
      const __half2 v = *reinterpret_cast<const __half2*>(&A[j][rho]);
      const int rsel = rho & 1;  // rho 0, 2: row gid; rho 1, 3: row gid + 8
      __half2 u;
      if constexpr (R == 8) {
        u = __hsub2(v, __hadd2(k1024, dz2[rsel]));  // dz2 holds z here: v - (1024 + z), exact
      } else {
        u = __hfma2(__hsub2(v, k1024), __float2half2_rn(code_mult<R>(rho)), dz2[rsel]);
      }
      const __half2 w = __hmul2(u, s2[rsel]);
      o[rho] = *reinterpret_cast<const uint32_t*>(&w);
    }
    // stmatrix: lane i addresses row (i % 8) of matrix (i / 8); matrices 0..3 = (rows 0-7,
    // k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15) of this 16x16 tile.
    const int mi = lane >> 3;
    const int row = t * 16 + (lane & 7) + 8 * (mi & 1);
    const int kloc = 32 * (W & 1) + 16 * j + 8 * (mi >> 1);  // input within the 64-wide slot
    const int chunk16 = kloc >> 3;
    const uint32_t addr = a_slot + row * 128 + ((chunk16 ^ (row & 7)) << 4);
    stmatrix_x4(addr, o[0], o[1], o[2], o[3]);
  }
}

// Scale bits and zero points of one 256-input chunk for a lane's rows (gid, gid + 8 of each of
// its row tiles), NG = 256 / GROUP groups; loaded before the chunk's planes are waited for.
template <int GROUP>
struct ChunkMeta {
  static constexpr int NG = kChunk / GROUP;
  uint32_t sb[kTilesPerWarp][NG][2];
  uint32_t zb[kTilesPerWarp][NG][2];
};

template <int GROUP>
__device__ __forceinline__ void load_chunk_meta(ChunkMeta<GROUP>& m, const PrefillParams& P, int kc, int rt0, int wq,
                                                int lane) {
  const int gid = lane >> 2;
#pragma unroll
  for (int tt = 0; tt < kTilesPerWarp; ++tt)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = (rt0 + kTilesPerWarp * (wq / kWarpsPerTile) + tt) * kTileRows + gid + 8 * h;
#pragma unroll
      for (int g = 0; g < ChunkMeta<GROUP>::NG; ++g) {
        m.sb[tt][g][h] = 0u;
        m.zb[tt][g][h] = 0u;
        if (row < P.N) {
          const size_t o = (size_t)row * P.G + (size_t)kc * ChunkMeta<GROUP>::NG + g;
          m.sb[tt][g][h] = P.scales[o];
          m.zb[tt][g][h] = P.zeros[o];
        }
      }
    }
}

template <int R, int BN, int GROUP, int Q>
__device__ __forceinline__ void dequant_substage(const LaneWords (&L)[kTilesPerWarp], const ChunkMeta<GROUP>& m,
                                                 int wq, int lane, uint32_t a_slot, float delta) {
  constexpr int g = (Q * kSubK) / GROUP;  // group of this 64-input slice inside the chunk
#pragma unroll
  for (int tt = 0; tt < kTilesPerWarp; ++tt) {
    const int t = kTilesPerWarp * (wq / kWarpsPerTile) + tt;
    __half2 s2[2], dz2[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float sv = __half2float(__ushort_as_half((unsigned short)m.sb[tt][g][h]));
      const float zf = (float)m.zb[tt][g][h];
      s2[h] = __float2half2_rn(sv);
      dz2[h] = __float2half2_rn(R == 8 ? zf : (delta - zf));
    }
    if constexpr (kWarpsPerTile == 1) {
      dequant_block<R, 2 * Q>(L[tt], s2, dz2, a_slot, t, lane);
      dequant_block<R, 2 * Q + 1>(L[tt], s2, dz2, a_slot, t, lane);
    } else if (wq % 2 == 0) {
      dequant_block<R, 2 * Q>(L[tt], s2, dz2, a_slot, t, lane);
    } else {
      dequant_block<R, 2 * Q + 1>(L[tt], s2, dz2, a_slot, t, lane);
    }
  }
}

// Extra-Precision fix-up of the fp16 weight tiles (compiled only into the kernels for calls with
// a list, so the dequantising loop of every other call carries none of it).  Lane l < 16 of a dequantising warp follows
// the list of row l of the warp's 16-row tile: a 16-entry window of the list (two 16-byte loads
// from the 8-entry boundary at or below the cursor, none past the row's end), refreshed at each
// chunk and whenever a slice uses it up, and the fp16 values s * (256 - z) of the chunk's
// groups.  After the slice's tile is in shared memory the lane overwrites the listed weights of
// the slice.
template <int GROUP>
struct OvfCursor {
  static constexpr int NG = kChunk / GROUP;
  int cur = 0, end = 0, base = 0;
  uint32_t win[8];
  uint16_t val[NG];

  __device__ __forceinline__ void load_window(const uint16_t* cols) {
    base = cur & ~7;
    const uint4 z4 = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
    const uint4 a = base < end ? *reinterpret_cast<const uint4*>(cols + base) : z4;
    const uint4 b = base + 8 < end ? *reinterpret_cast<const uint4*>(cols + base + 8) : z4;
    win[0] = a.x; win[1] = a.y; win[2] = a.z; win[3] = a.w;
    win[4] = b.x; win[5] = b.y; win[6] = b.z; win[7] = b.w;
  }

  // the row's list from its first input >= kstart (a K split starts past input 0)
  __device__ __forceinline__ void start_tile(const PrefillParams& P, int row, int kstart) {
    cur = end = 0;
    if (row < P.N) {
      cur = P.ovf_row_ptr[row];
      end = P.ovf_row_ptr[row + 1];
      if (kstart > 0) {
        int lo = cur, hi = end;  // first entry with k >= kstart
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if ((int)P.ovf_cols[mid] < kstart) lo = mid + 1;
          else hi = mid;
        }
        cur = lo;
      }
    }
  }

  __device__ __forceinline__ void start_chunk(const PrefillParams& P, int row, int kc) {
    load_window(P.ovf_cols);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      val[g] = 0;
      if (row < P.N && cur < end) {
        const size_t o = (size_t)row * P.G + (size_t)kc * NG + g;
        const __half s = __ushort_as_half(P.scales[o]);
        const __half v = __hmul(__float2half_rn(256.f - (float)P.zeros[o]), s);
        val[g] = __half_as_ushort(v);
      }
    }
  }

  // Overwrite the listed weights with inputs kc*256 + 64q .. +63 in the A slot (row arow of the
  // 128-row tile, 128-byte swizzled rows of 64 fp16 values).
  __device__ __forceinline__ void patch(const uint16_t* cols, int kc, int q, uint32_t a_slot, int arow) {
    const int k0 = kc * kChunk + q * kSubK;
    for (;;) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k = (int)((win[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
        if (base + j == cur && cur < end && k < k0 + kSubK) {
          const int kl = k - k0;
          const uint32_t addr = a_slot + arow * 128 + ((((kl >> 3) ^ (arow & 7))) << 4) + (kl & 7) * 2;
          const int gi = (k - kc * kChunk) / GROUP;
          uint16_t v = val[0];
#pragma unroll
          for (int g = 1; g < NG; ++g)
            if (gi == g) v = val[g];
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
          ++cur;
        }
      }
      if (cur < end && cur >= base + 16) {
        load_window(cols);  // the slice used the whole window: continue from the cursor
        continue;
      }
      break;
    }
  }
};

template <int R, int BN, int GROUP, bool EP, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_p0, const __grid_constant__ CUtensorMap tm_p1,
               const __grid_constant__ CUtensorMap tm_p2, const __grid_constant__ CUtensorMap tm_p3,
               const __grid_constant__ CUtensorMap tm_p4, const __grid_constant__ CUtensorMap tm_x,
               const PrefillParams P) {
  using S = PrefillSmem<R, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + kRawStages;
  uint64_t* a_full = raw_empty + kRawStages;
  uint64_t* a_empty = a_full + kAStages;
  uint64_t* b_full = a_empty + kAStages;
  uint64_t* b_empty = b_full + kBStages;
  uint64_t* acc_full = b_empty + kBStages;   // [2]: accumulator buffer complete (tcgen05.commit)
  uint64_t* acc_empty = acc_full + 2;        // [2]: accumulator buffer drained by the epilogue
  uint64_t* drain = acc_empty + 2;           // error path: completion of every MMA issued
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KC = P.K / kChunk;
  // Persistent: CTA b takes tiles b, b + grid, ...; tile t = (weight-row block, K split, token
  // tile), token tiles fastest so that the CTAs working on one row block at a time share its
  // planes through L2.  Two TMEM accumulators: the epilogue of tile i overlaps the MMAs of
  // tile i + 1.  With S > 1 K splits (small problems: too few tiles for the SMs) each tile
  // covers chunks [sp*KC/S, (sp+1)*KC/S) and writes fp32 partial sums.
  const int MT = (P.M + BN - 1) / BN;
  const int NS = SPLIT ? P.S : 1;  // K splits (compiled in only where a call splits)
  const int tiles = MT * ((P.N + kBM - 1) / kBM) * NS;
  // tile t -> (row block, first and end chunk, first token)
  struct TileCoord { int rb, kc0, kc1, m0, sp; };
  auto coord = [&](int t) {
    TileCoord c;
    const int mt = t % MT, rest = t / MT;
    if constexpr (SPLIT) {
      c.sp = rest % NS;
      c.rb = rest / NS;
      c.kc0 = (int)((long long)c.sp * KC / NS);
      c.kc1 = (int)((long long)(c.sp + 1) * KC / NS);
    } else {
      c.sp = 0;
      c.rb = rest;
      c.kc0 = 0;
      c.kc1 = KC;
    }
    c.m0 = mt * BN;
    return c;
  };
  const int my_tiles = (tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  constexpr int kNumPlanes = planes_for_width(R);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRawStages; ++i) { mbar_init(&raw_full[i], 1); mbar_init(&raw_empty[i], kDeqWarps); }
    for (int i = 0; i < kAStages; ++i) { mbar_init(&a_full[i], 32 * kDeqWarps); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < kBStages; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], kEpiWarps); }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)(2 * BN))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // x16 comes from the conversion kernel; y may be read by earlier kernels

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const CUtensorMap* maps[5] = {&tm_p0, &tm_p1, &tm_p2, &tm_p3, &tm_p4};
      bool ok = true;
      int ic = 0, ib = 0;  // running chunk (raw ring) and 64-input slice (B ring) counts
      int ic_sent = 0, ib_sent = 0;  // loads issued (the error path waits for the last of them)
      for (int i = 0; i < my_tiles && ok; ++i) {
        const TileCoord tc = coord((int)blockIdx.x + i * (int)gridDim.x);
        const int m0 = tc.m0, rt0 = tc.rb * (kBM / kTileRows);
        for (int kc = tc.kc0; kc < tc.kc1 && ok; ++kc, ++ic) {
          const int rs = ic % kRawStages;
          ok = mbar_wait(&raw_empty[rs], ((ic / kRawStages) & 1) ^ 1, P.err, 1);
          if (!ok) break;
          mbar_expect_tx(&raw_full[rs], raw_stage_bytes<R>());
          uint8_t* raw = smem + S::kRaw + rs * raw_stage_bytes<R>();
#pragma unroll
          for (int p = 0; p < kNumPlanes; ++p)
            tma_load_2d(raw + raw_plane_off(p), maps[p], kc * plane_bits(p) * 64, rt0, &raw_full[rs]);
          ic_sent = ic + 1;
          for (int q = 0; q < 4; ++q, ++ib) {
            const int bs = ib % kBStages;
            ok = mbar_wait(&b_empty[bs], ((ib / kBStages) & 1) ^ 1, P.err, 2);
            if (!ok) break;
            mbar_expect_tx(&b_full[bs], BN * 128);
            tma_load_2d(smem + S::kB + bs * BN * 128, &tm_x, kc * kChunk + q * kSubK, m0, &b_full[bs]);
            ib_sent = ib + 1;
          }
        }
      }
      if (!ok) {
        // error path: no copy may still be landing in shared memory when the CTA exits; every
        // load before the last ring's worth was consumed before its slot was reused
        for (int c = ic_sent > kRawStages ? ic_sent - kRawStages : 0; c < ic_sent; ++c)
          mbar_wait(&raw_full[c % kRawStages], (c / kRawStages) & 1, P.err, 1);
        for (int c = ib_sent > kBStages ? ib_sent - kBStages : 0; c < ib_sent; ++c)
          mbar_wait(&b_full[c % kBStages], (c / kBStages) & 1, P.err, 2);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      bool ok = true;
      int is = 0;  // running 64-input slice count (A and B rings advance together)
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int buf = i & 1;
        ok = mbar_wait(&acc_empty[buf], ((i >> 1) & 1) ^ 1, P.err, 128);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tmem_d + (uint32_t)(buf * BN);
        const TileCoord tc = coord((int)blockIdx.x + i * (int)gridDim.x);
        for (int sub = 0; sub < (tc.kc1 - tc.kc0) * 4 && ok; ++sub, ++is) {
          const int as = is % kAStages, bs = is % kBStages;
          ok = mbar_wait(&a_full[as], (is / kAStages) & 1, P.err, 4) && mbar_wait(&b_full[bs], (is / kBStages) & 1, P.err, 8);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + S::kA + as * kATileBytes);
          const uint32_t b_base = smem_u32(smem + S::kB + bs * BN * 128);
#pragma unroll
          for (int kk = 0; kk < kSubK / 16; ++kk)
            tc_mma_f16(d, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32), idesc,
                       (sub > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&a_empty[as]);
          tc_commit(&b_empty[bs]);
        }
        if (ok) tc_commit(&acc_full[buf]);
      }
      if (!ok) {
        // error path: wait (bounded) until every MMA issued so far has completed, before the
        // accumulators are deallocated
        tc_commit(drain);
        mbar_wait(drain, 0, P.err, 4);
      }
    }
  } else if (warp >= 4 && warp < 4 + kDeqWarps) {
    // ---------------- dequantisation ----------------
    const int wq = warp - 4;
    bool ok = true;
    int ic = 0, is = 0;  // running chunk and 64-input slice counts
    static_assert(kTilesPerWarp == 1 && kWarpsPerTile == 1, "the list fix-up assumes one 16-row tile per warp");
    constexpr bool ovf = EP;  // Extra-Precision list given (P.ovf_row_ptr non-null)
    OvfCursor<GROUP> oc;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const TileCoord tc = coord((int)blockIdx.x + i * (int)gridDim.x);
      const int rt0 = tc.rb * (kBM / kTileRows);
      const int orow = (rt0 + wq) * kTileRows + lane;  // the row whose list lane (< 16) follows
      ChunkMeta<GROUP> meta;
      load_chunk_meta<GROUP>(meta, P, tc.kc0, rt0, wq, lane);
      if (ovf && lane < 16) oc.start_tile(P, orow, tc.kc0 * kChunk);
      for (int kc = tc.kc0; kc < tc.kc1 && ok; ++kc, ++ic) {
        const int rs = ic % kRawStages;
        if (kc > tc.kc0) load_chunk_meta<GROUP>(meta, P, kc, rt0, wq, lane);
        if (ovf && lane < 16) oc.start_chunk(P, orow, kc);
        ok = mbar_wait(&raw_full[rs], (ic / kRawStages) & 1, P.err, 16);
        if (!ok) break;
        const uint8_t* raw = smem + S::kRaw + rs * raw_stage_bytes<R>();
        LaneWords L[kTilesPerWarp];
#pragma unroll
        for (int tt = 0; tt < kTilesPerWarp; ++tt)
          lds_lane_words<R>(raw, kTilesPerWarp * (wq / kWarpsPerTile) + tt, lane, L[tt]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&raw_empty[rs]);
#define MATQ_SUBSTAGE(Q)                                                                       \
        if (ok) {                                                                              \
          const int as = is % kAStages;                                                        \
          ok = mbar_wait(&a_empty[as], ((is / kAStages) & 1) ^ 1, P.err, 32);                  \
          if (ok) {                                                                            \
            const uint32_t a_slot = smem_u32(smem + S::kA + as * kATileBytes);                 \
            dequant_substage<R, BN, GROUP, Q>(L, meta, wq, lane, a_slot, P.delta);             \
            if (ovf) {                                                                         \
              __syncwarp();                                                                    \
              if (lane < 16) oc.patch(P.ovf_cols, kc, Q, a_slot, wq * kTileRows + lane);       \
              __syncwarp();                                                                    \
            }                                                                                  \
            fence_proxy_async();                                                               \
            mbar_arrive(&a_full[as]);                                                          \
          }                                                                                    \
          ++is;                                                                                \
        }
        MATQ_SUBSTAGE(0) MATQ_SUBSTAGE(1) MATQ_SUBSTAGE(2) MATQ_SUBSTAGE(3)
#undef MATQ_SUBSTAGE
      }
    }
  } else if (warp >= 4 + kDeqWarps) {
    // ---------------- epilogue ----------------
    // warp w reads TMEM lanes 32*(w%4) .. +31 = weight rows n0 + 32*(w%4) + lane
    const int q = warp & 3;
    bool ok = true;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const int buf = i & 1;
      ok = mbar_wait(&acc_full[buf], (i >> 1) & 1, P.err, 64);
      if (!ok) break;
      tc_fence_after();
      const TileCoord tc = coord((int)blockIdx.x + i * (int)gridDim.x);
      const int m0 = tc.m0, n = tc.rb * kBM + 32 * q + lane;
      const uint32_t taddr = tmem_d + (uint32_t)(buf * BN) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(taddr + c * 32, v);
        {
          // tokens whose activations were scaled down get their factor back (warp-uniform test)
          const int tl = m0 + c * 32 + lane;
          const float f = tl < P.M ? P.xscale[tl] : 1.f;
          if (__any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] *= __shfl_sync(0xffffffffu, f, k);
          }
        }
        if (SPLIT) {
          // K split: this split's fp32 partial sums, finished by prefill_finish_kernel
          if (n < P.N) {
            float* part = P.part + (size_t)tc.sp * P.M * P.N;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const int tok = m0 + c * 32 + k;
              if (tok < P.M) part[(size_t)tok * P.N + n] = v[k];
            }
          }
        } else if (P.y_mode == 3) {
          // gated mode: lanes 2i (gate row) and 2i + 1 (up row) share output column n / 2 of
          // y [M, N/2]; the even lane forms tokens 0..15 of the chunk, the odd lane 16..31,
          // each taking the value it lacks from its partner
          const bool even = (lane & 1) == 0;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float other = __shfl_xor_sync(0xffffffffu, even ? v[k + 16] : v[k], 1);
            const float g = even ? v[k] : other;
            const float u = even ? other : v[k + 16];
            const int tok = m0 + c * 32 + k + (even ? 0 : 16);
            if (n < P.N && tok < P.M)
              reinterpret_cast<__nv_bfloat16*>(P.y)[(size_t)tok * (P.N >> 1) + (n >> 1)] =
                  __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u);
          }
        } else if (n < P.N) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int tok = m0 + c * 32 + k;
            if (tok < P.M) {
              const size_t o = (size_t)tok * P.N + n;
              if (P.y_mode == 0) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v[k]);
              else if (P.y_mode == 1) reinterpret_cast<float*>(P.y)[o] = v[k];
              else reinterpret_cast<float*>(P.y)[o] += v[k];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_d), "r"((uint32_t)(2 * BN)) : "memory");
  }
}

// Sum of the S partial results of a K-split call, in split order (deterministic), finished in
// the call's output mode; one thread per output element (gated: per output column pair).
__global__ void __launch_bounds__(256) prefill_finish_kernel(const float* __restrict__ part, int S, int M, int N,
                                                            void* __restrict__ y, int y_mode) {
  pdl_launch_dependents();
  pdl_wait();  // the partial sums come from the split kernel
  const size_t MN = (size_t)M * N;
  const size_t cols = y_mode == 3 ? (size_t)(N >> 1) : (size_t)N;
  const size_t total = (size_t)M * cols;
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (size_t)gridDim.x * 256) {
    const size_t m = i / cols, j = i - m * cols;
    if (y_mode == 3) {
      const size_t o = m * N + 2 * j;
      float g = 0.f, u = 0.f;
      for (int sp = 0; sp < S; ++sp) {
        g += part[sp * MN + o];
        u += part[sp * MN + o + 1];
      }
      reinterpret_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u);
    } else {
      float v = 0.f;
      for (int sp = 0; sp < S; ++sp) v += part[sp * MN + i];
      if (y_mode == 0) reinterpret_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
      else if (y_mode == 1) reinterpret_cast<float*>(y)[i] = v;
      else reinterpret_cast<float*>(y)[i] += v;
    }
  }
}

// ---- host side -----------------------------------------------------------------------------
static size_t r256p(size_t b) { return (b + 255) & ~size_t(255); }

static int prefill_bn(int M) { return M <= 64 ? 64 : (M <= 128 ? 128 : 256); }

// K splits of a call: 1 when the (row block, token tile) tiles alone keep at least half the SMs
// busy; otherwise as many as the SMs allow, each at least two 256-input chunks, at most 8.
int prefill_splits(int M, int K, int N) {
  const int sms = sm_count(current_device());
  const long long tiles = (long long)((M + prefill_bn(M) - 1) / prefill_bn(M)) * ((N + kBM - 1) / kBM);
  if (2 * tiles >= sms) return 1;
  long long S = sms / tiles;
  const int KC = K / kChunk;
  if (S > KC / 2) S = KC / 2;
  if (S > 8) S = 8;
  while (S > 1 && S * M * (long long)N * 4 > (64LL << 20)) --S;  // partial sums: at most 64 MB
  return S < 2 ? 1 : (int)S;
}

// fp16 copy of x and one float per token (its scale factor): what every prefill call needs
size_t prefill_scratch_min_bytes(int M, int K) { return r256p((size_t)M * K * 2) + r256p((size_t)M * 4); }

// ... plus the K-split partial sums, used when the workspace has room for them
size_t prefill_scratch_bytes(int M, int K, int N) {
  const int S = prefill_splits(M, K, N);
  return prefill_scratch_min_bytes(M, K) + (S > 1 ? r256p((size_t)S * M * N * 4) : 0);
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
  }
  return fn;
}

static bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, int BN, int GROUP, bool EP, bool SPLIT>
static cudaError_t launch_t(const CUtensorMap (&maps)[6], const PrefillParams& P, cudaStream_t s) {
  using S = PrefillSmem<R, BN>;
  auto kern = prefill_kernel<R, BN, GROUP, EP, SPLIT>;
  // the shared-memory attribute is set once per device for this kernel
  static std::atomic<unsigned long long> attr_set{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(attr_set.load(std::memory_order_relaxed) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit, std::memory_order_relaxed);
  }
  // persistent: at most one CTA per SM (the kernel's shared memory allows no second one)
  const int sms = sm_count(dev);
  const long long tiles = (long long)((P.M + BN - 1) / BN) * ((P.N + kBM - 1) / kBM) * P.S;
  dim3 grid((unsigned)(tiles < sms ? tiles : sms));
  cudaError_t e = launch_pdl(kern, grid, dim3(kThreads), (size_t)S::kTotal, s, maps[0], maps[1], maps[2], maps[3],
                             maps[4], maps[5], P);
  if (e != cudaSuccess || P.S == 1) return e;
  const long long outs = (long long)P.M * (P.y_mode == 3 ? P.N / 2 : P.N);
  long long blocks = (outs + 255) / 256;
  if (blocks > 4 * sms) blocks = 4 * sms;
  return launch_pdl(prefill_finish_kernel, dim3((unsigned)blocks), dim3(256), 0, s, (const float*)P.part, P.S, P.M,
                    P.N, P.y, P.y_mode);
}

template <int BN, int GROUP, bool SPLIT>
static cudaError_t launch_bn_split(int r, const CUtensorMap (&maps)[6], const PrefillParams& P, cudaStream_t s) {
  switch (r) {
    case 2: return launch_t<2, BN, GROUP, false, SPLIT>(maps, P, s);
    case 3: return launch_t<3, BN, GROUP, false, SPLIT>(maps, P, s);
    case 4: return launch_t<4, BN, GROUP, false, SPLIT>(maps, P, s);
    case 6: return launch_t<6, BN, GROUP, false, SPLIT>(maps, P, s);
    default: return launch_t<8, BN, GROUP, false, SPLIT>(maps, P, s);
  }
}

// Kernel variants: true-prefix calls unsplit or K-split; Extra-Precision calls (the list
// fix-up compiled in, r < 8 only: width 8 rounds nothing) unsplit.
template <int BN, int GROUP>
static cudaError_t launch_bn(int r, const CUtensorMap (&maps)[6], const PrefillParams& P, cudaStream_t s) {
  if (P.ovf_row_ptr == nullptr || r == 8)
    return P.S > 1 ? launch_bn_split<BN, GROUP, true>(r, maps, P, s) : launch_bn_split<BN, GROUP, false>(r, maps, P, s);
  switch (r) {
    case 2: return launch_t<2, BN, GROUP, true, false>(maps, P, s);
    case 3: return launch_t<3, BN, GROUP, true, false>(maps, P, s);
    case 4: return launch_t<4, BN, GROUP, true, false>(maps, P, s);
    default: return launch_t<6, BN, GROUP, true, false>(maps, P, s);
  }
}

cudaError_t launch_prefill(const void* x, int M, int K, const void* planes, const PlaneGeom& g, const uint16_t* scales,
                           const uint8_t* zeros, int r, int group, float delta, const int* ovf_row_ptr,
                           const uint16_t* ovf_cols, void* y, int y_mode, void* workspace, size_t ws_bytes,
                           cudaStream_t s) {
  uint8_t* ws = (uint8_t*)workspace;
  int* err = (int*)(ws + 4);  // sticky prefill error word in the workspace header
  __half* x16 = (__half*)(ws + workspace_header_bytes());
  float* xscale = (float*)(ws + workspace_header_bytes() + ((((size_t)M * K * 2) + 255) & ~size_t(255)));
  {
    cudaError_t e = launch_pdl(xprep_prefill_kernel, dim3(M), dim3(kXprepThreads), 0, s, (const uint16_t*)x, K, x16,
                               xscale);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap maps[6];
  const uint8_t* base = (const uint8_t*)planes;
  for (int p = 0; p < kPlanes; ++p) {
    const int b = plane_bits(p);
    if (p < planes_for_width(r)) {
      if (!make_map_2d(&maps[p], CU_TENSOR_MAP_DATA_TYPE_UINT64, base + g.off[p], (uint64_t)g.KC * b * 64,
                       (uint64_t)g.RT, (uint64_t)g.KC * b * 512, (uint32_t)(b * 64), 8,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    } else {
      maps[p] = maps[0];  // unused by this width
    }
  }
  const int BN = prefill_bn(M);
  if (!make_map_2d(&maps[5], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64,
                   (uint32_t)BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  PrefillParams P;
  P.M = M;
  P.N = g.N;
  P.K = K;
  P.G = K / group;
  P.RT = g.RT;
  P.scales = scales;
  P.zeros = zeros;
  P.xscale = xscale;
  P.delta = delta;
  P.ovf_row_ptr = ovf_row_ptr;
  P.ovf_cols = ovf_cols;
  // K splits: when the workspace has room for the partial sums; Extra-Precision calls do not split
  P.S = (ovf_row_ptr == nullptr && workspace_header_bytes() + prefill_scratch_bytes(M, K, g.N) <= ws_bytes)
            ? prefill_splits(M, K, g.N)
            : 1;
  P.part = (float*)((uint8_t*)xscale + r256p((size_t)M * 4));
  P.y = y;
  P.y_mode = y_mode;
  P.err = err;
  if (group == 64) {
    if (BN == 64) return launch_bn<64, 64>(r, maps, P, s);
    if (BN == 128) return launch_bn<128, 64>(r, maps, P, s);
    return launch_bn<256, 64>(r, maps, P, s);
  }
  if (BN == 64) return launch_bn<64, 128>(r, maps, P, s);
  if (BN == 128) return launch_bn<128, 128>(r, maps, P, s);
  return launch_bn<256, 128>(r, maps, P, s);
}

}  // namespace matq
