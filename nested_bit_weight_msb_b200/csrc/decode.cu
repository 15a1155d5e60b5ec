// Decode path (M <= 16): one persistent, TMA-fed streaming kernel over the packed planes.
//
// Math ("MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models", App. A.1:
// delta folded into the zero point; §4: Y = X W_D computed as (W_D^T X^T)^T so that the
// weights fill the 16-row MMA operand and the tokens the 8-column one):
//
//   y[m, n] = sum_g s[n,g] * ( 2^(8-r) * sum_{k in g} x[m,k] * p[n,k]
//                              + (delta_r - z[n,g]) * sum_{k in g} x[m,k] )
//
// Operands.  A lane's plane words become fp16 A-operand registers in place: a mask-and-or
// against the fp16 bit pattern of 1024 gives 1024 + sigma * v exactly (operands.cuh).  The
// per-register powers of two sigma split into a per-row factor alpha (folded into the group
// scale) and a per-input factor beta (inputs 8..15 of every 16-input MMA slice enter the B
// operand divided by 16 for r <= 4, exact in fp16).  One more MMA per 16-input slice, with a
// constant A operand (rows 0..7: -1024, rows 8..15: beta_k), accumulates both per-token sums
// the algebra needs in registers: Dc = sum_k (-1024) * B_k (removes the 1024 bias) and
// Ds = sum_k beta_k * B_k = sum_k x_k (the zero-point term).  Per slice of a group, in fp32:
//
//   y += a_row * (D + Dc) + s * (delta_r - z) * Ds,   a_row = s * 2^(8-r) / alpha_row
//
// Everything is linear in the inputs, so a group may be split between warps.  No weight is
// ever rounded; x's fp16 operand equals x except below 2^-14 (fp16 subnormals).
//
// Schedule.  Work items are (row group of RG = 4 * RPW row tiles, 256-input chunk), ordered
// row-group-major.  One persistent CTA per SM takes a balanced contiguous range of items
// (stream-K style) and streams each into a shared-memory ring: the planes of width r (one
// 2-D TMA per plane: exactly r bits per weight leave HBM), the chunk's bf16 activation rows
// (one bulk copy per token into padded rows, so fragment loads are conflict-free) and the
// rows' scales and zero points (cp.async).  Eight warps split each item 4 x 2: four row
// slices of RPW row tiles times two 128-input slices; each warp reuses every activation
// fragment across its row tiles.  Row groups inside a CTA's range are written directly.  A
// row group split between CTAs is combined deterministically by whichever contributor finishes
// it last: every contributor stores its partial sums in its workspace slot and takes a ticket
// from the row group's counter; the one holding the last ticket adds the slots in CTA order and
// resets the counter.  No CTA waits for another, so the result does not depend on which CTAs
// are resident at the same time.  The counters live in the workspace header; every call leaves
// them at zero.
//
// Launch.  Programmatic dependent launch: the kernel streams planes (which depend on no
// earlier kernel) as soon as it is resident, and waits for the preceding kernel only before
// reading activations or touching counters and y.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "../../include/matq.h"
#include "common.cuh"
#include "internal.h"
#include "operands.cuh"
#include "sync.cuh"

namespace matq {

constexpr int kRowSlices = 4;        // warps split an item's row tiles four ways ...
// ... and its 256-input chunk into KSL = 2 slices of 128 inputs (8 warps, 256 threads: the
// register budget of a thread stays at 255, and only two code variants share the I-cache)
__host__ __device__ constexpr int k_slices(int NT) { return NT > 0 ? 2 : 2; }
__host__ __device__ constexpr int dec_threads(int NT) { return 32 * kRowSlices * k_slices(NT); }
// Resident CTAs per SM (CPS): two for M <= 8 and r in {2, 6, 8}, and for M <= 16 and r in
// {6, 8} (measured 12 % faster at r = 8), on matrices with K <= 4096
// (each CTA's 8 warps then fit 128 registers a thread, so an SM runs 16 warps and hides more
// latency: measured 7% faster at r = 2, the width with the shortest items; r = 6 and 8 carry
// the most operand-building work per item), otherwise one.  On long-K matrices a row group
// would be split between too many CTAs; at r = 3 and 4 the call measured slower with two.
constexpr int kMaxSMs = 160;  // bound on the SMs used, which sizes the partial-sum workspace
__host__ __device__ constexpr int max_ctas_per_sm(int NT) { return NT == 1 ? 2 : 1; }
constexpr int kXPitch = kChunk * 2 + 16;  // bytes per activation row in a stage (padded)

__host__ __device__ constexpr int rows_per_warp_tiles(int r) { return r <= 4 ? 4 : 2; }

struct DecodeParams {
  int N, K, KC, RT, G, M, y_mode, C, NRG;
  float delta;  // added to every level before the zero point: delta_r, or 0 for stored levels
  long long I;  // items
  const uint16_t* x;
  const uint16_t* scales;
  const uint8_t* zeros;
  float* partial;
  int* counters;
  void* y;
  int* err;
};

template <int R, int NT, int GROUP, int CPS>
struct DecodeLayout {
  static constexpr int RPW = rows_per_warp_tiles(R);
  // the split-row-group slots (decode_workspace_bytes) hold 8 = CPS * RPW * NT fragments a lane
  static_assert(CPS * RPW * NT <= 8, "partial-sum slots sized for CPS * RPW * NT <= 8");
  static constexpr int RG = kRowSlices * RPW;           // row tiles per item
  static constexpr int NG = kChunk / GROUP;             // groups per chunk
  static constexpr int NTOK = NT * 8;
  static constexpr int kPlanes = RG * R * 512;          // all planes of width r for the item
  static constexpr int kX = NTOK * kXPitch;             // activation rows of the chunk
  static constexpr int kMetaS = RG * 16 * 8;            // per row: up to 4 fp16 scales (8 B)
  static constexpr int kMetaZ = RG * 16 * 4;            // per row: one aligned 4-byte word of zeros
  static constexpr int oX = kPlanes;
  static constexpr int oS = oX + kX;
  static constexpr int oZ = oS + kMetaS;
  static constexpr int kStage = ((oZ + kMetaZ) + 127) & ~127;
  static constexpr int KSL = k_slices(NT);
  static constexpr int kThreads = dec_threads(NT);
  // k-slice reduction buffer: two of them at NT = 1, used by alternate flushes (the warps of
  // k-slices > 0 then pass a flush without waiting for the k-slice-0 warps' stores and ticket;
  // measured 1-3 % faster at M <= 8 and slower at M = 16)
  static constexpr bool kTwoRed = NT == 1;
  static constexpr int kRedHalf = (KSL - 1) * kRowSlices * RPW * NT * 4 * 32 * 4;
  static constexpr int kRed = (kTwoRed ? 2 : 1) * kRedHalf;
  // ring depth: up to 4 stages within the CTA's share of the SM's shared memory
  static constexpr int kSmemBudget = CPS == 2 ? 113 * 1024 : 224 * 1024;
  static constexpr int kStagesFit = (kSmemBudget - kRed - 256) / kStage;
  static constexpr int kStages = kStagesFit > 4 ? 4 : kStagesFit < 2 ? 2 : kStagesFit;
  static constexpr int oRed = kStages * kStage;     // k-slice reduction buffer
  static constexpr int oBar = oRed + kRed;
  static constexpr int kSmem = oBar + 2 * kStages * 8 + 128;
  static_assert(kSmem <= kSmemBudget, "decode stage ring exceeds the CTA's shared memory");
};

// plane p's offset inside an item's plane region (RG row tiles each)
template <int RG>
__device__ __forceinline__ int item_plane_off(int p) {
  return RG * 512 * (p == 0 ? 0 : p == 1 ? 2 : p == 2 ? 3 : p == 3 ? 4 : 6);
}

// Lane words of the NB blocks NB*KS .. NB*KS+NB-1 of row tile t (at their natural indices).
template <int R, int RG, int NB, int KS>
__device__ __forceinline__ void lds_slice_words(const uint8_t* planes, int t, int lane, LaneWords& L) {
  constexpr int w0 = NB * KS;                             // first block of the slice
  constexpr int half = w0 / 4, wo = (w0 % 4) * 4;         // 2-bit planes: 512-byte half, byte offset
  auto two_bit = [&](int p, uint32_t* dst) {
    const uint8_t* src = planes + item_plane_off<RG>(p) + t * 1024 + half * 512 + lane * 16 + wo;
    if constexpr (NB == 4) {
      const uint4 a = *reinterpret_cast<const uint4*>(src);
      dst[w0] = a.x; dst[w0 + 1] = a.y; dst[w0 + 2] = a.z; dst[w0 + 3] = a.w;
    } else {
      const uint2 a = *reinterpret_cast<const uint2*>(src);
      dst[w0] = a.x; dst[w0 + 1] = a.y;
    }
  };
  auto one_bit = [&](int p, uint32_t* dst) {
    const uint8_t* src = planes + item_plane_off<RG>(p) + t * 512 + lane * 16 + (w0 / 2) * 4;
    if constexpr (NB == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(src);
      dst[w0 / 2] = a.x; dst[w0 / 2 + 1] = a.y;
    } else {
      dst[w0 / 2] = *reinterpret_cast<const uint32_t*>(src);
    }
  };
  two_bit(0, L.p0);
  if constexpr (R >= 3) one_bit(1, L.p1);
  if constexpr (R >= 4) one_bit(2, L.p2);
  if constexpr (R >= 6) two_bit(3, L.p3);
  if constexpr (R >= 8) two_bit(4, L.p4);
}

// B-operand registers of one 16-input MMA slice (inputs k0..k0+15 of the chunk) for token
// tile nt, built from the bf16 activation rows in the stage: {x[k], x[k+1]} and
// {x[k+8], x[k+9]} * hi_scale as fp16 pairs, k = k0 + 2*(lane%4), token 8*nt + lane/4.
__device__ __forceinline__ void b_frag(const uint8_t* xs, int nt, int k0, int lane, float hi_scale, uint32_t& b0,
                                       uint32_t& b1) {
  const uint8_t* row = xs + (nt * 8 + (lane >> 2)) * kXPitch + (k0 + 2 * (lane & 3)) * 2;
  const uint32_t lo = *reinterpret_cast<const uint32_t*>(row);
  const uint32_t hi = *reinterpret_cast<const uint32_t*>(row + 16);
  __half2 l = __floats2half2_rn(__uint_as_float(lo << 16), __uint_as_float(lo & 0xFFFF0000u));
  __half2 h = __floats2half2_rn(__uint_as_float(hi << 16) * hi_scale, __uint_as_float(hi & 0xFFFF0000u) * hi_scale);
  b0 = *reinterpret_cast<uint32_t*>(&l);
  b1 = *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ long long item_begin(long long c, long long I, long long C) { return c * I / C; }
// CTA whose range holds item u (every CTA has at least one item: C <= I)
__device__ __forceinline__ long long item_owner(long long u, long long I, long long C) {
  return ((u + 1) * C - 1) / I;
}

// Work of one warp: RPW row tiles (row slice rs) x input slice KS of every item.
// Returns the number of ring refills this warp issued (warp 0's count is the TMA requests
// beyond the prologue).
template <int R, int NT, int GROUP, int CPS, int KS, typename Refill>
__device__ __forceinline__ int decode_warp(const DecodeParams& P, uint8_t* smem, uint64_t* full, uint64_t* empty,
                                            float* red, long long c, long long ib, long long ie, int rs, int lane,
                                            Refill&& refill) {
  using Lt = DecodeLayout<R, NT, GROUP, CPS>;
  constexpr int RPW = Lt::RPW, RG = Lt::RG, NG = Lt::NG, KSL = Lt::KSL;
  constexpr int NB = 8 / KSL;                                    // 32-input blocks per slice
  constexpr int kPromoteEvery = (GROUP / 32 < NB) ? GROUP / 32 : NB;  // blocks per scale group part
  constexpr float kHiScale = (R <= 4) ? 0.0625f : 1.0f;
  // constant A operands: -1024 everywhere (bias removal) and beta per input (token sums)
  constexpr uint32_t kNeg1024 = 0xE400E400u;
  constexpr uint32_t kOne = 0x3C003C00u, kBetaHi = (R <= 4) ? 0x4C004C00u : 0x3C003C00u;  // 1.0, 16.0
  constexpr int kLaneFloats = RPW * NT * 4;
  constexpr int kSlotFloats = kLaneFloats * 32;
  const int gid = lane >> 2, tg = lane & 3;
  const int nitems = (int)(ie - ib);
  float amul[2];
  if constexpr (R == 2) { amul[0] = 64.f; amul[1] = 16.f; }
  else if constexpr (R == 3) { amul[0] = amul[1] = 32.f; }
  else if constexpr (R == 4) { amul[0] = amul[1] = 16.f; }
  else { amul[0] = amul[1] = 1.f; }
  // One constant-A MMA yields both token sums: A rows 0..7 are -1024 (D rows 0..7 = Dc) and
  // rows 8..15 are beta_k (D rows 8..15 = Ds).  Fragment registers: {row g, k lo}, {row g+8,
  // k lo}, {row g, k hi}, {row g+8, k hi}; result {Dc(t), Dc(t+1), Ds(t), Ds(t+1)}.
  const uint32_t Acs[4] = {kNeg1024, kOne, kNeg1024, kBetaHi};

  float yacc[RPW][NT][4];
#pragma unroll
  for (int j = 0; j < RPW; ++j)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) yacc[j][nt][i] = 0.f;

  bool ok = true;
  // largest bf16 magnitude seen in this warp's share of the activations (packed pairs): the
  // fp16 operands hold |x| < 65536 only
  uint32_t xmax = 0;
  // (row group, chunk) of the current item, advanced item by item (no division in the loop)
  const int rg_first = (int)(ib / P.KC);
  int rg = rg_first, kc = (int)(ib - (long long)rg_first * P.KC);
  int refills = 0;
  int flushes = 0;  // flushes so far (selects the reduction buffer at NT = 1)
  for (int n = 0; n < nitems; ++n) {
    const int s = n % Lt::kStages;
    if (ok) ok = mbar_wait(&full[s], (n / Lt::kStages) & 1, P.err, 2);
    if (ok) {
      const uint8_t* st = smem + s * Lt::kStage;
      // range check of the activations this item converts: the warps of k-slice KS split its
      // tokens by row slice (every token of the slice is read by exactly one of them)
      for (int t = rs; t < P.M && t < Lt::NTOK; t += kRowSlices) {
        // inputs 128 * KS .. + 127 of the chunk (2 bytes each), 4 per lane
        const uint2 w = *reinterpret_cast<const uint2*>(st + Lt::oX + t * kXPitch + KS * 256 + lane * 8);
        xmax = __vmaxu2(xmax, __vmaxu2(w.x & 0x7FFF7FFFu, w.y & 0x7FFF7FFFu));
      }
      LaneWords L[RPW];
#pragma unroll
      for (int j = 0; j < RPW; ++j) lds_slice_words<R, RG, NB, KS>(st, rs * RPW + j, lane, L[j]);

      float d[RPW][NT][4], dcs[NT][4];
      auto zero_acc = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dcs[nt][i] = 0.f;
#pragma unroll
            for (int j = 0; j < RPW; ++j) d[j][nt][i] = 0.f;
          }
      };
      // Byte offset of this lane's zero points inside their 4-byte windows: the same for every
      // row the lane touches in the item (the rows differ by multiples of 8, and 8 * G is a
      // multiple of 4).
      const int zoff = (int)(((unsigned)gid * (unsigned)P.G + (unsigned)kc * NG) & 3u);
      const uint8_t* srow = st + Lt::oS + (rs * RPW * 16 + gid) * 8;
      const uint8_t* zrow = st + Lt::oZ + (rs * RPW * 16 + gid) * 4 + zoff;
      // fold the inputs accumulated so far (all in scale group gl) into the running sums.
      // Rows >= N read stale scales and zero points; their sums are never stored.
      auto promote = [&](int gl) {
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
          float a[2], cz[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int rr = j * 16 + 8 * h;  // row offset inside the warp's row slice
            const float sv = __half2float(*reinterpret_cast<const __half*>(srow + rr * 8 + gl * 2));
            const float zv = (float)zrow[rr * 4 + gl];
            a[h] = sv * amul[h];
            cz[h] = sv * (P.delta - zv);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              yacc[j][nt][i] = fmaf(cz[i >> 1], dcs[nt][2 + (i & 1)],
                                    fmaf(a[i >> 1], d[j][nt][i] + dcs[nt][i & 1], yacc[j][nt][i]));
        }
        zero_acc();
      };
      zero_acc();

#pragma unroll
      for (int wb = 0; wb < NB; ++wb) {
        uint32_t b0[2][NT], b1[2][NT];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            b_frag(st + Lt::oX, nt, (NB * KS + wb) * 32 + 16 * jj, lane, kHiScale, b0[jj][nt], b1[jj][nt]);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_f16(dcs[nt], Acs, b0[jj][nt], b1[jj][nt]);
          }
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
          uint32_t A[2][4];
          build_slice_operands<R, NB * KS>(L[j], wb, A);
#pragma unroll
          for (int jj = 0; jj < 2; ++jj)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_f16(d[j][nt], A[jj], b0[jj][nt], b1[jj][nt]);
        }
        if ((wb + 1) % kPromoteEvery == 0) promote(((NB * KS + wb) * 32) / GROUP);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    // the streaming warps (0..7) refill this slot with item n + S once every warp released it
    if (rs + kRowSlices * KS < 8 && n + Lt::kStages < nitems && ok) {
      ok = mbar_wait(&empty[s], (n / Lt::kStages) & 1, P.err, 1);
      if (ok) {
        int rg2 = rg, kc2 = kc + Lt::kStages;
        while (kc2 >= P.KC) {
          kc2 -= P.KC;
          ++rg2;
        }
        refill(n + Lt::kStages, rg2, kc2);
        ++refills;
      }
    }

    // flush at the end of a row group (or of this CTA's range); all warps get here for the
    // same items, so the four k-slices of a row slice meet at a named barrier
    if (n == nitems - 1 || kc == P.KC - 1) {
      // With two buffers, flush f + 2 reuses flush f's only after every warp passed flush
      // f + 1's barrier, which the k-slice-0 warps reach after reading flush f's sums.
      float* redf = red + (Lt::kTwoRed ? (flushes++ & 1) * (Lt::kRedHalf / 4) : 0);
      const long long g0 = (long long)rg * P.KC, g1 = g0 + P.KC;
      const bool whole = g0 >= ib && g1 <= ie;
      if (KS > 0) {
        float4* mine =
            reinterpret_cast<float4*>(redf + ((KS - 1) * kRowSlices + rs) * kSlotFloats + lane * kLaneFloats);
#pragma unroll
        for (int j = 0; j < RPW; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mine[j * NT + nt] = make_float4(yacc[j][nt][0], yacc[j][nt][1], yacc[j][nt][2], yacc[j][nt][3]);
      }
      asm volatile("bar.sync 1, %0;" ::"r"(Lt::kThreads) : "memory");
      if (KS == 0) {
#pragma unroll
        for (int k2 = 0; k2 < KSL - 1; ++k2) {
          const float4* o = reinterpret_cast<const float4*>(redf + (k2 * kRowSlices + rs) * kSlotFloats + lane * kLaneFloats);
#pragma unroll
          for (int j = 0; j < RPW; ++j)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const float4 v = o[j * NT + nt];
              yacc[j][nt][0] += v.x;
              yacc[j][nt][1] += v.y;
              yacc[j][nt][2] += v.z;
              yacc[j][nt][3] += v.w;
            }
        }
        auto store_y = [&](int j, int nt, int i, float v) {
          const int row = (rg * RG + rs * RPW + j) * 16 + gid + 8 * (i >> 1);
          const int tok = nt * 8 + 2 * tg + (i & 1);
          if (row < P.N && tok < P.M) {
            const size_t o = (size_t)tok * P.N + row;
            if (P.y_mode == 0) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v);
            else if (P.y_mode == 1) reinterpret_cast<float*>(P.y)[o] = v;
            else reinterpret_cast<float*>(P.y)[o] += v;
          }
        };
        // Four values of one (row tile j, token tile nt) fragment; the whole warp calls this.
        // Gated mode: even rows (gate) take the odd row below (up) from the lane 4 higher and
        // write silu(gate) * up at column row / 2 of y [M, N/2].
        auto store4 = [&](int j, int nt, float v0, float v1, float v2, float v3) {
          if (P.y_mode == 3) {
            const float vv[4] = {v0, v1, v2, v3};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float u = __shfl_down_sync(0xffffffffu, vv[i], 4);
              const int row = (rg * RG + rs * RPW + j) * 16 + gid + 8 * (i >> 1);
              const int tok = nt * 8 + 2 * tg + (i & 1);
              if ((gid & 1) == 0 && row < P.N && tok < P.M)
                reinterpret_cast<__nv_bfloat16*>(P.y)[(size_t)tok * (P.N >> 1) + (row >> 1)] =
                    __float2bfloat16_rn(__fdividef(vv[i], 1.0f + __expf(-vv[i])) * u);
            }
            return;
          }
          store_y(j, nt, 0, v0);
          store_y(j, nt, 1, v1);
          store_y(j, nt, 2, v2);
          store_y(j, nt, 3, v3);
        };
        if (whole) {
#pragma unroll
          for (int j = 0; j < RPW; ++j)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) store4(j, nt, yacc[j][nt][0], yacc[j][nt][1], yacc[j][nt][2], yacc[j][nt][3]);
        } else if (ok) {
          // Split row group: every contributor stores its partial sums in its workspace slot and
          // takes a ticket; the one that takes the last ticket adds all of them in CTA order
          // (deterministic: its own part from registers, the others' from the slots), writes y
          // and resets the counter.  No CTA ever waits for another.
          const long long cf = item_owner(g0, P.I, P.C), cl = item_owner(g1 - 1, P.I, P.C);
          int* cnt = &P.counters[rg * kRowSlices + rs];
          {
            const int side = (rg == rg_first) ? 0 : 1;
            float4* mine = reinterpret_cast<float4*>(
                P.partial + ((size_t)(c * 2 + side) * kRowSlices + rs) * kSlotFloats + lane * kLaneFloats);
#pragma unroll
            for (int j = 0; j < RPW; ++j)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                __stcg(&mine[j * NT + nt], make_float4(yacc[j][nt][0], yacc[j][nt][1], yacc[j][nt][2], yacc[j][nt][3]));
          }
          __syncwarp();  // the warp's partial sums are stored before lane 0 takes the ticket
          int ticket = 0;
          if (lane == 0) {
            // acquire-release ticket: releases the warp's partial sums (cumulative through the
            // warp barrier) and acquires every earlier contributor's
            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(cnt) : "memory");
            if (ticket == (int)(cl - cf)) *reinterpret_cast<volatile int*>(cnt) = 0;  // zero for the next call
          }
          ticket = __shfl_sync(0xffffffffu, ticket, 0);
          __syncwarp();  // orders the other lanes' loads after lane 0's acquire
          if (ticket == (int)(cl - cf)) {
            float4 acc[RPW * NT];
#pragma unroll
            for (int q = 0; q < RPW * NT; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            // every contributor in CTA order; kU at a time so the loads overlap
            constexpr int kU = CPS == 2 ? 1 : (RPW * NT >= 8) ? 2 : (16 / (RPW * NT));
            for (long long c2 = cf; c2 <= cl; c2 += kU) {
              float4 v[kU][RPW * NT];
#pragma unroll
              for (int u = 0; u < kU; ++u) {
                const long long cc = c2 + u;
                if (cc <= cl && cc != c) {
                  const int side2 = (rg == (int)(item_begin(cc, P.I, P.C) / P.KC)) ? 0 : 1;
                  const float4* src = reinterpret_cast<const float4*>(
                      P.partial + ((size_t)(cc * 2 + side2) * kRowSlices + rs) * kSlotFloats + lane * kLaneFloats);
#pragma unroll
                  for (int q = 0; q < RPW * NT; ++q) v[u][q] = __ldcg(&src[q]);
                } else if (cc == c) {
#pragma unroll
                  for (int j = 0; j < RPW; ++j)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                      v[u][j * NT + nt] = make_float4(yacc[j][nt][0], yacc[j][nt][1], yacc[j][nt][2], yacc[j][nt][3]);
                }
              }
#pragma unroll
              for (int u = 0; u < kU; ++u)
                if (c2 + u <= cl)
#pragma unroll
                  for (int q = 0; q < RPW * NT; ++q) {
                    acc[q].x += v[u][q].x;
                    acc[q].y += v[u][q].y;
                    acc[q].z += v[u][q].z;
                    acc[q].w += v[u][q].w;
                  }
            }
#pragma unroll
            for (int j = 0; j < RPW; ++j)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                store4(j, nt, acc[j * NT + nt].x, acc[j * NT + nt].y, acc[j * NT + nt].z, acc[j * NT + nt].w);
          }
        }
      }
      // one buffer: it may be overwritten only after the k-slice-0 warps have read it
      if constexpr (!Lt::kTwoRed) asm volatile("bar.sync 1, %0;" ::"r"(Lt::kThreads) : "memory");
#pragma unroll
      for (int j = 0; j < RPW; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) yacc[j][nt][i] = 0.f;
    }
    if (++kc == P.KC) {
      kc = 0;
      ++rg;
    }
  }
  // an activation of magnitude >= 65536 (bf16 magnitude bits >= 0x4780) has no fp16 operand:
  // the call's outputs are undefined and the status word says so
  const uint32_t big = max(xmax >> 16, xmax & 0xFFFFu);
  if (__any_sync(0xffffffffu, big >= 0x4780u) && lane == 0) atomicOr(P.err, MATQ_STATUS_XRANGE);
  return refills;
}

template <int R, int NT, int GROUP, int CPS>
__global__ void __launch_bounds__(dec_threads(NT), CPS)
decode_kernel(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
              const __grid_constant__ CUtensorMap tm2, const __grid_constant__ CUtensorMap tm3,
              const __grid_constant__ CUtensorMap tm4, const DecodeParams P) {
  using Lt = DecodeLayout<R, NT, GROUP, CPS>;
  constexpr int RG = Lt::RG, NG = Lt::NG, NTOK = Lt::NTOK;
  constexpr int kNumPlanes = planes_for_width(R);
  constexpr int kThreads = Lt::kThreads;
  constexpr int kStreamers = 256;  // threads of warps 0..7, which refill the ring

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lt::oBar);
  uint64_t* empty = full + Lt::kStages;
  float* red = reinterpret_cast<float*>(smem + Lt::oRed);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long c = blockIdx.x;
  const long long ib = item_begin(c, P.I, P.C), ie = item_begin(c + 1, P.I, P.C);
  const int nitems = (int)(ie - ib);
  const CUtensorMap* maps[5] = {&tm0, &tm1, &tm2, &tm3, &tm4};
  const int mrows = P.M < NTOK ? P.M : NTOK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Lt::kStages; ++s) {
      mbar_init(&full[s], 1 + kStreamers);  // thread 0's arrival + one arrival per streamer
      mbar_init(&empty[s], kThreads / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // activation rows >= M stay zero in every stage (nothing is ever copied there)
  for (int s = 0; s < Lt::kStages; ++s)
    for (int i = threadIdx.x; i < (NTOK - mrows) * kXPitch / 4; i += kThreads)
      reinterpret_cast<uint32_t*>(smem + s * Lt::kStage + Lt::oX + mrows * kXPitch)[i] = 0u;
  __syncthreads();
  // the next kernel in the stream may launch its prologue now
  pdl_launch_dependents();

  // Planes of item n into slot n % S (2-D TMA by thread 0): they depend on no earlier kernel.
  auto stream_planes = [&](int n, int rg, int kc) {
    if (threadIdx.x == 0) {
      const int s = n % Lt::kStages;
      uint8_t* st = smem + s * Lt::kStage;
      mbar_expect_tx_only(&full[s], Lt::kPlanes + mrows * kChunk * 2);
#pragma unroll
      for (int p = 0; p < kNumPlanes; ++p)
        tma_load_2d(st + item_plane_off<RG>(p), maps[p], kc * plane_bits(p) * 64, rg * RG, &full[s]);
    }
  };
  // Activation rows of item n: a bulk copy per token (counted in the bytes expected above).
  auto stream_x = [&](int n, int kc) {
    const int s = n % Lt::kStages;
    const int t = threadIdx.x;
    if (t < mrows)
      bulk_load(smem + s * Lt::kStage + Lt::oX + t * kXPitch, P.x + (size_t)t * P.K + (size_t)kc * kChunk,
                kChunk * 2, &full[s]);
  };
  // Scales and zero points (cp.async, one row per streamer thread) of item n, and the
  // streamers' arrivals; called by the streamer threads (warps 0..7) only.
  auto stream_meta = [&](int n, int rg, int kc) {
    const int s = n % Lt::kStages;
    uint8_t* st = smem + s * Lt::kStage;
    const int t = threadIdx.x;
    // scales (NG fp16) and the aligned 4-byte word of zeros holding this chunk's NG bytes.
    // The word never crosses the end of the zeros array except when its NG = 2 bytes are the
    // array's last two and start a word; that row is copied with a plain 2-byte load.
    const int row = rg * RG * 16 + t;
    bool plain = false;
    if (t < RG * 16 && row < P.N) {
      const uint16_t* sp = P.scales + (size_t)row * P.G + (size_t)kc * NG;
      if constexpr (NG == 2) cp_async4(st + Lt::oS + t * 8, sp);
      else cp_async8(st + Lt::oS + t * 8, sp);
      const size_t zi = (size_t)row * P.G + (size_t)kc * NG;
      if ((zi & 3) == 0 && zi + 4 > (size_t)P.N * P.G) {
        plain = true;
        *reinterpret_cast<uint16_t*>(st + Lt::oZ + t * 4) = *reinterpret_cast<const uint16_t*>(P.zeros + zi);
      } else {
        cp_async4(st + Lt::oZ + t * 4, P.zeros + (zi & ~(size_t)3));
      }
    }
    if (plain) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      mbar_arrive(&full[s]);  // a plain arrive releases the plain store too
    } else {
      cp_async_arrive_noinc(&full[s]);
    }
    if (t == 0) mbar_arrive(&full[s]);
  };
  auto refill = [&](int n, int rg, int kc) {
    stream_planes(n, rg, kc);
    stream_x(n, kc);
    stream_meta(n, rg, kc);
  };

  // Prologue: the weights of the first S items (planes, scales, zero points) depend on no
  // earlier kernel and are requested at once; the activations after the wait.
  const int pre = nitems < Lt::kStages ? nitems : Lt::kStages;
  const int rg0 = (int)(ib / P.KC), kc0 = (int)(ib - (long long)rg0 * P.KC);
  for (int n = 0, rg = rg0, kc = kc0; n < pre; ++n) {
    stream_planes(n, rg, kc);
    stream_meta(n, rg, kc);
    if (++kc == P.KC) { kc = 0; ++rg; }
  }
  pdl_wait();  // activations, counters and y belong to earlier kernels in the stream
  for (int n = 0, kc = kc0; n < pre; ++n) {
    stream_x(n, kc);
    if (++kc == P.KC) kc = 0;
  }

  const int rs = warp & 3, ks = warp >> 2;
  static_assert(Lt::KSL == 2, "two input slices per item");
  const int refills = ks == 0 ? decode_warp<R, NT, GROUP, CPS, 0>(P, smem, full, empty, red, c, ib, ie, rs, lane, refill)
                              : decode_warp<R, NT, GROUP, CPS, 1>(P, smem, full, empty, red, c, ib, ie, rs, lane, refill);
  // No copy may still be landing in shared memory when the CTA exits (after a bounded wait
  // gave up, items requested may not have been consumed): each thread's cp.async copies, then
  // thread 0 waits (bounded) for the ring's last requested items.  Every phase has completed on
  // the normal path, so these waits return at once.
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) {
    const int req = pre + refills;
    for (int i = req > Lt::kStages ? req - Lt::kStages : 0; i < req; ++i)
      mbar_wait(&full[i % Lt::kStages], (i / Lt::kStages) & 1, P.err, 2);
  }
}

// Failure-detection self-test: one warp waits, with the bounded wait every kernel uses, on a
// shared-memory barrier that nothing ever completes.  After about a second the wait gives up,
// ORs `code` into the status word and the kernel returns.
__global__ void wait_selftest_kernel(int* err, int code) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, code);
}

cudaError_t launch_wait_selftest(int* err, int code, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err, code);
  return cudaGetLastError();
}

// ---- host side -----------------------------------------------------------------------------
// Workspace: [header: error word + split-row-group counters, zero-filled once by the caller
// and left zero by every call][decode partial-sum slots | prefill scratch].
constexpr size_t kHeaderCounters = size_t(1) << 16;
constexpr size_t kHeaderBytes = 256 + kHeaderCounters * sizeof(int);

size_t workspace_header_bytes() { return kHeaderBytes; }
long long max_decode_rows() { return (long long)(kHeaderCounters / kRowSlices) * 8 * kTileRows; }

size_t decode_workspace_bytes(int M) {
  const int NT = (M <= 8) ? 1 : 2;
  const size_t partial =
      (size_t)2 * kMaxSMs * max_ctas_per_sm(NT) * kRowSlices * 4 * NT * 4 * 32 * sizeof(float);
  return kHeaderBytes + ((partial + 255) & ~size_t(255));
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

static cudaError_t plane_map(CUtensorMap* m, const uint8_t* base, const PlaneGeom& g, int p, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const int b = plane_bits(p);
  const cuuint64_t dims[2] = {(cuuint64_t)g.KC * b * 64, (cuuint64_t)g.RT};
  const cuuint64_t strides[1] = {(cuuint64_t)g.KC * b * 512};
  const cuuint32_t box[2] = {(cuuint32_t)(b * 64), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint8_t*>(base + g.off[p]), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int R, int NT, int GROUP, int CPS>
static cudaError_t launch_decode_t(const uint8_t* planes, const PlaneGeom& g, DecodeParams P, int sms,
                                   cudaStream_t s) {
  using Lt = DecodeLayout<R, NT, GROUP, CPS>;
  CUtensorMap maps[5];
  for (int p = 0; p < 5; ++p) {
    if (p < planes_for_width(R)) {
      cudaError_t e = plane_map(&maps[p], planes, g, p, Lt::RG);
      if (e != cudaSuccess) return e;
    } else {
      maps[p] = maps[0];
    }
  }
  P.NRG = (g.RT + Lt::RG - 1) / Lt::RG;
  P.I = (long long)P.NRG * g.KC;
  const long long ctas = (long long)sms * CPS;
  P.C = (int)(P.I < ctas ? P.I : ctas);
  auto kern = decode_kernel<R, NT, GROUP, CPS>;
  // the shared-memory attribute is set once per device for this kernel
  static std::atomic<unsigned long long> attr_set{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(attr_set.load(std::memory_order_relaxed) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lt::kSmem);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit, std::memory_order_relaxed);
  }
  return launch_pdl(kern, dim3(P.C), dim3(Lt::kThreads), (size_t)Lt::kSmem, s, maps[0], maps[1], maps[2], maps[3],
                    maps[4], P);
}

template <int NT, int GROUP, int CPS>
static cudaError_t launch_decode_r(int r, const uint8_t* planes, const PlaneGeom& g, const DecodeParams& P, int sms,
                                   cudaStream_t s) {
  switch (r) {
    case 2: return launch_decode_t<2, NT, GROUP, NT == 1 ? CPS : 1>(planes, g, P, sms, s);
    case 3: return launch_decode_t<3, NT, GROUP, 1>(planes, g, P, sms, s);
    case 4: return launch_decode_t<4, NT, GROUP, 1>(planes, g, P, sms, s);
    case 6: return launch_decode_t<6, NT, GROUP, CPS>(planes, g, P, sms, s);
    default: return launch_decode_t<8, NT, GROUP, CPS>(planes, g, P, sms, s);
  }
}

cudaError_t launch_decode(const void* x, int M, int K, const void* planes, const PlaneGeom& g, const uint16_t* scales,
                          const uint8_t* zeros, int r, int group, float delta, void* y, int y_mode,
                          void* workspace, cudaStream_t s) {
  const int NT = (M <= 8) ? 1 : 2;
  uint8_t* ws = (uint8_t*)workspace;
  int sms = sm_count(current_device());
  if (sms > kMaxSMs) sms = kMaxSMs;
  DecodeParams P;
  P.N = g.N;
  P.K = K;
  P.KC = g.KC;
  P.RT = g.RT;
  P.G = K / group;
  P.M = M;
  P.y_mode = y_mode;
  P.delta = delta;
  P.x = (const uint16_t*)x;
  P.scales = scales;
  P.zeros = zeros;
  P.err = (int*)ws;
  P.counters = (int*)(ws + 256);
  P.partial = (float*)(ws + kHeaderBytes);
  P.y = y;
  const uint8_t* pl = (const uint8_t*)planes;
  if (NT == 1 && g.KC <= 16)
    return group == 64 ? launch_decode_r<1, 64, 2>(r, pl, g, P, sms, s) : launch_decode_r<1, 128, 2>(r, pl, g, P, sms, s);
  if (NT == 1)
    return group == 64 ? launch_decode_r<1, 64, 1>(r, pl, g, P, sms, s) : launch_decode_r<1, 128, 1>(r, pl, g, P, sms, s);
  // M <= 16: two CTAs per SM on short-K matrices at r = 6 and 8 only (two row tiles a warp
  // there; at r <= 4 four row tiles of two token tiles need more than 128 registers a thread)
  if (g.KC <= 16 && r >= 6)
    return group == 64 ? launch_decode_r<2, 64, 2>(r, pl, g, P, sms, s) : launch_decode_r<2, 128, 2>(r, pl, g, P, sms, s);
  return group == 64 ? launch_decode_r<2, 64, 1>(r, pl, g, P, sms, s) : launch_decode_r<2, 128, 1>(r, pl, g, P, sms, s);
}

}  // namespace matq
