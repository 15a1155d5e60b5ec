// Decode path (M <= 16): a streaming sliced linear layer, bf16 mma.sync fed by a bulk-copy ring.
//
// Math ("MatGPTQ: Efficient and Accurate Inference over Nested Quantized Models", App. A.1:
// delta folded into the zero point; §4: Y = X W_D computed as (W_D^T X^T)^T so that the
// weights fill the 16-row MMA operand and the tokens the 8-column one).  Per group g of a row n:
//
//   y[m, n] += s * ( 2^(8-r) * sum_{k in g} p[n,k] x[m,k] + (delta_r - z) * sum_{k in g} x[m,k] )
//
// Operands.  A lane's plane words become bf16 A-operand registers in place (operands.cuh): a
// mask-and-or against the bf16 pattern of 128 gives 128 + alpha_h * v exactly, v a field of at
// most four bits and alpha_h a power of two fixed by the register's row half.  Widths 6 and 8 take
// two MMAs per tile (code bits 7..4, then bits 3..2 or 3..0).  The activations are the B operand
// as they are (bf16, loaded with ldmatrix): nothing is converted or rounded, so every bf16 input
// value keeps its range and precision.  With D the MMA sum of a group and Ds = sum_k x[m,k]:
//
//   y += a_main * D_main + a_lo * D_lo + s * (delta_r - z) * Ds,   a = s * (weight of the part) / alpha_h
//
// where each D starts the group at -128 * Ds (the C operand of the group's first MMA), so the
// 128 bias cancels inside the MMA sum (a one-hot x gives D = alpha_h * v exactly).  Ds per
// (token, group) is computed once per CTA with a constant-one MMA.
//
// Work split.  The row tiles (16 rows) are dealt to thread-block clusters in balanced contiguous
// ranges; the Q CTAs of a cluster split the 256-input chunks (K) among themselves.  Inside a CTA
// the work is a sequence of units (a group of RPW row tiles x one chunk; RPW = 2 for r <= 4, 1
// above), tile-group-major.  A producer warp streams stage after stage of eight consecutive units
// into a shared-memory ring (bulk copies of the planes of width r only: exactly r bits per weight
// leave HBM; scales and zero points by cp.async), and the eight consumer warps take one unit of
// each stage.  A warp accumulates a tile group over its consecutive units in registers; when a
// tile group is complete the warps' partial sums are added in warp order (shared memory,
// deterministic) and the result is written to y, or, with Q > 1, kept until the end of the
// kernel, when the CTAs of the cluster add their results in rank order through distributed
// shared memory.  No CTA ever waits on a CTA outside its cluster, and the cluster's CTAs are
// co-scheduled by the hardware.  The activations of the CTA's K range stay resident in shared
// memory for the whole kernel.
//
// Launch.  Programmatic dependent launch: the kernel streams planes, scales and zero points
// (which depend on no earlier kernel) as soon as it is resident, and waits for the preceding
// kernel only before reading activations or writing y.  Every wait is bounded (~1 s): on a
// timeout the kernel records a code in the workspace's status word and still reaches every
// barrier, so it returns.
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "../../include/matq.h"
#include "common.cuh"
#include "internal.h"
#include "operands.cuh"
#include "sync.cuh"

namespace matq {

constexpr int kDecConsumers = 8;                        // consumer warps (one unit of each stage each)
constexpr int kDecThreads = 32 * (kDecConsumers + 1);   // and one producer warp
constexpr int kDecMaxStages = 4;
constexpr int kDecSmemBudget = 225 * 1024;

__host__ __device__ constexpr int dec_rpw(int r) { return r <= 4 ? 2 : 1; }
// bits of the planes in front of plane p: a stage holds plane p at 8 * RPW * 512 * this
__host__ __device__ constexpr int dec_bits_before(int p) { return p == 0 ? 0 : p == 1 ? 2 : p == 2 ? 3 : p == 3 ? 4 : 6; }
__host__ __device__ constexpr int dec_stage_planes(int r) { return 8 * dec_rpw(r) * 512 * r; }
__host__ __device__ constexpr int dec_stage_bytes(int r) { return dec_stage_planes(r); }

struct DecodeParams {
  const uint8_t* planes;
  unsigned long long poff[5];
  const uint16_t* x;
  const uint16_t* scales;
  const uint8_t* zeros;
  void* y;
  int* err;
  int N, K, KC, RT, G, M, y_mode;
  int Q;       // CTAs per cluster; they split the chunks
  int ncl;     // clusters; they split the row tiles
  int S;       // ring depth
  int xpitch;  // bytes per activation row in shared memory
  int mspitch, mzpitch;  // bytes per row of the resident scales / zero points
  int o_x, o_zero, o_ds, o_ms, o_mz, o_slots, o_cbuf, o_ring, o_bar;  // shared-memory layout
};

// Operand kinds and dequantisation constants of each width (see the file comment).
template <int R>
struct DecWidth {
  static constexpr int kMain = R == 2 ? kOpP0 : R == 3 ? kOpNib3 : kOpNib4;
  static constexpr bool kLo = R >= 6;
  static constexpr int kLoKind = R == 6 ? kOpP3 : kOpNibLo;
  static constexpr float kDelta = (float)((1 << (8 - R)) - 1) * 0.5f;
  __device__ static float a_main(int h) {
    return (R <= 4 ? (float)(1 << (8 - R)) : 16.f) / (float)op_alpha(kMain, h);
  }
  __device__ static float a_lo(int h) { return kLo ? (R == 6 ? 4.f : 1.f) / (float)op_alpha(kLoKind, h) : 0.f; }
};

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }

// Scales (NG fp16, in NG / 2 words) and zero points (NG bytes) of the rows a consumer lane
// touches in one unit (tile j, row half h).
template <int RPW, int NG>
struct DecMeta {
  uint32_t s[RPW][2][NG / 2];
  uint32_t z[RPW][2];
};
// from the CTA's resident scales [row][group] and zero points [row][group] (rows of the cluster's
// tiles, groups of the CTA's chunks): unit of tile group p, chunk kcl
template <int RPW, int NG>
__device__ __forceinline__ void dec_meta_read(const DecodeParams& P, const uint8_t* smem, int p, int kcl, int lane,
                                              DecMeta<RPW, NG>& m) {
  const int gid = lane >> 2;
#pragma unroll
  for (int j = 0; j < RPW; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = 16 * (p * RPW + j) + gid + 8 * h;
      const uint8_t* ms = smem + P.o_ms + r * P.mspitch + kcl * NG * 2;
      const uint8_t* mz = smem + P.o_mz + r * P.mzpitch + kcl * NG;
      if constexpr (NG == 2) {
        m.s[j][h][0] = *reinterpret_cast<const uint32_t*>(ms);
        m.z[j][h] = *reinterpret_cast<const uint16_t*>(mz);
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(ms);
        m.s[j][h][0] = v.x;
        m.s[j][h][1] = v.y;
        m.z[j][h] = *reinterpret_cast<const uint32_t*>(mz);
      }
    }
}

// One unit: NTILES (<= RPW) row tiles x one 256-input chunk, accumulated into yacc.
//   st      the stage; slot: the unit's index in it (= the consumer warp)
//   kcl     chunk index inside the CTA's K range; kc: global chunk index
//   xaddr   per token tile: ldmatrix row address of this lane (shared::cta), and the byte step per
//           input (2, or 0 for the zero row that stands in for tokens >= M)
//   row0    global row of the unit's first row
template <int R, int NT, int GROUP, int NTILES>
__device__ __forceinline__ void dec_unit(const uint8_t* st, int slot, int kcl, const DecMeta<dec_rpw(R), kChunk / GROUP>& meta,
                                         const uint32_t (&xaddr)[NT], const uint32_t (&xstep)[NT], const float* ds_s,
                                         int lane, float (&yacc)[dec_rpw(R)][NT][4]) {
  using Wd = DecWidth<R>;
  constexpr int RPW = dec_rpw(R);
  constexpr int NG = kChunk / GROUP;   // groups per chunk
  constexpr int BPG = GROUP / 32;      // 32-input blocks per group
  constexpr int NPL = planes_for_width(R);
  constexpr int CH = (NT == 1 && !Wd::kLo) ? 2 : 1;  // independent MMA chains per (tile, token tile)
  const int tg = lane & 3;

  float d[NTILES][NT][CH][4], dl[NTILES][NT][4], dsv[NT][2];
#pragma unroll
  for (int hc = 0; hc < 2; ++hc) {
    HalfWords Hw[NTILES];
#pragma unroll
    for (int j = 0; j < NTILES; ++j) {
      auto two_bit = [&](int p, uint32_t* dst) {
        const uint4 v = lds128(st + dec_bits_before(p) * 8 * RPW * 512 + (j * 8 + slot) * 1024 + hc * 512 + lane * 16);
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
      };
      auto one_bit = [&](int p, uint32_t* dst) {
        const uint2 v = lds64(st + dec_bits_before(p) * 8 * RPW * 512 + (j * 8 + slot) * 512 + lane * 16 + hc * 8);
        dst[0] = v.x; dst[1] = v.y;
      };
      two_bit(0, Hw[j].p0);
      if constexpr (NPL >= 2) one_bit(1, Hw[j].p1);
      if constexpr (NPL >= 3) one_bit(2, Hw[j].p2);
      if constexpr (NPL >= 4) two_bit(3, Hw[j].p3);
      if constexpr (NPL >= 5) two_bit(4, Hw[j].p4);
    }
#pragma unroll
    for (int wb = 0; wb < 4; ++wb) {
      const int W = 4 * hc + wb;
      if (W % BPG == 0) {
        // a new group: its activation sums, and every accumulator starts at -128 * Ds
        const int gq = W / BPG;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const float2 v = *reinterpret_cast<const float2*>(ds_s + (kcl * NG + gq) * 16 + 8 * nt + 2 * tg);
          dsv[nt][0] = v.x;
          dsv[nt][1] = v.y;
        }
#pragma unroll
        for (int j = 0; j < NTILES; ++j)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float b = -128.f * dsv[nt][i & 1];
              d[j][nt][0][i] = b;
#pragma unroll
              for (int c = 1; c < CH; ++c) d[j][nt][c][i] = 0.f;
              dl[j][nt][i] = b;
            }
      }
      uint32_t b[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        ldmatrix_x4(xaddr[nt] + xstep[nt] * (uint32_t)(kcl * kChunk + 32 * W), b[nt][0], b[nt][1], b[nt][2], b[nt][3]);
#pragma unroll
      for (int j = 0; j < NTILES; ++j) {
        uint32_t A[2][4];
        switch (wb) {
          case 0: build_bf16<Wd::kMain, 0>(Hw[j], A); break;
          case 1: build_bf16<Wd::kMain, 1>(Hw[j], A); break;
          case 2: build_bf16<Wd::kMain, 2>(Hw[j], A); break;
          default: build_bf16<Wd::kMain, 3>(Hw[j], A); break;
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_bf16(d[j][nt][jj % CH], A[jj], b[nt][2 * jj], b[nt][2 * jj + 1]);
        if constexpr (Wd::kLo) {
          switch (wb) {
            case 0: build_bf16<Wd::kLoKind, 0>(Hw[j], A); break;
            case 1: build_bf16<Wd::kLoKind, 1>(Hw[j], A); break;
            case 2: build_bf16<Wd::kLoKind, 2>(Hw[j], A); break;
            default: build_bf16<Wd::kLoKind, 3>(Hw[j], A); break;
          }
#pragma unroll
          for (int jj = 0; jj < 2; ++jj)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_bf16(dl[j][nt], A[jj], b[nt][2 * jj], b[nt][2 * jj + 1]);
        }
      }
      if (W % BPG == BPG - 1) {
        // fold the group into the running sums
        const int gq = W / BPG;  // group inside the chunk
#pragma unroll
        for (int j = 0; j < NTILES; ++j)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t sbits = meta.s[j][h][gq >> 1] >> (16 * (gq & 1));
            const float s = __half2float(__ushort_as_half((unsigned short)(sbits & 0xFFFFu)));
            const float z = (float)((meta.z[j][h] >> (8 * gq)) & 0xFFu);
            const float am = s * Wd::a_main(h);
            const float al = s * Wd::a_lo(h);
            const float c = s * (Wd::kDelta - z);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int i = 2 * h + e;
                float dm = d[j][nt][0][i];
                if constexpr (CH == 2) dm += d[j][nt][1][i];
                float acc = fmaf(c, dsv[nt][e], yacc[j][nt][i]);
                acc = fmaf(am, dm, acc);
                if constexpr (Wd::kLo) acc = fmaf(al, dl[j][nt][i], acc);
                yacc[j][nt][i] = acc;
              }
          }
      }
    }
  }
}

// Write one fragment value of a finished tile group to y (all 32 lanes call this together with
// the same k, so the gated mode can pair rows 2i and 2i + 1 across lanes 4 apart).
template <int NT>
__device__ __forceinline__ void dec_out(const DecodeParams& P, float v, int k, int row0, int ntiles, int lane) {
  const int gid = lane >> 2, tg = lane & 3;
  const int j = k / (NT * 4), nt = (k >> 2) % NT, i = k & 3;
  const int row = row0 + 16 * j + gid + 8 * (i >> 1);
  const int tok = 8 * nt + 2 * tg + (i & 1);
  const bool valid = j < ntiles && row < P.N && tok < P.M;
  if (P.y_mode == MATQ_OUT_SILU_GATED) {
    const float u = __shfl_down_sync(0xffffffffu, v, 4);
    if ((gid & 1) == 0 && valid)
      reinterpret_cast<__nv_bfloat16*>(P.y)[(size_t)tok * (P.N >> 1) + (row >> 1)] =
          __float2bfloat16_rn(__fdividef(v, 1.0f + __expf(-v)) * u);
    return;
  }
  if (!valid) return;
  const size_t o = (size_t)tok * P.N + row;
  if (P.y_mode == MATQ_OUT_BF16) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v);
  else if (P.y_mode == MATQ_OUT_F32) reinterpret_cast<float*>(P.y)[o] = v;
  else reinterpret_cast<float*>(P.y)[o] += v;
}

template <int R, int NT, int GROUP>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeParams P) {
  constexpr int RPW = dec_rpw(R);
  constexpr int NG = kChunk / GROUP;
  constexpr int NPL = planes_for_width(R);
  constexpr int FR = RPW * NT * 4;  // fragment values per lane of a tile group
  constexpr int kStage = dec_stage_bytes(R);

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P.o_bar);
  uint64_t* empty = full + kDecMaxStages;
  uint64_t* xbar = empty + kDecMaxStages;
  uint8_t* ring = smem + P.o_ring;
  float* ds_s = reinterpret_cast<float*>(smem + P.o_ds);
  float* slots = reinterpret_cast<float*>(smem + P.o_slots);  // [2][8 warps][FR][32 lanes]
  float* cbuf = reinterpret_cast<float*>(smem + P.o_cbuf);    // [tile group][FR][32 lanes]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's row tiles (its cluster's) and chunks
  const int q = P.Q > 1 ? (int)cluster_rank() : 0;
  const int cl = blockIdx.x / P.Q;
  const int t0 = (int)((long long)P.RT * cl / P.ncl), t1 = (int)((long long)P.RT * (cl + 1) / P.ncl);
  const int T = t1 - t0;
  const int NP = (T + RPW - 1) / RPW;
  const int kc0 = (int)((long long)P.KC * q / P.Q), kc1 = (int)((long long)P.KC * (q + 1) / P.Q);
  const int KCc = kc1 - kc0;
  const int U = NP * KCc;
  const int NST = (U + kDecConsumers - 1) / kDecConsumers;
  const int S = P.S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);  // the producer's expect-tx arrival (+ the planes' bytes)
      mbar_init(&empty[s], kDecConsumers);
    }
    mbar_init(xbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the row that stands in for tokens >= M
  if (threadIdx.x < 8) reinterpret_cast<uint32_t*>(smem + P.o_zero)[threadIdx.x] = 0u;
  __syncthreads();
  pdl_launch_dependents();

  bool ok = true;
  if (warp == kDecConsumers) {
    // ---------------- producer warp ----------------
    // planes of stage n (lane 0): bulk copies, the bytes announced on the stage's barrier
    auto issue_planes = [&](int n) {
      const int s = n % S;
      uint8_t* st = ring + s * kStage;
      const int u0 = n * kDecConsumers, u1 = min(u0 + kDecConsumers, U);
      uint32_t bytes = 0;
      for (int u = u0; u < u1;) {
        const int p = u / KCc, ue = min(u1, (p + 1) * KCc);
        bytes += (uint32_t)((ue - u) * min(RPW, T - p * RPW) * 512 * R);
        u = ue;
      }
      mbar_expect_tx(&full[s], bytes);
      for (int u = u0; u < u1;) {
        const int p = u / KCc, ue = min(u1, (p + 1) * KCc);
        const int kcs = kc0 + (u - p * KCc);
        const int ntl = min(RPW, T - p * RPW);
        for (int j = 0; j < ntl; ++j) {
          const size_t rt = (size_t)(t0 + p * RPW + j);
#pragma unroll
          for (int pl = 0; pl < NPL; ++pl) {
            const int b = plane_bits(pl);
            bulk_load(st + dec_bits_before(pl) * 8 * RPW * 512 + (j * 8 + (u - u0)) * b * 512,
                      P.planes + P.poff[pl] + (rt * P.KC + kcs) * b * 512, (uint32_t)((ue - u) * b * 512), &full[s]);
          }
        }
        u = ue;
      }
    };
    // the planes of the first stages depend on no earlier kernel
    const int pre = min(S, NST);
    if (lane == 0)
      for (int n = 0; n < pre; ++n) issue_planes(n);
    pdl_wait();  // activations (and y) belong to earlier kernels in the stream
    if (lane == 0) mbar_expect_tx(xbar, (uint32_t)(P.M * KCc * kChunk * 2));
    __syncwarp();
    for (int m = lane; m < P.M; m += 32)
      bulk_load(smem + P.o_x + m * P.xpitch, P.x + (size_t)m * P.K + (size_t)kc0 * kChunk, (uint32_t)(KCc * kChunk * 2),
                xbar);
    for (int n = pre; n < NST; ++n) {
      if (lane == 0) {
        if (ok) ok = mbar_wait(&empty[n % S], ((n / S) - 1) & 1, P.err, 2);
        if (ok) issue_planes(n);
      }
    }
  } else {
    // ---------------- consumer warps ----------------
    const int gid = lane >> 2, tg = lane & 3;
    {
      // scales and zero points of the cluster's rows for this CTA's chunks, resident for the whole
      // kernel (they depend on no earlier kernel); eight loads in flight per thread
      const int rows = 16 * T;
      const int sw = KCc * NG / 2;  // 4-byte words of scales per row
      const int zw = KCc * NG / 2;  // 2-byte words of zero points per row
      const int ct = threadIdx.x, nct = 32 * kDecConsumers;
      const int total = rows * (sw + zw);
      for (int base = 0; base < total; base += 8 * nct) {
        uint32_t v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int idx = base + k * nct + ct;
          v[k] = 0u;
          if (idx < total) {
            const int row = idx < rows * sw ? idx / sw : (idx - rows * sw) / zw;
            const int grow = 16 * t0 + row;
            if (grow < P.N) {
              if (idx < rows * sw)
                v[k] = __ldg(reinterpret_cast<const unsigned int*>(P.scales + (size_t)grow * P.G + (size_t)kc0 * NG) +
                             (idx - row * sw));
              else
                v[k] = __ldg(reinterpret_cast<const unsigned short*>(P.zeros + (size_t)grow * P.G + (size_t)kc0 * NG) +
                             (idx - rows * sw - row * zw));
            }
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int idx = base + k * nct + ct;
          if (idx < total) {
            if (idx < rows * sw) {
              const int row = idx / sw;
              *reinterpret_cast<uint32_t*>(smem + P.o_ms + row * P.mspitch + (idx - row * sw) * 4) = v[k];
            } else {
              const int row = (idx - rows * sw) / zw;
              *reinterpret_cast<uint16_t*>(smem + P.o_mz + row * P.mzpitch + (idx - rows * sw - row * zw) * 2) =
                  (uint16_t)v[k];
            }
          }
        }
      }
    }
    pdl_wait();
    // ldmatrix row addresses: lane l reads row l % 8 (a token) of matrix l / 8 (inputs +8 each)
    uint32_t xaddr[NT], xstep[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = 8 * nt + (lane & 7);
      if (tok < P.M) {
        xaddr[nt] = smem_u32(smem + P.o_x + tok * P.xpitch + (lane >> 3) * 16);
        xstep[nt] = 2;
      } else {
        xaddr[nt] = smem_u32(smem + P.o_zero);
        xstep[nt] = 0;
      }
    }
    ok = mbar_wait(xbar, 0, P.err, 4);
    // Ds[group][token] = sum of the group's activations, with a constant-one A operand
    if (ok) {
      const uint32_t kOnes[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // bf16 1.0
      for (int gl = warp; gl < KCc * NG; gl += kDecConsumers) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float dd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int blk = 0; blk < GROUP / 32; ++blk) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(xaddr[nt] + xstep[nt] * (uint32_t)(gl * GROUP + 32 * blk), b0, b1, b2, b3);
            mma_bf16(dd, kOnes, b0, b1);
            mma_bf16(dd, kOnes, b2, b3);
          }
          if (gid == 0) *reinterpret_cast<float2*>(ds_s + gl * 16 + 8 * nt + 2 * tg) = make_float2(dd[0], dd[1]);
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecConsumers) : "memory");

    float yacc[RPW][NT][4];
#pragma unroll
    for (int j = 0; j < RPW; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) yacc[j][nt][i] = 0.f;
    auto flush = [&](int p) {
      float* dst = slots + ((p & 1) * kDecConsumers + warp) * FR * 32 + lane;
#pragma unroll
      for (int j = 0; j < RPW; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dst[((j * NT + nt) * 4 + i) * 32] = yacc[j][nt][i];
            yacc[j][nt][i] = 0.f;
          }
    };

    int cur = -1;
    for (int n = 0; n < NST; ++n) {
      const int s = n % S;
      const int u = n * kDecConsumers + warp;
      const bool has = u < U;
      const int p = has ? u / KCc : -1;
      if (ok) ok = mbar_wait(&full[s], (n / S) & 1, P.err, 1);
      if (has && p != cur) {
        if (cur >= 0) flush(cur);
        cur = p;
      }
      if (has && ok) {
        const int kcl = u - p * KCc;
        const uint8_t* st = ring + s * kStage;
        DecMeta<RPW, NG> meta;
        dec_meta_read<RPW, NG>(P, smem, p, kcl, lane, meta);
        if (RPW == 2 && T - p * RPW >= 2)
          dec_unit<R, NT, GROUP, RPW>(st, warp, kcl, meta, xaddr, xstep, ds_s, lane, yacc);
        else
          dec_unit<R, NT, GROUP, 1>(st, warp, kcl, meta, xaddr, xstep, ds_s, lane, yacc);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // tile groups whose last unit is in this stage: add the warps' sums (warp order) and finish
      const int plo = (n * kDecConsumers + KCc) / KCc - 1;
      const int phi = min(NP - 1, (n * kDecConsumers + kDecConsumers) / KCc - 1);
      for (int pc = plo; pc <= phi; ++pc) {
        if (cur == pc) {
          flush(pc);
          cur = -1;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecConsumers) : "memory");
        const int row0 = 16 * (t0 + pc * RPW);
        const int ntl = min(RPW, T - pc * RPW);
        for (int k = warp; k < FR; k += kDecConsumers) {
          float v = 0.f;
          for (int w = 0; w < kDecConsumers; ++w) {
            // warp w holds part of tile group pc iff one of its units u = w (mod 8) lies in it
            const bool touched = KCc >= kDecConsumers || ((((w - pc * KCc) % kDecConsumers) + kDecConsumers) % kDecConsumers) < KCc;
            if (touched) v += slots[(((pc & 1) * kDecConsumers + w) * FR + k) * 32 + lane];
          }
          if (P.Q == 1) dec_out<NT>(P, v, k, row0, ntl, lane);
          else cbuf[(pc * FR + k) * 32 + lane] = v;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecConsumers) : "memory");
      }
    }
  }

  if (P.Q > 1) {
    // the cluster's CTAs add their tile-group sums in rank order; each finishes a share of them
    cluster_sync_all();
    if (warp < kDecConsumers) {
      for (int pc = (int)((long long)NP * q / P.Q); pc < (int)((long long)NP * (q + 1) / P.Q); ++pc) {
        const int row0 = 16 * (t0 + pc * RPW);
        const int ntl = min(RPW, T - pc * RPW);
        for (int k = warp; k < FR; k += kDecConsumers) {
          const float* src = cbuf + (pc * FR + k) * 32 + lane;
          float v = 0.f;
          for (int rk = 0; rk < P.Q; ++rk) v += ld_dsmem_f32(dsmem_addr(src, (uint32_t)rk));
          dec_out<NT>(P, v, k, row0, ntl, lane);
        }
      }
    }
    cluster_sync_all();
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
// Workspace: [header: device status words (decode at byte 0, prefill at byte 4)][prefill scratch].
constexpr size_t kHeaderBytes = 256;

size_t workspace_header_bytes() { return kHeaderBytes; }
long long max_decode_rows() { return 1LL << 30; }
size_t decode_workspace_bytes(int) { return kHeaderBytes; }

namespace {

struct DecLayout {
  int S, xpitch, mspitch, mzpitch, o_x, o_zero, o_ds, o_ms, o_mz, o_slots, o_cbuf, o_ring, o_bar, smem;
};

// Shared-memory layout for a CTA with up to KCc chunks and NP tile groups; false if it cannot hold
// two stages.
template <int R, int NT, int GROUP>
bool dec_layout(int M, int KCc, int NP, int Q, DecLayout& L) {
  constexpr int NG = kChunk / GROUP;
  constexpr int RPW = dec_rpw(R), FR = RPW * NT * 4;
  auto up = [](int v, int a) { return (v + a - 1) / a * a; };
  L.xpitch = KCc * kChunk * 2 + 16;  // +16 B: ldmatrix rows fall in distinct banks
  int o = 0;
  L.o_x = o;
  o = up(o + M * L.xpitch, 128);
  L.o_zero = o;
  o += 128;
  L.o_ds = o;
  o = up(o + KCc * NG * 16 * 4, 128);
  L.mspitch = KCc * NG * 2;
  L.mzpitch = up(KCc * NG, 4);
  L.o_ms = o;
  o = up(o + NP * RPW * 16 * L.mspitch, 128);
  L.o_mz = o;
  o = up(o + NP * RPW * 16 * L.mzpitch, 128);
  L.o_slots = o;
  o += 2 * kDecConsumers * FR * 32 * 4;
  L.o_cbuf = o;
  if (Q > 1) o += NP * FR * 32 * 4;
  L.o_bar = o;
  o = up(o + (2 * kDecMaxStages + 1) * 8, 1024);
  L.o_ring = o;
  const int room = kDecSmemBudget - o;
  int S = room / dec_stage_bytes(R);
  if (S > kDecMaxStages) S = kDecMaxStages;
  if (S < 2) return false;
  L.S = S;
  L.smem = o + S * dec_stage_bytes(R);
  return true;
}

// Clusters of Q CTAs (with this much shared memory) that can be resident at once, per device.
int max_clusters(const void* kern, int Q, int smem, int sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, int, int>, int> cache;
  const int dev = current_device();
  const auto key = std::make_tuple(dev, kern, Q, smem);
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int n = 0;
  if (Q == 1) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecThreads, smem) != cudaSuccess) per_sm = 0;
    n = per_sm * sms;
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(Q * sms);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = Q;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();  // a failed query is not an error of the call
  std::lock_guard<std::mutex> g(mu);
  cache[key] = n;
  return n;
}

template <int R, int NT, int GROUP>
cudaError_t launch_decode_t(DecodeParams P, int sms, cudaStream_t s) {
  auto kern = decode_kernel<R, NT, GROUP>;
  static std::mutex mu;
  static unsigned long long attr_set = 0;  // devices whose shared-memory attribute is set
  const int dev = current_device();
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev >= 64 || !(attr_set & (1ull << dev))) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemBudget);
      if (e != cudaSuccess) return e;
      if (dev < 64) attr_set |= 1ull << dev;
    }
  }
  // Choose Q (CTAs per cluster splitting K): the smallest per-CTA share of the work
  // (row tiles x chunks, a two-stage ring counted 15% slower) among the layouts that fit, fewer
  // CTAs per cluster on a tie.  None fits when the CTA's activations cannot stay resident even
  // at Q = 8: the caller then takes another path.
  int bestQ = 0, best_ncl = 0;
  long long best_cost = 0;
  DecLayout best{};
  for (int Q = 1; Q <= 8 && Q <= P.KC; Q *= 2) {
    const int KCc = (P.KC + Q - 1) / Q;
    DecLayout L;
    // tile groups per cluster are bounded after the cluster count is known; size for the worst
    int ncl_try = sms / Q;
    if (ncl_try < 1) ncl_try = 1;
    if (ncl_try > P.RT) ncl_try = P.RT;
    int tiles = (P.RT + ncl_try - 1) / ncl_try;
    if (!dec_layout<R, NT, GROUP>(P.M, KCc, (tiles + dec_rpw(R) - 1) / dec_rpw(R), Q, L)) continue;
    int ncl = max_clusters((const void*)kern, Q, L.smem, sms);
    if (ncl < 1) continue;
    if (ncl > P.RT) ncl = P.RT;
    if (ncl != ncl_try) {
      tiles = (P.RT + ncl - 1) / ncl;
      if (!dec_layout<R, NT, GROUP>(P.M, KCc, (tiles + dec_rpw(R) - 1) / dec_rpw(R), Q, L)) continue;
    }
    const long long cost = (long long)tiles * KCc * (L.S >= 3 ? 20 : 23);
    if (bestQ == 0 || cost < best_cost) {
      bestQ = Q;
      best_cost = cost;
      best_ncl = ncl;
      best = L;
    }
  }
  if (bestQ == 0) return cudaErrorNotSupported;
  P.Q = bestQ;
  P.ncl = best_ncl;
  P.S = best.S;
  P.xpitch = best.xpitch;
  P.o_x = best.o_x;
  P.o_zero = best.o_zero;
  P.o_ds = best.o_ds;
  P.o_ms = best.o_ms;
  P.o_mz = best.o_mz;
  P.mspitch = best.mspitch;
  P.mzpitch = best.mzpitch;
  P.o_slots = best.o_slots;
  P.o_cbuf = best.o_cbuf;
  P.o_ring = best.o_ring;
  P.o_bar = best.o_bar;
  return launch_pdl_cluster(kern, dim3(best_ncl * bestQ), dim3(kDecThreads), (size_t)best.smem, bestQ, s, P);
}

template <int NT, int GROUP>
cudaError_t launch_decode_r(int r, const DecodeParams& P, int sms, cudaStream_t s) {
  switch (r) {
    case 2: return launch_decode_t<2, NT, GROUP>(P, sms, s);
    case 3: return launch_decode_t<3, NT, GROUP>(P, sms, s);
    case 4: return launch_decode_t<4, NT, GROUP>(P, sms, s);
    case 6: return launch_decode_t<6, NT, GROUP>(P, sms, s);
    default: return launch_decode_t<8, NT, GROUP>(P, sms, s);
  }
}

}  // namespace

cudaError_t launch_decode(const void* x, int M, int K, const void* planes, const PlaneGeom& g, const uint16_t* scales,
                          const uint8_t* zeros, int r, int group, void* y, int y_mode, void* workspace,
                          cudaStream_t s) {
  const int NT = (M <= 8) ? 1 : 2;
  const int sms = sm_count(current_device());
  DecodeParams P{};
  P.planes = (const uint8_t*)planes;
  for (int p = 0; p < kPlanes; ++p) P.poff[p] = g.off[p];
  P.x = (const uint16_t*)x;
  P.scales = scales;
  P.zeros = zeros;
  P.y = y;
  P.err = (int*)workspace;
  P.N = g.N;
  P.K = K;
  P.KC = g.KC;
  P.RT = g.RT;
  P.G = K / group;
  P.M = M;
  P.y_mode = y_mode;
  if (NT == 1) return group == 64 ? launch_decode_r<1, 64>(r, P, sms, s) : launch_decode_r<1, 128>(r, P, sms, s);
  return group == 64 ? launch_decode_r<2, 64>(r, P, sms, s) : launch_decode_r<2, 128>(r, P, sms, s);
}

}  // namespace matq
