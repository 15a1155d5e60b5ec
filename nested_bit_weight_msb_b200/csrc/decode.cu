// Decode path (M <= 16): warp-level streaming skinny GEMM over the packed r-bit planes.
//
// Math (MatGPTQ App. A.1, delta folded into the zero point; MatGPTQ §4, Y = X W_D computed
// as (W_D^T X^T)^T so that weights fill the 16-row MMA operand and tokens the 8-column one):
//
//   y[m, n] = sum_g s[n,g] * ( 2^(8-r) * sum_{k in g} x[m,k] * p[n,k]
//                              + (delta_r - z[n,g]) * sum_{k in g} x[m,k] )
//
// Each warp owns a 16-row tile and a range of 256-input chunks.  It streams the planes of
// width r with 16-byte-per-lane coalesced loads, turns the bits into fp16 MMA operand
// registers in place (a mask-and-or against the fp16 bit pattern of 1024 gives 1024 + p*sigma
// exactly, sigma a power of two fixed by the bit position), and feeds mma.sync m16n8k16 with
// fp32 accumulation.  The per-position factors sigma are split into a per-row factor alpha
// (folded into the group scale) and a per-input factor beta (folded into the activations:
// inputs 8..15 of every 16-input MMA slice are pre-divided by 16 for r <= 4).  The 1024 bias
// is removed per group with the exact sum Bs of the fp16 activation operands, and the zero
// point term uses Sx, the plain per-group sum of x.  Per group, in fp32:
//
//   y += a_row * (D - 1024 * Bs) + s * (delta_r - z) * Sx,   a_row = s * 2^(8-r) / alpha_row
//
// D is the fp32 MMA accumulator of that group.  No weight is ever rounded: the operands are
// exact integers and x's fp16 operand equals x except below 2^-14 (fp16 subnormals).
#include "common.cuh"
#include "internal.h"
#include "operands.cuh"

namespace matq {

// ---- activation preparation ----------------------------------------------------------------
// xfrag[(kt * NT + nt) * 32 + lane] = the m16n8k16 B-operand registers of lane `lane` for
// input tile kt (16 inputs) and token tile nt (8 tokens): {x[t][k0], x[t][k0+1]} and
// {x[t][k0+8], x[t][k0+9]} / beta_hi as fp16 pairs, t = 8*nt + lane/4, k0 = 16*kt + 2*(lane%4).
// xsum[(g * NT*8 + t) * 2 + {0,1}] = {Bs, Sx}: sum over group g of the fp16 operands as used,
// and sum of x.
__device__ __forceinline__ float operand_value(const uint16_t* __restrict__ xrow, int k, float hi_scale) {
  const float v = bf16_bits_to_float(xrow[k]);
  const float sc = ((k & 15) >= 8) ? hi_scale : 1.0f;
  return __half2float(__float2half_rn(v * sc));
}

__global__ void xprep_decode_kernel(const uint16_t* __restrict__ x, int M, int K, int NT, int G, int group,
                                    float hi_scale, uint2* __restrict__ xfrag, float* __restrict__ xsum,
                                    int frag_blocks) {
  if ((int)blockIdx.x < frag_blocks) {
    const int KT = K / 16;
    const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (long long)KT * NT * 32) return;
    const int lane = (int)(e & 31);
    const int nt = (int)((e >> 5) % NT);
    const int kt = (int)((e >> 5) / NT);
    const int t = nt * 8 + (lane >> 2);
    const int k0 = kt * 16 + 2 * (lane & 3);
    uint2 out = make_uint2(0u, 0u);
    if (t < M) {
      const uint16_t* xr = x + (size_t)t * K;
      __half2 lo = __floats2half2_rn(bf16_bits_to_float(xr[k0]), bf16_bits_to_float(xr[k0 + 1]));
      __half2 hi = __floats2half2_rn(bf16_bits_to_float(xr[k0 + 8]) * hi_scale,
                                     bf16_bits_to_float(xr[k0 + 9]) * hi_scale);
      out.x = *reinterpret_cast<uint32_t*>(&lo);
      out.y = *reinterpret_cast<uint32_t*>(&hi);
    }
    xfrag[e] = out;
  } else {
    const int NTOK = NT * 8;
    const int e = (blockIdx.x - frag_blocks) * blockDim.x + threadIdx.x;
    if (e >= G * NTOK) return;
    const int g = e / NTOK, t = e % NTOK;
    float bs = 0.f, sx = 0.f;
    if (t < M) {
      const uint16_t* xr = x + (size_t)t * K;
      for (int k = g * group; k < (g + 1) * group; ++k) {
        bs += operand_value(xr, k, hi_scale);
        sx += bf16_bits_to_float(xr[k]);
      }
    }
    xsum[2 * e] = bs;
    xsum[2 * e + 1] = sx;
  }
}

// ---- the kernel ------------------------------------------------------------------------------
struct DecodeParams {
  const uint8_t* planes;
  PlaneGeom g;
  const uint16_t* scales;
  const uint8_t* zeros;
  int G;
  const uint2* xfrag;
  const float* xsum;
  int M;
  void* y;
  int y_mode;
  int cpw;  // chunks per warp
};

template <int R, int NT, int GROUP>
__global__ void __launch_bounds__(256)
decode_kernel(const DecodeParams P) {
  constexpr int kBlocksPerGroup = GROUP / 32;
  constexpr float kDelta = (float)((1 << (8 - R)) - 1) * 0.5f;
  extern __shared__ float red[];  // [warps][NT*4][32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int gid = lane >> 2, tg = lane & 3;
  const int rt = blockIdx.x;
  const PlaneGeom& g = P.g;
  const int kc0 = warp * P.cpw;
  const int kc1 = min(g.KC, kc0 + P.cpw);

  // per-row promotion factors: a = s * 2^(8-r) / alpha_row
  float amul[2];
  if constexpr (R == 2) { amul[0] = 64.f; amul[1] = 16.f; }
  else if constexpr (R == 3) { amul[0] = amul[1] = 32.f; }
  else if constexpr (R == 4) { amul[0] = amul[1] = 16.f; }
  else { amul[0] = amul[1] = 1.f; }
  const int row0 = rt * kTileRows + gid, row1 = row0 + 8;
  const bool v0 = row0 < g.N, v1 = row1 < g.N;

  float yacc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) yacc[nt][i] = 0.f;

  bool bvalid[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) bvalid[nt] = (nt * 8 + gid) < P.M;

  for (int kc = kc0; kc < kc1; ++kc) {
    LaneWords L;
    load_lane_words<R>(P.planes, g, (size_t)rt * g.KC + kc, lane, L);
    uint2 bfr[16][NT];
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        bfr[i][nt] = bvalid[nt] ? __ldg(&P.xfrag[((size_t)(kc * 16 + i) * NT + nt) * 32 + lane]) : make_uint2(0u, 0u);

    float d[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) d[nt][i] = 0.f;

#define MATQ_BLOCK(W)                                                                  \
    {                                                                                  \
      uint32_t A[2][4];                                                                \
      build_operands<R, W>(L, A);                                                      \
      _Pragma("unroll") for (int j = 0; j < 2; ++j)                                    \
      _Pragma("unroll") for (int nt = 0; nt < NT; ++nt)                                \
        mma_f16(d[nt], A[j], bfr[2 * (W) + j][nt].x, bfr[2 * (W) + j][nt].y);          \
      if (((W) + 1) % kBlocksPerGroup == 0) {                                          \
        const int gi = (kc * kChunk + 32 * ((W) + 1)) / GROUP - 1;                     \
        promote(gi, d);                                                                \
      }                                                                                \
    }
    auto promote = [&](int gi, float (&dd)[NT][4]) {
      float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
      if (v0) {
        const float s = __half2float(__ushort_as_half(P.scales[(size_t)row0 * P.G + gi]));
        a0 = s * amul[0];
        c0 = s * (kDelta - (float)P.zeros[(size_t)row0 * P.G + gi]);
      }
      if (v1) {
        const float s = __half2float(__ushort_as_half(P.scales[(size_t)row1 * P.G + gi]));
        a1 = s * amul[1];
        c1 = s * (kDelta - (float)P.zeros[(size_t)row1 * P.G + gi]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float4 xs = *reinterpret_cast<const float4*>(P.xsum + ((size_t)gi * NT * 8 + nt * 8 + 2 * tg) * 2);
        // xs = {Bs(t0), Sx(t0), Bs(t1), Sx(t1)}
        yacc[nt][0] = fmaf(c0, xs.y, fmaf(a0, fmaf(-1024.f, xs.x, dd[nt][0]), yacc[nt][0]));
        yacc[nt][1] = fmaf(c0, xs.w, fmaf(a0, fmaf(-1024.f, xs.z, dd[nt][1]), yacc[nt][1]));
        yacc[nt][2] = fmaf(c1, xs.y, fmaf(a1, fmaf(-1024.f, xs.x, dd[nt][2]), yacc[nt][2]));
        yacc[nt][3] = fmaf(c1, xs.w, fmaf(a1, fmaf(-1024.f, xs.z, dd[nt][3]), yacc[nt][3]));
#pragma unroll
        for (int i = 0; i < 4; ++i) dd[nt][i] = 0.f;
      }
    };
    MATQ_BLOCK(0) MATQ_BLOCK(1) MATQ_BLOCK(2) MATQ_BLOCK(3)
    MATQ_BLOCK(4) MATQ_BLOCK(5) MATQ_BLOCK(6) MATQ_BLOCK(7)
#undef MATQ_BLOCK
  }

  // reduce the warps' partial sums (fixed order) and store
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[((warp * NT + nt) * 4 + i) * 32 + lane] = yacc[nt][i];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v = 0.f;
        for (int w = 0; w < nwarps; ++w) v += red[((w * NT + nt) * 4 + i) * 32 + lane];
        const int row = (i < 2) ? row0 : row1;
        const int tok = nt * 8 + 2 * tg + (i & 1);
        if (row < g.N && tok < P.M) {
          const size_t o = (size_t)tok * g.N + row;
          if (P.y_mode == 0) reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v);
          else if (P.y_mode == 1) reinterpret_cast<float*>(P.y)[o] = v;
          else reinterpret_cast<float*>(P.y)[o] += v;
        }
      }
  }
}

// ---- host launch ---------------------------------------------------------------------------
size_t decode_workspace_bytes(int M, int K, int group) {
  const int NT = (M <= 8) ? 1 : 2;
  const size_t frag = (size_t)(K / 16) * NT * 32 * sizeof(uint2);
  const size_t sums = (size_t)(K / group) * NT * 8 * 2 * sizeof(float);
  return ((frag + 255) & ~size_t(255)) + ((sums + 255) & ~size_t(255));
}

template <int R, int NT, int GROUP>
static cudaError_t launch_decode_t(const DecodeParams& P, int warps, cudaStream_t s) {
  const size_t smem = (size_t)warps * NT * 4 * 32 * sizeof(float);
  decode_kernel<R, NT, GROUP><<<P.g.RT, warps * 32, smem, s>>>(P);
  return cudaGetLastError();
}

template <int NT, int GROUP>
static cudaError_t launch_decode_r(int r, const DecodeParams& P, int warps, cudaStream_t s) {
  switch (r) {
    case 2: return launch_decode_t<2, NT, GROUP>(P, warps, s);
    case 3: return launch_decode_t<3, NT, GROUP>(P, warps, s);
    case 4: return launch_decode_t<4, NT, GROUP>(P, warps, s);
    case 6: return launch_decode_t<6, NT, GROUP>(P, warps, s);
    default: return launch_decode_t<8, NT, GROUP>(P, warps, s);
  }
}

cudaError_t launch_decode(const void* x, int M, int K, const void* planes, const PlaneGeom& g, const uint16_t* scales,
                          const uint8_t* zeros, int r, int group, void* y, int y_mode, void* workspace,
                          cudaStream_t s) {
  const int NT = (M <= 8) ? 1 : 2;
  const int G = K / group;
  uint8_t* ws = (uint8_t*)workspace;
  const size_t frag = (size_t)(K / 16) * NT * 32 * sizeof(uint2);
  uint2* xfrag = (uint2*)ws;
  float* xsum = (float*)(ws + ((frag + 255) & ~size_t(255)));
  const float hi_scale = (r <= 4) ? 0.0625f : 1.0f;
  {
    const int threads = 256;
    const long long nfrag = (long long)(K / 16) * NT * 32;
    const int fb = (int)((nfrag + threads - 1) / threads);
    const int sb = (G * NT * 8 + threads - 1) / threads;
    xprep_decode_kernel<<<fb + sb, threads, 0, s>>>((const uint16_t*)x, M, K, NT, G, group, hi_scale, xfrag, xsum,
                                                    fb);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  DecodeParams P;
  P.planes = (const uint8_t*)planes;
  P.g = g;
  P.scales = scales;
  P.zeros = zeros;
  P.G = G;
  P.xfrag = xfrag;
  P.xsum = xsum;
  P.M = M;
  P.y = y;
  P.y_mode = y_mode;
  int warps = g.KC >= 8 ? 8 : g.KC;
  P.cpw = (g.KC + warps - 1) / warps;
  warps = (g.KC + P.cpw - 1) / P.cpw;
  if (NT == 1) {
    return group == 64 ? launch_decode_r<1, 64>(r, P, warps, s) : launch_decode_r<1, 128>(r, P, warps, s);
  } else {
    return group == 64 ? launch_decode_r<2, 64>(r, P, warps, s) : launch_decode_r<2, 128>(r, P, warps, s);
  }
}

}  // namespace matq
