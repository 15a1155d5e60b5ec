// Parent-code choice for several widths at once ("MatGPTQ: Efficient and Accurate Inference over
// Nested Quantized Models", §3.2 item 2; App. A.2, Algorithm 2, quant_MatGPTQ).  Every weight w
// takes the code q in [0, 255] that minimises
//     total(q) = sum_i lambda_i * (w - s * (q_hat_{r_i}(q) - z))^2
// over the caller's widths r_0 < r_1 < ... (shared group scale s and zero point z), in fp32
// with every operation rounded on its own and the terms added in width order; on a tie the
// smallest code wins.  The page scores all 256 candidates.  This kernel compares the same fp32
// totals but forms few of them, using two facts that hold whenever s > 0:
//   * q_hat_r(q) depends on q only through its r-bit prefix, so inside a "cell" (the codes that
//     share the prefix of the second-finest width) every term but the finest one is the same
//     number S, and total = fl(S + t_f);
//   * t_f depends on the finest width's prefix p only, through w_hat = s*(q_hat - z), which is
//     exact in fp32 and increases with p.  fl(w - w_hat), its square, the product with lambda
//     and fl(S + .) are monotone, so total(p) falls and then rises across a cell: its minimum
//     lies next to the fp32 estimate of the nearest level, and the codes that tie it form one
//     run, whose first code a short walk to the left finds.
// Cells are skipped when a partial sum already exceeds the best total (later terms are >= 0 and
// so is every rounded sum of them).  Inputs outside the range where these bounds hold (s <= 0,
// non-finite values, |w| > 1e6 or lambda > 1e20) take the literal 256-candidate scan, whose
// NaN handling is argmin's: the first NaN if there is one, else the first minimum.
#include "common.cuh"
#include "internal.h"

namespace matq {

struct ChooseParams {
  const float* w;
  const __half* scales;
  const uint8_t* zeros;
  uint8_t* codes;
  int N, K, G, gshift, nw, fast;
  int r[5];
  float lam[5];
  float delta[5];  // reconstruction offset of each width (0 for raw truncation)
  float cell[5];   // 2^(8 - r): code distance between two levels of a width
};

// lambda * (w - w_hat)^2 with e, e*e, the product and (by the caller) the sum each rounded on
// their own; w_hat must be the exact s * (q_hat - z).
__device__ __forceinline__ float choice_err(float w, float w_hat, float lam) {
  const float e = __fsub_rn(w, w_hat);
  return __fmul_rn(lam, __fmul_rn(e, e));
}

// The literal definition: all 256 candidates, argmin's first NaN or first minimum.
__device__ __noinline__ uint8_t choose_scan(float w, float s, float z, const ChooseParams& P) {
  int best_q = 0;
  float best = 0.f;
  for (int q = 0; q < 256; ++q) {
    float tot = 0.f;
    for (int i = 0; i < P.nw; ++i) {
      const int sh = 8 - P.r[i];
      const float v = __fadd_rn((float)((q >> sh) << sh), P.delta[i]);
      const float t = choice_err(w, __fmul_rn(s, __fsub_rn(v, z)), P.lam[i]);
      tot = i == 0 ? t : __fadd_rn(tot, t);
    }
    if (q == 0) {
      best = tot;
    } else if (!isnan(best) && (isnan(tot) || tot < best)) {
      best = tot;
      best_q = q;
    }
  }
  return (uint8_t)best_q;
}

// The cell search for NW widths (0 < s <= 65504, |w| <= 1e6, lambdas <= 1e20: every total is
// finite).  Level p of width i has w_hat = p * step_i + base_i with step_i = s * 2^(8 - r_i)
// and base_i = s * (delta_i - z); both are exact products, and so is the fused p*step + base
// (the result, s times a half-integer below 256, needs at most 21 significant bits), so w_hat
// equals the definition's s * (q_hat - z) exactly.
template <int NW>
__device__ __forceinline__ uint8_t choose_cells(float w, float s, float z, const ChooseParams& P) {
  float step[NW], base[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    step[i] = __fmul_rn(s, P.cell[i]);
    base[i] = __fmul_rn(s, __fsub_rn(P.delta[i], z));
  }
  auto term = [&](int i, float pf) { return choice_err(w, fmaf(pf, step[i], base[i]), P.lam[i]); };
  constexpr int F = NW - 1;                      // finest width
  const int rf = P.r[F];
  const int rc = NW >= 2 ? P.r[NW - 2] : 0;      // cell width (second finest)
  const int per_cell = 1 << (rf - rc);           // finest levels in a cell
  const int nf = 1 << rf;
  // estimate of the finest level nearest to w (a hint: the search window surrounds it)
  const float uf = fminf(fmaxf(__fdividef(__fsub_rn(w, base[F]), step[F]), -4.f), (float)(nf + 3));
  const int pu = __float2int_rn(uf);

  float best = INFINITY;
  int best_p = nf;  // finest level of the best code (code = level << (8 - rf))
  // minimum over the cell whose finest levels are lo .. lo + per_cell - 1, partial sum S
  auto cell = [&](int lo, float S) {
    const int hi = lo + per_cell - 1;
    // the minimum over all levels is at p* or p* + 1 (p* the last level with w_hat <= w), and
    // the estimate pu is one of the two: the levels next to it (clamped to the cell) hold it
    const int pc = min(max(pu, lo), hi);
    const int a = max(lo, pc - 1), b = min(hi, pc + 1);
    auto total = [&](float pf) {
      const float t = term(F, pf);
      return NW >= 2 ? __fadd_rn(S, t) : t;
    };
    float pf = (float)a;
    float m = total(pf);
    int pm = a;
    for (int p = a + 1; p <= b; ++p) {
      pf += 1.f;
      const float x = total(pf);
      if (x < m) {
        m = x;
        pm = p;
      }
    }
    for (float pl = (float)(pm - 1); pm > lo && total(pl) == m; pl -= 1.f) --pm;
    if (m < best || (m == best && pm < best_p)) {
      best = m;
      best_p = pm;
    }
  };
  if constexpr (NW == 1) {
    cell(0, 0.f);
  } else {
    const int r0 = P.r[0];
    const int sub = 1 << (rc - r0);              // cells under one coarsest level
    auto partial = [&](int c, float t0) {        // sum over the widths before the finest
      float S = t0;
#pragma unroll
      for (int i = 1; i < NW - 1; ++i) S = __fadd_rn(S, term(i, (float)(c >> (rc - P.r[i]))));
      return S;
    };
    // the cell of the nearest finest level first: it usually holds the answer and prunes the rest
    const int c0 = min(max(pu, 0), nf - 1) >> (rf - rc);
    cell(c0 * per_cell, partial(c0, term(0, (float)(c0 >> (rc - r0)))));
    // Coarsest levels outward from the one holding c0.  t0, a lower bound of every total under
    // its level, falls up to the level p0* (the last with w_hat <= w) and rises after p0* + 1;
    // the estimate f0 is within one of p0*, so past f0 + 1 to the right and f0 - 1 to the left
    // a level that fails its bound is followed only by levels that fail it too.
    const int n0 = 1 << r0;
    const int f0 = (int)floorf(fminf(fmaxf(__fdividef(__fsub_rn(w, base[0]), step[0]), -4.f), (float)(n0 + 3)));
    auto level = [&](int p0, bool right) {      // true: the bound rules the level out
      const float t0 = term(0, (float)p0);
      if (t0 > best || (right && t0 == best && p0 * sub * per_cell > best_p)) return true;
      for (int c = p0 * sub; c < (p0 + 1) * sub; ++c) {
        if (c == c0) continue;
        const float S = partial(c, t0);
        if (S > best || (S == best && c * per_cell > best_p)) continue;
        cell(c * per_cell, S);
      }
      return false;
    };
    const int p0c = c0 >> (rc - r0);
    for (int p0 = p0c; p0 < n0; ++p0)
      if (level(p0, true) && p0 >= f0 + 2) break;
    for (int p0 = p0c - 1; p0 >= 0; --p0)
      if (level(p0, false) && p0 <= f0 - 1) break;
  }
  return (uint8_t)(best_p << (8 - rf));
}

template <int NW>
__device__ __forceinline__ uint8_t choose_one(float w, float s, float z, const ChooseParams& P) {
  const bool fast = P.fast && s > 0.f && s <= 65504.f && fabsf(w) <= 1e6f;  // NaN w fails the test
  return fast ? choose_cells<NW>(w, s, z, P) : choose_scan(w, s, z, P);
}

// One block strides over rows; a thread takes one weight of the row at a time.
template <int NW>
__global__ void __launch_bounds__(256) choose_kernel(const __grid_constant__ ChooseParams P) {
  for (int row = blockIdx.x; row < P.N; row += gridDim.x) {
    const size_t r0 = (size_t)row * P.K, g0 = (size_t)row * P.G;
    for (int k = threadIdx.x; k < P.K; k += blockDim.x) {
      const size_t g = g0 + (k >> P.gshift);
      P.codes[r0 + k] = choose_one<NW>(P.w[r0 + k], __half2float(P.scales[g]), (float)P.zeros[g], P);
    }
  }
}

cudaError_t launch_choose(const float* w, int N, int K, const uint16_t* scales, const uint8_t* zeros, int group,
                          int n_widths, const int* widths, const float* lambdas, int truncate, uint8_t* codes,
                          cudaStream_t s) {
  ChooseParams P{};
  P.w = w;
  P.scales = reinterpret_cast<const __half*>(scales);
  P.zeros = zeros;
  P.codes = codes;
  P.N = N;
  P.K = K;
  P.G = K / group;
  P.gshift = group == 64 ? 6 : 7;
  P.nw = n_widths;
  P.fast = 1;
  for (int i = 0; i < n_widths; ++i) {
    P.r[i] = widths[i];
    P.lam[i] = lambdas[i];
    P.delta[i] = truncate ? 0.f : (float)((1 << (8 - widths[i])) - 1) * 0.5f;
    P.cell[i] = (float)(1 << (8 - widths[i]));
    if (!(lambdas[i] <= 1e20f)) P.fast = 0;
  }
  const int dev = current_device();
  const int blocks = N < sm_count(dev) * 8 ? N : sm_count(dev) * 8;
  switch (n_widths) {
    case 1: choose_kernel<1><<<blocks, 256, 0, s>>>(P); break;
    case 2: choose_kernel<2><<<blocks, 256, 0, s>>>(P); break;
    case 3: choose_kernel<3><<<blocks, 256, 0, s>>>(P); break;
    case 4: choose_kernel<4><<<blocks, 256, 0, s>>>(P); break;
    default: choose_kernel<5><<<blocks, 256, 0, s>>>(P); break;
  }
  return cudaGetLastError();
}

}  // namespace matq
