// Extra-Precision MatQuant on the decode path: the sparse correction of the weights whose
// rounded level is 2^r.
//
// "Matryoshka Quantization | Summary" §7 (Errata): without the clamp after rounding, a width-r
// slice has 2^r + 1 levels; the top one, 2^r, needs one extra bit for the few weights that
// take it.  libmatq stores such a slice as the clamped level (a width-r pack read by the dense
// kernels with level offset 0) plus the list of the weights at 2^r (CSR by row, inputs
// ascending).  A listed weight's value is s * (2^r * 2^(8-r) - z); the dense kernels served
// s * ((2^r - 1) * 2^(8-r) - z), so each listed weight adds s * 2^(8-r) * x[m, k] to y[m, n].
//
// One CTA per block of rows.  Their lists are one contiguous stretch of `cols` (CSR), read in
// tiles of 256 entries: lane l of a warp takes entries 8l .. 8l + 7 of a tile with one 16-byte
// load (coalesced across the warp), so a lane's entries are contiguous and follow its rows
// forward from a binary search in the block's row pointers.  The block's scales and the
// activations (a window of inputs at a time, transposed: input-major, MP tokens per input,
// tokens >= M zero) sit in shared memory.  At the end of a tile a segmented warp sum over
// lanes on the same row leaves one shared-memory atomic add per row run.  After the last
// window the block's sums finish the output: added in place (fp32 modes), or added to the
// dense fp32 result and rounded to bf16, or formed into the SiLU-gated product (row pairs).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>

#include "../../include/matq.h"
#include "common.cuh"
#include "internal.h"
#include "sync.cuh"

namespace matq {

constexpr int kCorrThreads = 256;
constexpr int kCorrWarps = kCorrThreads / 32;
constexpr int kCorrSmem = 160 * 1024;   // activation window + block scales + sums
constexpr int kCorrScaleBytes = 32 * 1024;
constexpr int kSmemPerSM = 228 * 1024;   // shared memory of an SM

struct CorrParams {
  const __nv_bfloat16* x;
  int M, K, N, G, gshift, RPC, KW;
  float step;  // 2^(8-r)
  const int* row_ptr;
  const uint16_t* cols;
  const uint16_t* scales;
  const float* y32;  // dense fp32 result (bf16 and gated outputs); null: y is updated in place
  void* y;
  int y_mode;
};

// The MP staged activations of one input (MP consecutive bf16) as floats: one 16-byte load per
// eight tokens, one 8- or 4-byte load below that.  The window is 16-byte aligned for MP >= 2
// (the sums and row pointers before it fill whole 16-byte units), so every load is aligned.
template <int MP>
__device__ __forceinline__ void load_tokens(const __nv_bfloat16* xr, float (&xv)[MP]) {
  if constexpr (MP == 1) {
    xv[0] = __bfloat162float(xr[0]);
  } else {
    uint32_t u[MP / 2];
    if constexpr (MP >= 8) {
#pragma unroll
      for (int v = 0; v < MP / 8; ++v) {
        const uint4 q = reinterpret_cast<const uint4*>(xr)[v];
        u[4 * v] = q.x;
        u[4 * v + 1] = q.y;
        u[4 * v + 2] = q.z;
        u[4 * v + 3] = q.w;
      }
    } else if constexpr (MP == 4) {
      const uint2 q = *reinterpret_cast<const uint2*>(xr);
      u[0] = q.x;
      u[1] = q.y;
    } else {
      u[0] = *reinterpret_cast<const uint32_t*>(xr);
    }
#pragma unroll
    for (int i = 0; i < MP / 2; ++i) {
      xv[2 * i] = __uint_as_float(u[i] << 16);  // bf16 is the high half of an fp32
      xv[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
}

template <int MP>
__global__ void __launch_bounds__(kCorrThreads) overflow_correct_kernel(const __grid_constant__ CorrParams P) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* acc = reinterpret_cast<float*>(smem);                          // [RPC][MP]
  int* rp = reinterpret_cast<int*>(acc + (size_t)P.RPC * MP);           // [RPC + 1] row pointers
  uint16_t* sc = reinterpret_cast<uint16_t*>(rp + ((P.RPC + 5) & ~3));  // [RPC][G] fp16 scales
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(
      reinterpret_cast<uint8_t*>(sc) + (((size_t)P.RPC * P.G * 2 + 15) & ~size_t(15)));  // [KW][MP]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * P.RPC;
  const int nrows = min(P.RPC, P.N - r0);
  // The next kernel may launch only once this one has done its work (below): launched earlier,
  // a persistent kernel that follows would find the SMs held by this grid's waiting blocks.
  pdl_wait();  // x, the list and the dense result come from earlier kernels
  // The block's entries [E0, E1), from the 8-entry boundary at or below E0, in tiles of 256:
  // lane l of a warp reads entries 8l .. 8l + 7 of a tile with one 16-byte load (the warp's
  // load is one 512-byte run), so a lane's entries are contiguous and its row changes rarely.
  // Warp w takes a contiguous range of tiles.  Entries outside [E0, E1) are skipped (the list
  // is padded to whole 8-entry blocks, so no load leaves it).  Everything the block reads is
  // requested before anything waits: the first kPre tiles of the lane's entries, the row
  // pointers, the scales and the first window of activations.
  const int warp = tid >> 5, lane = tid & 31;
  const int E0 = P.row_ptr[r0], E1 = P.row_ptr[r0 + nrows];
  const int A0 = E0 & ~7;
  const int ntiles = (E1 - A0 + 255) / 256;
  const int tpw = (ntiles + kCorrWarps - 1) / kCorrWarps;
  const int t0 = min(ntiles, warp * tpw), t1 = min(ntiles, t0 + tpw);
  constexpr int kPre = 4;
  const uint4 kNone = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
  uint4 pre[kPre];
#pragma unroll
  for (int u = 0; u < kPre; ++u) {
    const int eb = A0 + (t0 + u) * 256 + 8 * lane;
    pre[u] = (t0 + u < t1 && eb < E1) ? *reinterpret_cast<const uint4*>(P.cols + eb) : kNone;
  }
  for (int i = tid; i < nrows * MP; i += kCorrThreads) acc[i] = 0.f;
  for (int i = tid; i <= nrows; i += kCorrThreads) rp[i] = P.row_ptr[r0 + i];
  {
    // the block's scales: a contiguous run of nrows * G fp16 values; 8 loads in flight a thread
    const uint16_t* src = P.scales + (size_t)r0 * P.G;
    const int n = nrows * P.G;
    for (int i0 = tid; i0 < n; i0 += 8 * kCorrThreads) {
      uint16_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kCorrThreads;
        v[u] = i < n ? src[i] : (uint16_t)0;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kCorrThreads;
        if (i < n) sc[i] = v[u];
      }
    }
  }
  // a window of activations: 16-byte loads (8 inputs of one token; kw and kw0 are multiples of
  // 256), several in flight a thread, scattered into the input-major layout; tokens >= M zero
  auto stage_x = [&](int kw0, int kw) {
    const int nv = kw / 8;
    for (int v0 = tid; v0 < nv * MP; v0 += 4 * kCorrThreads) {
      uint4 val[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * kCorrThreads, m = v / nv, kk = (v - m * nv) * 8;
        val[u] = make_uint4(0u, 0u, 0u, 0u);
        if (v < nv * MP && m < P.M) val[u] = *reinterpret_cast<const uint4*>(P.x + (size_t)m * P.K + kw0 + kk);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * kCorrThreads, m = v / nv, kk = (v - m * nv) * 8;
        if (v < nv * MP) {
          const uint16_t* h = reinterpret_cast<const uint16_t*>(&val[u]);
#pragma unroll
          for (int j = 0; j < 8; ++j) reinterpret_cast<uint16_t*>(xs)[(kk + j) * MP + m] = h[j];
        }
      }
    }
  };
  stage_x(0, min(P.KW, P.K));
  __syncthreads();
  auto row_of = [&](int e) {  // last row whose list starts at or before e
    int lo = 0, hi = nrows - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (rp[mid] <= e) lo = mid;
      else hi = mid - 1;
    }
    return lo;
  };
  const int row_start = row_of(max(E0, A0 + t0 * 256 + 8 * lane));
  for (int kw0 = 0; kw0 < P.K; kw0 += P.KW) {
    const int kw = min(P.KW, P.K - kw0);
    const int kend = kw0 + kw;
    if (kw0 > 0) {
      __syncthreads();  // the previous window is no longer read
      stage_x(kw0, kw);
      __syncthreads();
    }
    int row = row_start, next = rp[row_start + 1];
    for (int t = t0; t < t1; ++t) {
      const int eb = A0 + t * 256 + 8 * lane;
      uint4 raw = kNone;
      if (kw0 == 0 && t - t0 < kPre) {
#pragma unroll
        for (int u = 0; u < kPre; ++u)
          if (t - t0 == u) raw = pre[u];
      } else if (eb < E1) {
        raw = *reinterpret_cast<const uint4*>(P.cols + eb);
      }
      const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
      float a[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) a[m] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = eb + j;
        if (e < E0 || e >= E1) continue;
        const int k = (int)((wv[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
        if (e >= next) {  // a later row: add this lane's sums of the earlier one (rare)
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            if (m < P.M && a[m] != 0.f) atomicAdd(&acc[row * MP + m], a[m]);
            a[m] = 0.f;
          }
          do {
            ++row;
            next = rp[row + 1];
          } while (e >= next);
        }
        if (k >= kw0 && k < kend) {
          const float w = __half2float(__ushort_as_half(sc[row * P.G + (k >> P.gshift)])) * P.step;
          float xv[MP];
          load_tokens<MP>(xs + (size_t)(k - kw0) * MP, xv);
#pragma unroll
          for (int m = 0; m < MP; ++m) a[m] = fmaf(w, xv[m], a[m]);
        }
      }
      // end of the tile: the lanes' current rows are non-decreasing across the warp (a lane
      // past the list's end, whose row is stale, takes a key above every row and adds
      // nothing); a segmented sum over equal keys leaves each run's total in its first lane
      const int key = eb >= E1 ? 0x7fffffff : row;
      const int prev_key = __shfl_up_sync(0xffffffffu, key, 1);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int okey = __shfl_down_sync(0xffffffffu, key, o);
        const bool take = lane + o < 32 && okey == key;
#pragma unroll
        for (int m = 0; m < MP; ++m) {
          const float ov = __shfl_down_sync(0xffffffffu, a[m], o);
          if (take) a[m] += ov;
        }
      }
      if ((lane == 0 || prev_key != key) && key != 0x7fffffff) {
#pragma unroll
        for (int m = 0; m < MP; ++m)
          if (m < P.M && a[m] != 0.f) atomicAdd(&acc[row * MP + m], a[m]);
      }
    }
  }
  __syncthreads();
  if (P.y_mode == MATQ_OUT_SILU_GATED) {
    const int pairs = nrows >> 1, F = P.N >> 1;
    for (int i = tid; i < P.M * pairs; i += kCorrThreads) {
      const int m = i / pairs, pi = i - m * pairs;
      const int n = r0 + 2 * pi;
      const float g = P.y32[(size_t)m * P.N + n] + acc[(2 * pi) * MP + m];
      const float u = P.y32[(size_t)m * P.N + n + 1] + acc[(2 * pi + 1) * MP + m];
      reinterpret_cast<__nv_bfloat16*>(P.y)[(size_t)m * F + (n >> 1)] =
          __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u);
    }
  } else {
    for (int i = tid; i < P.M * nrows; i += kCorrThreads) {
      const int m = i / nrows, rr = i - m * nrows;
      const size_t o = (size_t)m * P.N + r0 + rr;
      if (P.y_mode == MATQ_OUT_BF16)
        reinterpret_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(P.y32[o] + acc[rr * MP + m]);
      else
        reinterpret_cast<float*>(P.y)[o] += acc[rr * MP + m];
    }
  }
  pdl_launch_dependents();
}

// Rows per CTA (even, so that gated row pairs stay together): enough CTAs for one wave of as
// many per SM as fit (four, fewer when the activation window is large: every CTA stages the
// activations, so a CTA more per SM costs another copy of them), at least 16 rows, and the
// block's scales within kCorrScaleBytes.  Window: the rest of the shared memory holds KW
// inputs x MP tokens of bf16 activations.
size_t overflow_correct_smem(int M, int K, int N, int G, int* rpc_out, int* kw_out) {
  const int MP = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
  const int sms = sm_count(current_device());
  const long long cap = kCorrScaleBytes / (2LL * G);
  long long rpc = 0, kw = 0;
  size_t smem = 0;
  auto layout = [&](long long per_sm) {
    rpc = ((long long)N + per_sm * sms - 1) / (per_sm * sms);
    if (rpc > 512) rpc = 512;
    if (rpc > cap) rpc = cap;
    if (rpc < 16) rpc = 16;
    rpc = (rpc + 1) & ~1LL;
    const size_t fixed = (size_t)rpc * MP * 4 + (((size_t)rpc + 5) & ~size_t(3)) * 4 + (((size_t)rpc * G * 2 + 15) & ~size_t(15));
    kw = (((long long)kCorrSmem - (long long)fixed) / (MP * 2)) & ~255LL;  // whole chunks
    if (kw > K) kw = K;
    smem = fixed + (size_t)kw * MP * 2;
  };
  layout(4);
  const long long fit = (long long)kSmemPerSM / (long long)(smem + 1024);  // + the runtime's reserve
  if (fit < 4) layout(fit < 1 ? 1 : fit);
  if (rpc_out) *rpc_out = (int)rpc;
  if (kw_out) *kw_out = (int)kw;
  return smem;
}

template <int MP>
static cudaError_t launch_corr_t(const CorrParams& P, size_t smem, cudaStream_t s) {
  auto kern = overflow_correct_kernel<MP>;
  // the shared-memory attribute (the most any call asks for) is set once per device
  static std::atomic<unsigned long long> attr_set{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(attr_set.load(std::memory_order_relaxed) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kCorrSmem);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit, std::memory_order_relaxed);
  }
  const unsigned grid = (unsigned)((P.N + P.RPC - 1) / P.RPC);
  // a plain launch: with a programmatic one, this grid's blocks would become resident while the
  // dense kernel still runs and wait there, in that kernel's way
  overflow_correct_kernel<MP><<<grid, kCorrThreads, smem, s>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_overflow_correct(const void* x, int M, int K, int N, int group, int r, const int* row_ptr,
                                    const uint16_t* cols, const uint16_t* scales, const float* y32, void* y,
                                    int y_mode, cudaStream_t s) {
  CorrParams P;
  P.x = (const __nv_bfloat16*)x;
  P.M = M;
  P.K = K;
  P.N = N;
  P.G = K / group;
  P.gshift = group == 64 ? 6 : 7;
  P.step = (float)(1 << (8 - r));
  P.row_ptr = row_ptr;
  P.cols = cols;
  P.scales = scales;
  P.y32 = y32;
  P.y = y;
  P.y_mode = y_mode;
  const size_t smem = overflow_correct_smem(M, K, N, P.G, &P.RPC, &P.KW);
  if (M <= 1) return launch_corr_t<1>(P, smem, s);
  if (M <= 2) return launch_corr_t<2>(P, smem, s);
  if (M <= 4) return launch_corr_t<4>(P, smem, s);
  if (M <= 8) return launch_corr_t<8>(P, smem, s);
  return launch_corr_t<16>(P, smem, s);
}

}  // namespace matq
