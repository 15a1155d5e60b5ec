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
// One CTA per block of rows.  The activations are staged in shared memory one window of
// inputs at a time, transposed (input-major, MP tokens per input, tokens >= M zero), so a
// listed weight costs one coalesced read of its column index, one read of its group's scale
// and MP shared-memory values.  A warp takes a row at a time: each lane one listed weight,
// per-lane partial sums over the MP tokens, then a butterfly reduction that leaves the sum of
// token (lane >> (5 - log2 MP)) in lane groups' first lanes.  After the last window the
// row block's sums finish the output: added in place (fp32 modes), or added to the dense fp32
// result and rounded to bf16, or formed into the SiLU-gated product (row pairs).
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
constexpr int kCorrXBytes = 96 * 1024;  // staged activation window

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

template <int MP>
__global__ void __launch_bounds__(kCorrThreads) overflow_correct_kernel(const __grid_constant__ CorrParams P) {
  constexpr int LOGMP = MP == 1 ? 0 : MP == 2 ? 1 : MP == 4 ? 2 : MP == 8 ? 3 : 4;
  extern __shared__ __align__(16) uint8_t smem[];
  float* acc = reinterpret_cast<float*>(smem);                       // [RPC][MP]
  int* cur = reinterpret_cast<int*>(acc + (size_t)P.RPC * MP);       // [RPC] next listed weight
  int* endp = cur + P.RPC;                                           // [RPC] end of the row's list
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(endp + P.RPC);  // [KW][MP]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.x * P.RPC;
  const int nrows = min(P.RPC, P.N - r0);
  pdl_launch_dependents();
  pdl_wait();  // x, the list and the dense result come from earlier kernels
  for (int i = tid; i < nrows * MP; i += kCorrThreads) acc[i] = 0.f;
  for (int i = tid; i < nrows; i += kCorrThreads) {
    cur[i] = P.row_ptr[r0 + i];
    endp[i] = P.row_ptr[r0 + i + 1];
  }
  for (int kw0 = 0; kw0 < P.K; kw0 += P.KW) {
    const int kw = min(P.KW, P.K - kw0);
    const int kend = kw0 + kw;
    __syncthreads();  // the previous window is no longer read; cur / endp / acc are set
    for (int i = tid; i < kw * MP; i += kCorrThreads) {
      const int m = i / kw, kk = i - m * kw;
      xs[kk * MP + m] = m < P.M ? P.x[(size_t)m * P.K + kw0 + kk] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int rr = warp; rr < nrows; rr += kCorrWarps) {
      const int n = r0 + rr;
      int c = cur[rr];
      const int end = endp[rr];
      float a[MP];
#pragma unroll
      for (int m = 0; m < MP; ++m) a[m] = 0.f;
      while (c < end) {
        const int e = c + lane;
        const int k = e < end ? (int)P.cols[e] : 0x7fffffff;
        const bool v = k < kend;
        const unsigned bal = __ballot_sync(0xffffffffu, v);
        if (v) {
          const float w = __half2float(__ushort_as_half(P.scales[(size_t)n * P.G + (k >> P.gshift)])) * P.step;
          const __nv_bfloat16* xr = xs + (size_t)(k - kw0) * MP;
#pragma unroll
          for (int m = 0; m < MP; ++m) a[m] = fmaf(w, __bfloat162float(xr[m]), a[m]);
        }
        const int nv = __popc(bal);
        c += nv;
        if (nv < 32) break;
      }
      // butterfly: after step o the lane keeps the half of its values selected by bit o
      int nvals = MP;
#pragma unroll
      for (int o = 16; o >= 32 / MP && nvals > 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
        const int h = nvals / 2;
#pragma unroll
        for (int i = 0; i < MP / 2; ++i) {
          if (i < h) {
            const float send = upper ? a[i] : a[i + h];
            const float keep = upper ? a[i + h] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        nvals = h;
      }
#pragma unroll
      for (int o = (32 >> LOGMP) / 2; o >= 1; o >>= 1) a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
      const int tok = lane >> (5 - LOGMP);
      if ((lane & ((32 >> LOGMP) - 1)) == 0) acc[rr * MP + tok] += a[0];
      if (lane == 0) cur[rr] = c;
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
}

size_t overflow_correct_smem(int M, int K, int N, int* rpc_out, int* kw_out) {
  const int MP = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
  const int sms = sm_count(current_device());
  long long rpc = ((long long)N + 2LL * sms - 1) / (2LL * sms);
  rpc = rpc < 128 ? 128 : rpc > 512 ? 512 : rpc;
  rpc = (rpc + 1) & ~1LL;  // even: the gated output pairs rows 2i, 2i + 1
  int kw = kCorrXBytes / (MP * 2);
  if (kw > K) kw = K;
  if (rpc_out) *rpc_out = (int)rpc;
  if (kw_out) *kw_out = kw;
  return (size_t)rpc * (MP * 4 + 8) + (size_t)kw * MP * 2;
}

template <int MP>
static cudaError_t launch_corr_t(const CorrParams& P, size_t smem, cudaStream_t s) {
  auto kern = overflow_correct_kernel<MP>;
  // the shared-memory attribute (set to the largest size any call can ask for) is set once per
  // device for this kernel
  static std::atomic<unsigned long long> attr_set{0};
  const int dev = current_device();
  const unsigned long long bit = 1ull << (dev & 63);
  if (dev >= 64 || !(attr_set.load(std::memory_order_relaxed) & bit)) {
    const int most = 512 * (MP * 4 + 8) + kCorrXBytes;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit, std::memory_order_relaxed);
  }
  const unsigned grid = (unsigned)((P.N + P.RPC - 1) / P.RPC);
  return launch_pdl(kern, dim3(grid), dim3(kCorrThreads), smem, s, P);
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
  const size_t smem = overflow_correct_smem(M, K, N, &P.RPC, &P.KW);
  if (M <= 1) return launch_corr_t<1>(P, smem, s);
  if (M <= 2) return launch_corr_t<2>(P, smem, s);
  if (M <= 4) return launch_corr_t<4>(P, smem, s);
  if (M <= 8) return launch_corr_t<8>(P, smem, s);
  return launch_corr_t<16>(P, smem, s);
}

}  // namespace matq
