// Glue of the Mix'n'Match FFN stack ("Matryoshka Quantization | Summary" §4.3, MatGPTQ §5.4):
// unit-gain RMSNorm in front of the gate/up projections and the SiLU-gated product between
// the two FFN halves.  The pages give no block formula; the reading taken is the Llama-style
// block h <- h + down(silu(gate(n)) * up(n)), n = h / sqrt(mean(h^2) + eps).  Both kernels
// are HBM-bound elementwise passes with fp32 arithmetic and bf16 outputs.
#include "common.cuh"
#include "internal.h"
#include "sync.cuh"

namespace matq {

// One block per row.  Rows of D <= kHeld * 4 * 256 values with D % 4 == 0 are read once with
// 16-byte loads and kept in registers between the sum of squares and the scaling; others take
// two scalar passes.
constexpr int kRmsHeld = 8;
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ h, int D, float eps,
                                                      __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x;
  const float* hr = h + (size_t)row * D;
  __nv_bfloat16* orow = out + (size_t)row * D;
  const bool held = (D & 3) == 0 && D <= kRmsHeld * 4 * 256;
  float4 v[kRmsHeld];
  float ss = 0.f;
  if (held) {
#pragma unroll
    for (int u = 0; u < kRmsHeld; ++u) {
      const int i = threadIdx.x + u * 256;
      v[u] = i < D / 4 ? reinterpret_cast<const float4*>(hr)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kRmsHeld; ++u)
      ss = fmaf(v[u].x, v[u].x, fmaf(v[u].y, v[u].y, fmaf(v[u].z, v[u].z, fmaf(v[u].w, v[u].w, ss))));
  } else {
    for (int i = threadIdx.x; i < D; i += blockDim.x) ss = fmaf(hr[i], hr[i], ss);
  }
  __shared__ float part[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
  const float inv = rsqrtf(tot / (float)D + eps);
  if (held) {
#pragma unroll
    for (int u = 0; u < kRmsHeld; ++u) {
      const int i = threadIdx.x + u * 256;
      if (i < D / 4) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v[u].x * inv, v[u].y * inv);
        const __nv_bfloat162 b = __floats2bfloat162_rn(v[u].z * inv, v[u].w * inv);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t*>(&a);
        o.y = *reinterpret_cast<const uint32_t*>(&b);
        reinterpret_cast<uint2*>(orow)[i] = o;
      }
    }
  } else {
    for (int i = threadIdx.x; i < D; i += blockDim.x) orow[i] = __float2bfloat16_rn(hr[i] * inv);
  }
}

__device__ __forceinline__ float silu_f(float t) { return t / (1.0f + expf(-t)); }

__global__ void __launch_bounds__(256) silu_mul_kernel(const __nv_bfloat16* __restrict__ gate,
                                                       const __nv_bfloat16* __restrict__ up, size_t n,
                                                       __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t nvec = n / 8;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t v = (size_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += stride) {
    const uint4 g4 = reinterpret_cast<const uint4*>(gate)[v];
    const uint4 u4 = reinterpret_cast<const uint4*>(up)[v];
    const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&g4);
    const __nv_bfloat16* ub = reinterpret_cast<const __nv_bfloat16*>(&u4);
    uint4 o4;
    __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o4);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      ob[i] = __float2bfloat16_rn(silu_f(__bfloat162float(gb[i])) * __bfloat162float(ub[i]));
    reinterpret_cast<uint4*>(out)[v] = o4;
  }
  // scalar tail
  const size_t tail0 = nvec * 8;
  for (size_t i = tail0 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = __float2bfloat16_rn(silu_f(__bfloat162float(gate[i])) * __bfloat162float(up[i]));
}

// Same product for the output of one fused gate+up projection: gu [M, 2F], row m holding
// gate in columns 0..F-1 and up in F..2F-1; out [M, F].  Vector path needs F % 8 == 0.
__global__ void __launch_bounds__(256) silu_mul_gu_kernel(const __nv_bfloat16* __restrict__ gu, int M, int F,
                                                          __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  const int stride = gridDim.x * blockDim.x;
  for (int m = blockIdx.y; m < M; m += gridDim.y) {
    const __nv_bfloat16* g = gu + (size_t)m * 2 * F;
    const __nv_bfloat16* u = g + F;
    __nv_bfloat16* o = out + (size_t)m * F;
    if ((F & 7) == 0) {
      for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < F / 8; v += stride) {
        const uint4 g4 = reinterpret_cast<const uint4*>(g)[v];
        const uint4 u4 = reinterpret_cast<const uint4*>(u)[v];
        const __nv_bfloat16* gb = reinterpret_cast<const __nv_bfloat16*>(&g4);
        const __nv_bfloat16* ub = reinterpret_cast<const __nv_bfloat16*>(&u4);
        uint4 o4;
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(&o4);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          ob[i] = __float2bfloat16_rn(silu_f(__bfloat162float(gb[i])) * __bfloat162float(ub[i]));
        reinterpret_cast<uint4*>(o)[v] = o4;
      }
    } else {
      for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < F; i += stride)
        o[i] = __float2bfloat16_rn(silu_f(__bfloat162float(g[i])) * __bfloat162float(u[i]));
    }
  }
}

cudaError_t launch_rmsnorm(const float* h, int M, int D, float eps, void* out, cudaStream_t s) {
  return launch_pdl(rmsnorm_kernel, dim3(M), dim3(256), 0, s, h, D, eps, (__nv_bfloat16*)out);
}

cudaError_t launch_silu_mul(const void* gate, const void* up, int M, int F, void* out, cudaStream_t s) {
  const size_t n = (size_t)M * F;
  const size_t nvec = (n + 7) / 8;
  int blocks = (int)((nvec + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(silu_mul_kernel, dim3(blocks), dim3(256), 0, s, (const __nv_bfloat16*)gate,
                    (const __nv_bfloat16*)up, n, (__nv_bfloat16*)out);
}

}  // namespace matq

namespace matq {
cudaError_t launch_silu_mul_gu(const void* gu, int M, int F, void* out, cudaStream_t s) {
  const int per_row = ((F & 7) == 0 ? F / 8 : F);
  int bx = (per_row + 255) / 256;
  if (bx > 148 * 4) bx = 148 * 4;
  if (bx < 1) bx = 1;
  int by = M < 65535 ? M : 65535;
  // keep the grid near a few waves of the SMs
  while (by > 1 && (long long)bx * by > 148 * 16) by = (by + 1) / 2;
  return launch_pdl(silu_mul_gu_kernel, dim3(bx, by), dim3(256), 0, s, (const __nv_bfloat16*)gu, M, F,
                    (__nv_bfloat16*)out);
}
}  // namespace matq
