// C ABI of libmatq (declared in include/matq.h): host-side validation and dispatch.
// Every argument error is caught here, before any CUDA call, and returned as a status.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <atomic>
#include <cmath>

#include "../../include/matq.h"
#include "common.cuh"
#include "internal.h"

using namespace matq;

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MATQ_OK;
  g_last_cuda_error = (int)e;
  return MATQ_ECUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool valid_nk(int N, int K) {
  if (N < 1 || K < kChunk || K % kChunk != 0) return false;
  // keep every byte offset and index comfortably inside 64-bit / int ranges
  if ((long long)N * (long long)K > (1LL << 40)) return false;
  if ((long long)((N + 15) / 16) * (K / kChunk) > (1LL << 31) - 1) return false;
  return true;
}

int check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_status(e);
  return major == 10 ? MATQ_OK : MATQ_EDEVICE;
}

size_t packed_bytes(int N, int K, int r_keep) {
  const PlaneGeom g = make_geom(N, K);
  size_t total = 0;
  for (int p = 0; p < planes_for_width(r_keep); ++p) total += (size_t)plane_bytes(g.RT, g.KC, p);
  return total;
}

}  // namespace

namespace matq {
int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// SM count per device, queried once (the attribute cannot change during the process).
int sm_count(int dev) {
  static std::atomic<int> cache[64];
  if (dev < 0 || dev >= 64) {
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    n = 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Status helpers for the other translation units of the C ABI.
int record_cuda_error(cudaError_t e) { return cuda_status(e); }
int check_sm100_device() { return check_device(); }
}  // namespace matq

namespace matq {
size_t linear_workspace_min(int M, int K, int N, int group) {
  if (M < 1 || N < 1 || K < kChunk || K % kChunk || (group != 64 && group != 128)) return 0;
  const size_t dec = decode_workspace_bytes(M <= kDecodeMaxM ? M : kDecodeMaxM);
  if (M <= kDecodeMaxM) return dec;
  const size_t pre = workspace_header_bytes() + prefill_scratch_min_bytes(M, K);
  return pre > dec ? pre : dec;
}
}  // namespace matq

extern "C" {

int matq_version(void) { return 100; }

const char* matq_strerror(int status) {
  switch (status) {
    case MATQ_OK: return "ok";
    case MATQ_EINVAL_R: return "invalid width r (must be 2, 3, 4, 6 or 8)";
    case MATQ_EINVAL_SHAPE: return "invalid shape (N >= 1, M >= 1, K a positive multiple of 256)";
    case MATQ_EINVAL_GROUP: return "invalid group size (must be 64 or 128)";
    case MATQ_EALIGN: return "device pointer not 16-byte aligned";
    case MATQ_ENULL: return "required pointer is NULL";
    case MATQ_ETRUNC: return "pack holds fewer planes than width r needs (r > r_keep)";
    case MATQ_ECUDA: return "CUDA call failed (see matq_last_cuda_error)";
    case MATQ_ESIZE: return "caller buffer too small";
    case MATQ_EDTYPE: return "unknown output mode";
    case MATQ_EDEVICE: return "current device is not an sm_100 (B200-class) GPU";
    case MATQ_ESCRATCH:
      return "sizes need more scratch than matq_linear_noalloc's fixed array (MATQ_NOALLOC_SCRATCH_BYTES); "
             "use matq_linear with a caller workspace";
    case MATQ_EINVAL_ARG: return "invalid argument (a lambda negative or not finite, or an unknown slicing mode)";
    default: return "unknown status";
  }
}

int matq_last_cuda_error(void) { return g_last_cuda_error; }

int matq_plane_count(int r) { return planes_for_width(r); }

size_t matq_packed_bytes(int N, int K, int r_keep) {
  if (!valid_width(r_keep) || !valid_nk(N, K)) return 0;
  return packed_bytes(N, K, r_keep);
}

int matq_pack(const uint8_t* codes, int N, int K, int r_keep, void* planes, size_t planes_bytes, void* stream) {
  if (!valid_width(r_keep)) return MATQ_EINVAL_R;
  if (!valid_nk(N, K)) return MATQ_EINVAL_SHAPE;
  if (!codes || !planes) return MATQ_ENULL;
  if (!aligned16(codes) || !aligned16(planes)) return MATQ_EALIGN;
  if (planes_bytes < packed_bytes(N, K, r_keep)) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_pack(codes, make_geom(N, K), r_keep, planes, (cudaStream_t)stream));
}

int matq_slice(const void* planes, int N, int K, int r_keep, int r, uint8_t* prefix_out, void* stream) {
  if (!valid_width(r) || !valid_width(r_keep)) return MATQ_EINVAL_R;
  if (r > r_keep) return MATQ_ETRUNC;
  if (!valid_nk(N, K)) return MATQ_EINVAL_SHAPE;
  if (!planes || !prefix_out) return MATQ_ENULL;
  if (!aligned16(planes) || !aligned16(prefix_out)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_slice(planes, make_geom(N, K), r, prefix_out, (cudaStream_t)stream));
}

int matq_slice_copy(const void* planes, int N, int K, int r_keep, int r, void* planes_r, size_t bytes,
                    void* stream) {
  if (!valid_width(r) || !valid_width(r_keep)) return MATQ_EINVAL_R;
  if (r > r_keep) return MATQ_ETRUNC;
  if (!valid_nk(N, K)) return MATQ_EINVAL_SHAPE;
  if (!planes || !planes_r) return MATQ_ENULL;
  if (!aligned16(planes) || !aligned16(planes_r)) return MATQ_EALIGN;
  const size_t need = packed_bytes(N, K, r);
  if (bytes < need) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  return cuda_status(cudaMemcpyAsync(planes_r, planes, need, cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
}

size_t matq_linear_workspace(int M, int K, int N, int group) {
  if (M < 1 || N < 1 || K < kChunk || K % kChunk || (group != 64 && group != 128)) return 0;
  // sized so that it also serves every smaller M (decode or prefill) with these K, N
  const size_t dec = decode_workspace_bytes(M <= kDecodeMaxM ? M : kDecodeMaxM);
  if (M <= kDecodeMaxM) return dec;
  const size_t pre = workspace_header_bytes() + prefill_scratch_bytes(M, K, N);
  return pre > dec ? pre : dec;
}


int matq_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return MATQ_ENULL;
  if (!aligned16(workspace)) return MATQ_EALIGN;
  if (ws_bytes < workspace_header_bytes()) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  return cuda_status(cudaMemsetAsync(workspace, 0, workspace_header_bytes(), (cudaStream_t)stream));
}

int matq_workspace_status(const void* workspace, int* status_out) {
  if (!workspace || !status_out) return MATQ_ENULL;
  if (!aligned16(workspace)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  int words[2] = {0, 0};
  cudaError_t e = cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  *status_out = words[0] | words[1];
  return MATQ_OK;
}

int matq_selftest_timeout(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return MATQ_ENULL;
  if (!aligned16(workspace)) return MATQ_EALIGN;
  if (ws_bytes < workspace_header_bytes()) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_wait_selftest((int*)workspace, MATQ_STATUS_SELFTEST, (cudaStream_t)stream));
}

// The sliced linear with the level offset `delta` added to every stored level before the zero
// point: delta_r for true-prefix slices (matq_linear), 0 for packs of rounded levels
// (matq_linear_rounded).
static int linear_with_delta(const void* x, int M, int K, const void* planes, int r_keep, const uint16_t* scales,
                             const uint8_t* zeros, int N, int r, int group, float delta, void* y, int y_mode,
                             void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_width(r) || !valid_width(r_keep)) return MATQ_EINVAL_R;
  if (r > r_keep) return MATQ_ETRUNC;
  if (!valid_nk(N, K) || M < 1 || (long long)M * K > (1LL << 40) || (long long)M * N > (1LL << 40))
    return MATQ_EINVAL_SHAPE;
  if (M <= kDecodeMaxM && (long long)N > max_decode_rows()) return MATQ_EINVAL_SHAPE;
  if (group != 64 && group != 128) return MATQ_EINVAL_GROUP;
  if (y_mode < MATQ_OUT_BF16 || y_mode > MATQ_OUT_SILU_GATED) return MATQ_EDTYPE;
  if (y_mode == MATQ_OUT_SILU_GATED && (N & 1)) return MATQ_EINVAL_SHAPE;
  if (!x || !planes || !scales || !zeros || !y || !workspace) return MATQ_ENULL;
  if (!aligned16(x) || !aligned16(planes) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y) ||
      !aligned16(workspace))
    return MATQ_EALIGN;
  if (ws_bytes < linear_workspace_min(M, K, N, group)) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  const PlaneGeom g = make_geom(N, K);
  cudaError_t e;
  if (M <= kDecodeMaxM)
    e = launch_decode(x, M, K, planes, g, scales, zeros, r, group, delta, y, y_mode, workspace,
                      (cudaStream_t)stream);
  else
    e = launch_prefill(x, M, K, planes, g, scales, zeros, r, group, delta, nullptr, nullptr, y, y_mode, workspace,
                       ws_bytes, (cudaStream_t)stream);
  return cuda_status(e);
}

int matq_linear(const void* x, int M, int K, const void* planes, int r_keep, const uint16_t* scales,
                const uint8_t* zeros, int N, int r, int group, void* y, int y_mode, void* workspace,
                size_t ws_bytes, void* stream) {
  const float delta = valid_width(r) ? (float)((1 << (8 - r)) - 1) * 0.5f : 0.f;
  return linear_with_delta(x, M, K, planes, r_keep, scales, zeros, N, r, group, delta, y, y_mode, workspace,
                           ws_bytes, stream);
}

// ---- rounded slicing: strict and Extra-Precision MatQuant -----------------------------------

namespace {
// The width whose planes hold code bit 7 - r (the bit that rounds the r-bit prefix).
int rounding_width(int r) { return r == 2 ? 3 : r == 3 ? 4 : r == 4 ? 6 : 8; }
size_t round256(size_t b) { return (b + 255) & ~size_t(255); }
}  // namespace

size_t matq_round_scratch_bytes(int N, int K) {
  if (!valid_nk(N, K)) return 0;
  return round256((size_t)N * (size_t)(K / kChunk) * sizeof(int));
}

int matq_round_extract(const void* planes, int N, int K, int r_keep, int r, void* levels, size_t levels_bytes,
                       int32_t* row_ptr, uint16_t* cols, size_t cols_cap, void* scratch, size_t scratch_bytes,
                       void* stream) {
  if (!valid_width(r) || !valid_width(r_keep)) return MATQ_EINVAL_R;
  if (r_keep < rounding_width(r)) return MATQ_ETRUNC;
  if (!valid_nk(N, K) || K > 65536 || (long long)N * K > 0x7FFFFFFFLL) return MATQ_EINVAL_SHAPE;
  if (!planes || !levels || !row_ptr || !scratch) return MATQ_ENULL;
  if (!aligned16(planes) || !aligned16(levels) || !aligned16(row_ptr) || !aligned16(scratch) ||
      (cols && !aligned16(cols)))
    return MATQ_EALIGN;
  if (levels_bytes < packed_bytes(N, K, r) || scratch_bytes < matq_round_scratch_bytes(N, K)) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  const PlaneGeom g = make_geom(N, K);
  return cuda_status(launch_round_extract(planes, g, r, rounding_width(r), levels, (int*)scratch, row_ptr, cols,
                                          (long long)cols_cap, (cudaStream_t)stream));
}

size_t matq_linear_rounded_workspace(int M, int K, int N, int group) {
  const size_t base = matq_linear_workspace(M, K, N, group);
  if (base == 0 || M > kDecodeMaxM) return base;
  return round256(base) + round256((size_t)M * (size_t)N * sizeof(float));
}

int matq_linear_rounded(const void* x, int M, int K, const void* levels, int r, const uint16_t* scales,
                        const uint8_t* zeros, int N, int group, const int32_t* row_ptr, const uint16_t* cols, void* y,
                        int y_mode, void* workspace, size_t ws_bytes, void* stream) {
  if (!valid_width(r)) return MATQ_EINVAL_R;
  if ((row_ptr == nullptr) != (cols == nullptr)) return MATQ_ENULL;
  if (!row_ptr)  // strict MatQuant: the clamped levels alone
    return linear_with_delta(x, M, K, levels, r, scales, zeros, N, r, group, 0.f, y, y_mode, workspace, ws_bytes,
                             stream);
  if (!valid_nk(N, K) || M < 1 || K > 65536 || (long long)M * K > (1LL << 40) || (long long)M * N > (1LL << 40))
    return MATQ_EINVAL_SHAPE;
  if (M <= kDecodeMaxM && (long long)N > max_decode_rows()) return MATQ_EINVAL_SHAPE;
  if (group != 64 && group != 128) return MATQ_EINVAL_GROUP;
  if (y_mode < MATQ_OUT_BF16 || y_mode > MATQ_OUT_SILU_GATED) return MATQ_EDTYPE;
  if (y_mode == MATQ_OUT_SILU_GATED && (N & 1)) return MATQ_EINVAL_SHAPE;
  if (!x || !levels || !scales || !zeros || !y || !workspace) return MATQ_ENULL;
  if (!aligned16(x) || !aligned16(levels) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y) ||
      !aligned16(workspace) || !aligned16(row_ptr) || !aligned16(cols))
    return MATQ_EALIGN;
  if (ws_bytes < matq_linear_rounded_workspace(M, K, N, group)) return MATQ_ESIZE;
  int st = check_device();
  if (st) return st;
  const PlaneGeom g = make_geom(N, K);
  cudaStream_t s = (cudaStream_t)stream;
  if (M > kDecodeMaxM)  // the prefill kernel patches the listed weights into its fp16 tiles
    return cuda_status(launch_prefill(x, M, K, levels, g, scales, zeros, r, group, 0.f, row_ptr, cols, y, y_mode,
                                      workspace, ws_bytes, s));
  // decode: the dense call, then the correction (in place for fp32 outputs; from an fp32 copy
  // of the dense result in the workspace for bf16 and gated outputs)
  const bool in_place = y_mode == MATQ_OUT_F32 || y_mode == MATQ_OUT_F32_ACCUM;
  float* y32 = in_place ? nullptr
                        : (float*)((uint8_t*)workspace + round256(matq_linear_workspace(M, K, N, group)));
  cudaError_t e = launch_decode(x, M, K, levels, g, scales, zeros, r, group, 0.f, in_place ? y : (void*)y32,
                                in_place ? y_mode : MATQ_OUT_F32, workspace, s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_overflow_correct(x, M, K, N, group, r, row_ptr, cols, scales, y32, y, y_mode, s));
}

int matq_rmsnorm(const float* h, int M, int D, float eps, void* n_out, void* stream) {
  if (M < 1 || D < 1 || (long long)M * D > (1LL << 40)) return MATQ_EINVAL_SHAPE;
  if (!h || !n_out) return MATQ_ENULL;
  if (!aligned16(h) || !aligned16(n_out)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_rmsnorm(h, M, D, eps, n_out, (cudaStream_t)stream));
}

int matq_silu_mul_gu(const void* gu, int M, int F, void* a_out, void* stream) {
  if (M < 1 || F < 1 || (long long)M * F > (1LL << 40)) return MATQ_EINVAL_SHAPE;
  if (!gu || !a_out) return MATQ_ENULL;
  if (!aligned16(gu) || !aligned16(a_out)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_silu_mul_gu(gu, M, F, a_out, (cudaStream_t)stream));
}

int matq_choose_codes(const float* w, int N, int K, const uint16_t* scales, const uint8_t* zeros, int group,
                      int n_widths, const int* widths, const float* lambdas, int slice_mode, uint8_t* codes,
                      void* stream) {
  if (group != 64 && group != 128) return MATQ_EINVAL_GROUP;
  if (N < 1 || K < group || K % group != 0 || (long long)N * (long long)K > (1LL << 40)) return MATQ_EINVAL_SHAPE;
  if (!widths || !lambdas) return MATQ_ENULL;
  if (n_widths < 1 || n_widths > 5) return MATQ_EINVAL_R;
  for (int i = 0; i < n_widths; ++i)
    if (!valid_width(widths[i]) || (i > 0 && widths[i] <= widths[i - 1])) return MATQ_EINVAL_R;
  for (int i = 0; i < n_widths; ++i)
    if (!(lambdas[i] >= 0.f) || !std::isfinite(lambdas[i])) return MATQ_EINVAL_ARG;
  if (slice_mode != MATQ_SLICE_TRUE_PREFIX && slice_mode != MATQ_SLICE_TRUNCATE) return MATQ_EINVAL_ARG;
  if (!w || !scales || !zeros || !codes) return MATQ_ENULL;
  if (!aligned16(w) || !aligned16(scales) || !aligned16(zeros) || !aligned16(codes)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_choose(w, N, K, scales, zeros, group, n_widths, widths, lambdas,
                                   slice_mode == MATQ_SLICE_TRUNCATE, codes, (cudaStream_t)stream));
}

int matq_silu_mul(const void* gate, const void* up, int M, int F, void* a_out, void* stream) {
  if (M < 1 || F < 1 || (long long)M * F > (1LL << 40)) return MATQ_EINVAL_SHAPE;
  if (!gate || !up || !a_out) return MATQ_ENULL;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(a_out)) return MATQ_EALIGN;
  int st = check_device();
  if (st) return st;
  return cuda_status(launch_silu_mul(gate, up, M, F, a_out, (cudaStream_t)stream));
}

}  // extern "C"
