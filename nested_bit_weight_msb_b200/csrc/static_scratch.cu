// matq_linear_noalloc: the sliced linear layer with its scratch in a fixed device array that
// belongs to libmatq, for callers that cannot hand the library a workspace (declared in
// include/matq.h, which states the contract).  The kernels are the ones matq_linear launches;
// only where their scratch lives differs.  Nothing here allocates device or host memory.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <mutex>

#include "../../include/matq.h"
#include "common.cuh"
#include "internal.h"

using namespace matq;

namespace {

// Capacity of the library-owned scratch.  It holds the workspace header (status words and
// split-row counters) with the decode path's partial-sum slots for any M <= 16, and the
// prefill path's fp16 copy of x while header + M * K * 2 bytes fit.
constexpr size_t kStaticScratchBytes = MATQ_NOALLOC_SCRATCH_BYTES;

// One instance per device (the module is loaded into each device's context separately).
// Its contents persist from call to call; the header part is cleared by every call.
static __device__ __align__(256) uint8_t g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

struct DeviceScratch {
  bool ready = false;
  void* ptr = nullptr;  // device address of g_scratch on that device
};

std::mutex g_setup_mutex;
DeviceScratch g_devices[kMaxDevices];

// Set-up, once per device, with that device current: look up the device address of the
// array.  Later calls on the device read the cached address.
int scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return MATQ_EDEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceScratch& d = g_devices[dev];
  if (!d.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    if (p == nullptr) return record_cuda_error(cudaErrorInvalidSymbol);
    d.ptr = p;
    d.ready = true;
  }
  *out = d.ptr;
  return MATQ_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" int matq_linear_noalloc(const void* x, int M, int K, const void* planes, int r_keep,
                                   const uint16_t* scales, const uint8_t* zeros, int N, int r, int group,
                                   void* y, int y_mode, int* status_out, void* stream) {
  // matq_linear's argument checks, in its order, made here so that a rejected call launches
  // nothing; then the size check against the fixed capacity.
  if (!valid_width(r) || !valid_width(r_keep)) return MATQ_EINVAL_R;
  if (r > r_keep) return MATQ_ETRUNC;
  const size_t need = linear_workspace_min(M, K, N, group);  // 0 for a bad M, K, N or group
  if (N < 1 || M < 1 || K < kChunk || K % kChunk != 0 || (long long)M * K > (1LL << 40) ||
      (long long)M * N > (1LL << 40) || (long long)N * K > (1LL << 40) ||
      (long long)((N + 15) / 16) * (K / kChunk) > (1LL << 31) - 1)
    return MATQ_EINVAL_SHAPE;
  if (M <= kDecodeMaxM && (long long)N > max_decode_rows()) return MATQ_EINVAL_SHAPE;
  if (group != 64 && group != 128) return MATQ_EINVAL_GROUP;
  if (y_mode < MATQ_OUT_BF16 || y_mode > MATQ_OUT_SILU_GATED) return MATQ_EDTYPE;
  if (y_mode == MATQ_OUT_SILU_GATED && (N & 1)) return MATQ_EINVAL_SHAPE;
  if (!x || !planes || !scales || !zeros || !y) return MATQ_ENULL;
  if (!aligned16(x) || !aligned16(planes) || !aligned16(scales) || !aligned16(zeros) || !aligned16(y) ||
      ((uintptr_t)status_out & 3u))
    return MATQ_EALIGN;
  if (need == 0 || need > kStaticScratchBytes) return MATQ_ESCRATCH;
  int st = check_sm100_device();
  if (st) return st;

  void* ws = nullptr;
  st = scratch_for_current_device(&ws);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // The header must start at zero.  Every completed call leaves it zero, but one whose
  // device-side wait ran out does not, so each call clears it; the rest of the scratch is
  // written before it is read.
  cudaError_t e = cudaMemsetAsync(ws, 0, workspace_header_bytes(), s);
  if (e != cudaSuccess) return record_cuda_error(e);
  st = matq_linear(x, M, K, planes, r_keep, scales, zeros, N, r, group, y, y_mode, ws, kStaticScratchBytes,
                   stream);
  if (st) return st;
  if (status_out) {
    // status word of the path taken: decode at byte 0 of the header, prefill at byte 4
    const uint8_t* word = static_cast<const uint8_t*>(ws) + (M <= kDecodeMaxM ? 0 : 4);
    e = cudaMemcpyAsync(status_out, word, sizeof(int), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return record_cuda_error(e);
  }
  return MATQ_OK;
}
