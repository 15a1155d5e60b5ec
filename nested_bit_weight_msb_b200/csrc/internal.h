// Launchers shared between libmatq's translation units (not part of the public ABI).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include "common.cuh"

namespace matq {

cudaError_t launch_pack(const uint8_t* codes, const PlaneGeom& g, int r_keep, void* planes, cudaStream_t s);
cudaError_t launch_slice(const void* planes, const PlaneGeom& g, int r, uint8_t* out, cudaStream_t s);

// Workspace = [header: device error words + split-row-group counters; zero-filled once by the
// caller, left zero by every call][scratch of the path taken].
size_t workspace_header_bytes();
long long max_decode_rows();
size_t decode_workspace_bytes(int M);  // header included
// Bounded-wait self-test: a kernel whose wait runs out ORs `code` into *err and returns.
cudaError_t launch_wait_selftest(int* err, int code, cudaStream_t s);
cudaError_t launch_decode(const void* x, int M, int K, const void* planes, const PlaneGeom& g,
                          const uint16_t* scales, const uint8_t* zeros, int r, int group, float delta, void* y,
                          int y_mode, void* workspace, cudaStream_t s);

size_t prefill_scratch_bytes(int M, int K, int N);  // after the header, K-split partial sums included
size_t prefill_scratch_min_bytes(int M, int K);      // after the header, without them
int prefill_splits(int M, int K, int N);            // K splits of a prefill call (1: none)
cudaError_t launch_prefill(const void* x, int M, int K, const void* planes, const PlaneGeom& g,
                           const uint16_t* scales, const uint8_t* zeros, int r, int group, float delta,
                           const int* ovf_row_ptr, const uint16_t* ovf_cols, void* y, int y_mode, void* workspace,
                           size_t ws_bytes, cudaStream_t s);
// Smallest workspace a matq_linear call accepts (a prefill call then runs without K splits).
size_t linear_workspace_min(int M, int K, int N, int group);

// Rounded slicing (strict / Extra-Precision MatQuant): the clamped-level pack of width r from
// a pack holding width r_in's planes, per-(row, chunk) counts in cnt (N * KC ints, replaced by
// their exclusive prefix sum), row_ptr [N + 1], and (if cols) the listed inputs.
cudaError_t launch_round_extract(const void* planes, const PlaneGeom& g, int r, int r_in, void* levels, int* cnt,
                                 int* row_ptr, uint16_t* cols, long long cols_cap, cudaStream_t s);
// Decode-path correction of the weights listed at level 2^r (see rounded.cu).
cudaError_t launch_overflow_correct(const void* x, int M, int K, int N, int group, int r, const int* row_ptr,
                                    const uint16_t* cols, const uint16_t* scales, const float* y32, void* y,
                                    int y_mode, cudaStream_t s);

cudaError_t launch_rmsnorm(const float* h, int M, int D, float eps, void* out, cudaStream_t s);
cudaError_t launch_silu_mul(const void* gate, const void* up, int M, int F, void* out, cudaStream_t s);
cudaError_t launch_silu_mul_gu(const void* gu, int M, int F, void* out, cudaStream_t s);
cudaError_t launch_choose(const float* w, int N, int K, const uint16_t* scales, const uint8_t* zeros, int group,
                          int n_widths, const int* widths, const float* lambdas, int truncate, uint8_t* codes,
                          cudaStream_t s);

// Host-side per-device caches (api.cu): the SM count of the current device, and the device
// index with which a launcher records that a kernel's shared-memory attribute is set.
int current_device();
int sm_count(int dev);

// C-ABI status helpers (api.cu): record a failed CUDA call as the thread's last CUDA error and
// return MATQ_ECUDA; check that the current device is an sm_100 part.
int record_cuda_error(cudaError_t e);
int check_sm100_device();

// Largest M served by the decode (mma.sync streaming) path; larger M takes the prefill path.
constexpr int kDecodeMaxM = 16;

}  // namespace matq
