// ssm_internal.h -- launch interface between the C ABI and the CUDA kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ssm.h"

namespace ssm {

// Element strides of every strided tensor (already resolved from the ABI's
// "0 = dense" convention).
struct Strides {
  int64_t x_tok, x_seq, z_tok, z_seq, y_tok, y_seq;
  int64_t bc_tok, bc_seq, dt_seq;
};

// Arguments of both modes. For decode, L is 1 and the *_in / *_out cache
// pointers are the same in-out buffers.
struct KernelArgs {
  const void* x;
  const void* z;
  const float* B;
  const float* C;
  const float* dt_raw;
  const float* conv_w;
  const float* conv_b;
  const float* w_dt;
  const float* dt_bias;
  const float* A_log;
  const float* D;
  const void* conv_cache_in;
  const float* ssm_state_in;
  void* y;
  void* conv_cache_out;
  float* ssm_state_out;
  int64_t batch, L, E;
  Strides s;
  float dt_min, dt_max;
  int decay_path;  // prefill: 0 = powers of one exponential where A_n = (n+1) A_0, 1 = one exponential per state
  int* err;        // device error word: a kernel whose bounded wait gave up writes a code here
};

// Prefill launch shape: kernel 3 (pipelined state slices, register budget of
// three CTAs per SM), kernel 4 (the same at two CTAs per SM) or kernel 5 (the
// state slices and the per-token work in separate warps of one CTA).
struct PrefillShape {
  int kernel;
};

// per_state: every CTA will run per-state exponentials (ZOH, or per-state
// decays forced), as opposed to the per-CTA choice of the auto decay path.
PrefillShape choose_prefill_shape(int64_t batch, int64_t E, int64_t L, int num_sms, bool per_state);
bool prefill_shape_supported(PrefillShape sh);
// pdl: overlap the launch with the kernel before it on the stream (that must
// be a kernel, not a copy or memset); the kernel reads its inputs only after
// that kernel has finished.
cudaError_t launch_prefill(const KernelArgs& a, bool io_bf16, bool zoh, PrefillShape sh, cudaStream_t st,
                           bool pdl = false);
cudaError_t launch_decode(const KernelArgs& a, bool io_bf16, bool zoh, cudaStream_t st);

// C[M][N] = A[M][K] . B[N][K]^T, bf16 operands and output, fp32 accumulation,
// on the tensor cores (gemm.cu). K and N multiples of 8, pointers 16-byte
// aligned. ws: gemm_workspace_bytes() of device scratch (the counters of tiles
// cut between CTA pairs, first, then their fp32 partials; 0 bytes when none is
// cut). The counters must be zero on entry and are zero again after a launch
// that completed: counters_zeroed skips the memset that ensures it. pdl: the
// launch may overlap the kernel before it on the stream (programmatic
// dependent launch), which must be a kernel, not a copy or memset.
cudaError_t gemm_bf16_tn(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K, void* ws,
                         size_t ws_bytes, int num_sms, int* err, cudaStream_t st, bool pdl = false,
                         bool counters_zeroed = false);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
size_t gemm_counter_bytes(int64_t M, int64_t N, int64_t K, int num_sms);  // leading part of the workspace

// Shared by the entry points (ssm_api.cu): validation with the ABI's
// "0 = dense" stride defaults, and the calling thread's last-error message.
ssm_status check_dims(const ssm_dims* d, bool prefill, Strides* s);
ssm_status check_weights(const ssm_weights* w);
ssm_status check_prefill_caches(const void* conv_cache_in, const float* ssm_state_in, const void* conv_cache_out,
                                const float* ssm_state_out);
// ssm_prefill_ex with the launch overlapped with the kernel before it (pdl, as
// for launch_prefill); the block forward's core step.
ssm_status prefill_entry(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                         const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                         void* y, void* conv_cache_out, float* ssm_state_out, const ssm_tuning* tuning, bool pdl,
                         void* stream);
bool aligned(const void* p, size_t a);
ssm_status fail(ssm_status st, const char* fmt, ...);
int* device_error_ptr();  // the device error word of the current device

}  // namespace ssm
