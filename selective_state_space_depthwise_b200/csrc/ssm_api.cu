// ssm_api.cu -- the extern "C" boundary declared in include/ssm.h.
//
// Host-side only: argument checks, stride resolution, launch-shape choice and
// one kernel launch per call on the caller's stream. No device memory is
// allocated and no host synchronisation happens on the compute entry points.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "sm100_ptx.cuh"
#include "ssm.h"
#include "ssm_internal.h"

namespace {
thread_local char g_last_error[512] = "";
}  // namespace

namespace ssm {

ssm_status fail(ssm_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

// Checks shared by both modes. `prefill` selects the dense stride defaults.
ssm_status check_dims(const ssm_dims* d, bool prefill, ssm::Strides* s) {
  if (!d) return fail(SSM_ERR_INVALID_ARG, "dims is NULL");
  if (d->d_state != 16) return fail(SSM_ERR_UNSUPPORTED, "d_state=%d: only 16 is built", d->d_state);
  if (d->d_conv != 4) return fail(SSM_ERR_UNSUPPORTED, "d_conv=%d: only 4 is built", d->d_conv);
  if (d->batch <= 0) return fail(SSM_ERR_INVALID_ARG, "batch=%lld must be > 0", (long long)d->batch);
  if (prefill && d->seqlen < 0) return fail(SSM_ERR_INVALID_ARG, "seqlen=%lld must be >= 0", (long long)d->seqlen);
  if (d->d_inner <= 0 || d->d_inner % 8 != 0)
    return fail(SSM_ERR_INVALID_ARG, "d_inner=%lld must be a positive multiple of 8", (long long)d->d_inner);
  if (!(d->dt_min > 0.0f) || !(d->dt_max >= d->dt_min))
    return fail(SSM_ERR_INVALID_ARG, "need 0 < dt_min <= dt_max (got %g, %g)", d->dt_min, d->dt_max);
  if (d->io_dtype != SSM_F32 && d->io_dtype != SSM_BF16)
    return fail(SSM_ERR_INVALID_ARG, "io_dtype=%d unknown", d->io_dtype);
  if (d->discretization != SSM_DISC_EULER_B && d->discretization != SSM_DISC_ZOH)
    return fail(SSM_ERR_INVALID_ARG, "discretization=%d unknown", d->discretization);
  const int64_t E = d->d_inner;
  const int64_t L = prefill ? d->seqlen : 1;
  s->x_tok = d->x_tok_stride ? d->x_tok_stride : E;
  s->z_tok = d->z_tok_stride ? d->z_tok_stride : E;
  s->y_tok = d->y_tok_stride ? d->y_tok_stride : E;
  s->x_seq = d->x_seq_stride ? d->x_seq_stride : (prefill ? L * s->x_tok : s->x_tok);
  s->z_seq = d->z_seq_stride ? d->z_seq_stride : (prefill ? L * s->z_tok : s->z_tok);
  s->y_seq = d->y_seq_stride ? d->y_seq_stride : (prefill ? L * s->y_tok : s->y_tok);
  s->bc_tok = d->bc_tok_stride ? d->bc_tok_stride : 16;
  s->bc_seq = d->bc_seq_stride ? d->bc_seq_stride : (prefill ? L * s->bc_tok : s->bc_tok);
  s->dt_seq = d->dt_seq_stride ? d->dt_seq_stride : (prefill ? L : 1);
  const int64_t io[6] = {s->x_tok, s->x_seq, s->z_tok, s->z_seq, s->y_tok, s->y_seq};
  for (int i = 0; i < 6; ++i)
    if (io[i] < 0 || io[i] % 8 != 0)
      return fail(SSM_ERR_INVALID_ARG, "x/z/y strides must be non-negative multiples of 8 elements");
  if (s->x_tok < E || s->z_tok < E || s->y_tok < E)
    return fail(SSM_ERR_INVALID_ARG, "x/z/y token strides must be >= d_inner");
  if (s->bc_tok < 16 || s->bc_tok % 4 != 0 || s->bc_seq < 0 || s->bc_seq % 4 != 0)
    return fail(SSM_ERR_INVALID_ARG, "B/C strides: token stride >= 16 and both multiples of 4");
  if (s->dt_seq < 0) return fail(SSM_ERR_INVALID_ARG, "dt_raw sequence stride must be >= 0");
  return SSM_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ssm_status check_weights(const ssm_weights* w) {
  if (!w) return fail(SSM_ERR_INVALID_ARG, "weights is NULL");
  const float* p[6] = {w->conv_w, w->conv_b, w->w_dt, w->dt_bias, w->A_log, w->D};
  const char* names[6] = {"conv_w", "conv_b", "w_dt", "dt_bias", "A_log", "D"};
  for (int i = 0; i < 6; ++i) {
    if (!p[i]) return fail(SSM_ERR_INVALID_ARG, "weights.%s is NULL", names[i]);
    const size_t need = (i == 0 || i == 4) ? 16 : 4;  // conv_w and A_log rows are read as 16-byte vectors
    if (!aligned(p[i], need)) return fail(SSM_ERR_INVALID_ARG, "weights.%s is not %zu-byte aligned", names[i], need);
  }
  return SSM_OK;
}

ssm_status check_prefill_caches(const void* conv_cache_in, const float* ssm_state_in, const void* conv_cache_out,
                                const float* ssm_state_out) {
  if (!conv_cache_out || !aligned(conv_cache_out, 16))
    return fail(SSM_ERR_INVALID_ARG, "conv_cache_out is NULL or not 16-byte aligned");
  if (!ssm_state_out || !aligned(ssm_state_out, 16))
    return fail(SSM_ERR_INVALID_ARG, "ssm_state_out is NULL or not 16-byte aligned");
  if (conv_cache_in && !aligned(conv_cache_in, 16)) return fail(SSM_ERR_INVALID_ARG, "conv_cache_in not 16-byte aligned");
  if (ssm_state_in && !aligned(ssm_state_in, 4)) return fail(SSM_ERR_INVALID_ARG, "ssm_state_in not 4-byte aligned");
  return SSM_OK;
}

}  // namespace ssm

namespace {
using ssm::aligned;
using ssm::check_dims;
using ssm::check_prefill_caches;
using ssm::check_weights;
using ssm::fail;

ssm_status ok() {
  g_last_error[0] = '\0';
  return SSM_OK;
}

ssm_status check_io_ptr(const void* p, const char* name, size_t align) {
  if (!p) return fail(SSM_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(SSM_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return SSM_OK;
}

int num_sms_current() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

void fill_weights(ssm::KernelArgs& a, const ssm_weights* w) {
  a.conv_w = w->conv_w;
  a.conv_b = w->conv_b;
  a.w_dt = w->w_dt;
  a.dt_bias = w->dt_bias;
  a.A_log = w->A_log;
  a.D = w->D;
}

__device__ int g_device_error = 0;

// One thread arms an mbarrier for two arrivals and gives it one, so the phase
// can never complete; its bounded wait gives up after limit_ns, writes `code`
// to the error word and the kernel returns. No memory operation is pending on
// the barrier when the CTA exits.
__global__ void bounded_wait_selftest_kernel(int* err, uint64_t limit_ns, int code) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ssm::smem_u32(&bar);
  ssm::mbar_init(b, 2);
  ssm::mbar_fence_init();
  ssm::mbar_arrive(b);
  ssm::mbar_wait_bounded_ns(b, 0u, err, code, limit_ns);
}

}  // namespace

namespace ssm {
// Device address of the error word on the current device (looked up once per
// device; host code must not pass the symbol itself to a kernel).
// Any host thread may call this; the per-device cache entries are atomics
// (two threads that race on an empty entry both look the address up and
// store the same value).
int* device_error_ptr() {
  static std::atomic<int*> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  const bool cached = dev >= 0 && dev < 64;
  if (cached) {
    int* p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  if (cached) cache[dev].store(static_cast<int*>(p), std::memory_order_release);
  return static_cast<int*>(p);
}
}  // namespace ssm

namespace {
using ssm::device_error_ptr;

// The prefill launch shape for `dims` and `tuning` on a GPU of `num_sms` SMs:
// the automatic choice, or the one `tuning` names; the tuning's fields are
// checked here. Host-only.
ssm_status resolve_prefill_shape(const ssm_dims* dims, const ssm_tuning* tuning, int num_sms,
                                 ssm::PrefillShape* sh, int* decay_path) {
  const bool per_state = dims->discretization == SSM_DISC_ZOH || (tuning && tuning->decay_path == 1);
  *sh = ssm::choose_prefill_shape(dims->batch, dims->d_inner, dims->seqlen, num_sms, per_state);
  *decay_path = 0;
  if (tuning) {
    if (tuning->kernel) sh->kernel = tuning->kernel;
    if (!ssm::prefill_shape_supported(*sh))
      return fail(SSM_ERR_INVALID_ARG, "tuning: kernel=%d is not built (3, 4 or 5)", sh->kernel);
    if (tuning->decay_path != 0 && tuning->decay_path != 1)
      return fail(SSM_ERR_INVALID_ARG, "tuning: decay_path=%d (0 = auto, 1 = per-state exponentials)",
                  tuning->decay_path);
    *decay_path = tuning->decay_path;
  }
  return SSM_OK;
}

}  // namespace

namespace ssm {

ssm_status prefill_entry(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                         const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                         void* y, void* conv_cache_out, float* ssm_state_out, const ssm_tuning* tuning, bool pdl,
                         void* stream) {
  ssm::Strides s;
  ssm_status st = check_dims(dims, true, &s);
  if (st != SSM_OK) return st;
  if ((st = check_weights(w)) != SSM_OK) return st;
  if (dims->seqlen > 0) {  // with L == 0 the token tensors are not read and may be NULL
    if ((st = check_io_ptr(x, "x", 16)) != SSM_OK) return st;
    if ((st = check_io_ptr(z, "z", 16)) != SSM_OK) return st;
    if ((st = check_io_ptr(y, "y", 16)) != SSM_OK) return st;
    if ((st = check_io_ptr(B, "B", 16)) != SSM_OK) return st;
    if ((st = check_io_ptr(C, "C", 16)) != SSM_OK) return st;
    if ((st = check_io_ptr(dt_raw, "dt_raw", 4)) != SSM_OK) return st;
    if (y == x || y == z) return fail(SSM_ERR_INVALID_ARG, "y must not alias x or z");
  }
  if ((st = check_prefill_caches(conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out)) != SSM_OK) return st;

  ssm::PrefillShape sh;
  int decay_path = 0;
  if ((st = resolve_prefill_shape(dims, tuning, num_sms_current(), &sh, &decay_path)) != SSM_OK) return st;

  ssm::KernelArgs a{};
  a.x = x;
  a.z = z;
  a.B = B;
  a.C = C;
  a.dt_raw = dt_raw;
  fill_weights(a, w);
  a.conv_cache_in = conv_cache_in;
  a.ssm_state_in = ssm_state_in;
  a.y = y;
  a.conv_cache_out = conv_cache_out;
  a.ssm_state_out = ssm_state_out;
  a.batch = dims->batch;
  a.L = dims->seqlen;
  a.E = dims->d_inner;
  a.s = s;
  a.dt_min = dims->dt_min;
  a.dt_max = dims->dt_max;
  a.decay_path = decay_path;
  a.err = device_error_ptr();
  if (!a.err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  cudaError_t err = ssm::launch_prefill(a, dims->io_dtype == SSM_BF16, dims->discretization == SSM_DISC_ZOH, sh,
                                        static_cast<cudaStream_t>(stream), pdl);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(err));
  return ok();
}

}  // namespace ssm

extern "C" {

size_t ssm_prefill_workspace_bytes(const ssm_dims* dims) {
  (void)dims;
  return 0;
}

int32_t ssm_prefill_kernel(const ssm_dims* dims, const ssm_tuning* tuning, int32_t num_sms) {
  ssm::Strides s;
  if (check_dims(dims, true, &s) != SSM_OK) return 0;
  ssm::PrefillShape sh;
  int decay_path = 0;
  if (resolve_prefill_shape(dims, tuning, num_sms > 0 ? num_sms : num_sms_current(), &sh, &decay_path) != SSM_OK)
    return 0;
  return sh.kernel;
}

ssm_status ssm_prefill_ex(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                          const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                          void* y, void* conv_cache_out, float* ssm_state_out, void* workspace, size_t workspace_bytes,
                          const ssm_tuning* tuning, void* stream) {
  if (workspace_bytes < ssm_prefill_workspace_bytes(dims)) return fail(SSM_ERR_INVALID_ARG, "workspace too small");
  (void)workspace;
  return ssm::prefill_entry(dims, w, x, z, B, C, dt_raw, conv_cache_in, ssm_state_in, y, conv_cache_out,
                            ssm_state_out, tuning, false, stream);
}

ssm_status ssm_prefill(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                       const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                       void* y, void* conv_cache_out, float* ssm_state_out, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return ssm_prefill_ex(dims, w, x, z, B, C, dt_raw, conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                        workspace, workspace_bytes, nullptr, stream);
}

ssm_status ssm_decode_step(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                           const float* C, const float* dt_raw, void* y, void* conv_cache, float* ssm_state,
                           void* stream) {
  ssm::Strides s;
  ssm_status st = check_dims(dims, false, &s);
  if (st != SSM_OK) return st;
  if ((st = check_weights(w)) != SSM_OK) return st;
  const size_t io_size = dims->io_dtype == SSM_BF16 ? 2 : 4;
  if ((st = check_io_ptr(x, "x", io_size)) != SSM_OK) return st;
  if ((st = check_io_ptr(z, "z", io_size)) != SSM_OK) return st;
  if ((st = check_io_ptr(y, "y", io_size)) != SSM_OK) return st;
  if ((st = check_io_ptr(B, "B", 16)) != SSM_OK) return st;
  if ((st = check_io_ptr(C, "C", 16)) != SSM_OK) return st;
  if ((st = check_io_ptr(dt_raw, "dt_raw", 4)) != SSM_OK) return st;
  if ((st = check_io_ptr(conv_cache, "conv_cache", io_size)) != SSM_OK) return st;
  if ((st = check_io_ptr(ssm_state, "ssm_state", 16)) != SSM_OK) return st;
  if (y == x || y == z) return fail(SSM_ERR_INVALID_ARG, "y must not alias x or z");

  ssm::KernelArgs a{};
  a.x = x;
  a.z = z;
  a.B = B;
  a.C = C;
  a.dt_raw = dt_raw;
  fill_weights(a, w);
  a.conv_cache_in = conv_cache;
  a.ssm_state_in = ssm_state;
  a.y = y;
  a.conv_cache_out = conv_cache;
  a.ssm_state_out = ssm_state;
  a.batch = dims->batch;
  a.L = 1;
  a.E = dims->d_inner;
  a.s = s;
  a.dt_min = dims->dt_min;
  a.dt_max = dims->dt_max;
  a.err = device_error_ptr();
  if (!a.err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  cudaError_t err = ssm::launch_decode(a, dims->io_dtype == SSM_BF16, dims->discretization == SSM_DISC_ZOH,
                                       static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
  return ok();
}

ssm_status ssm_check_device_error(void* stream) {
  int v = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
  if (err == cudaSuccess) err = cudaStreamSynchronize(st);
  if (err != cudaSuccess) return fail(SSM_ERR_CUDA, "device error check: %s", cudaGetErrorString(err));
  if (v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    cudaStreamSynchronize(st);
    return fail(SSM_ERR_DEVICE, "a kernel reported device error code %d", v);
  }
  return ok();
}

ssm_status ssm_selftest_bounded_wait(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 2000000000LL)
    return fail(SSM_ERR_INVALID_ARG, "limit_ns=%lld must be in [1e3, 2e9]", (long long)limit_ns);
  int* err = device_error_ptr();
  if (!err) return fail(SSM_ERR_CUDA, "device error word: %s", cudaGetErrorString(cudaGetLastError()));
  bounded_wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      err, static_cast<uint64_t>(limit_ns), SSM_SELFTEST_WAIT_CODE);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SSM_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return ok();
}

const char* ssm_status_string(ssm_status s) {
  switch (s) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported configuration";
    case SSM_ERR_CUDA: return "CUDA error";
    case SSM_ERR_DEVICE: return "device-side failure";
  }
  return "unknown status";
}

const char* ssm_last_error(void) { return g_last_error; }

const char* ssm_version(void) { return "0.1.0"; }

}  // extern "C"
