// stream_prefill.cu -- ssm_prefill_host and ssm_prefill_host_static: prefill
// from and to host memory with the copies overlapped (host code, plus the
// static device scratch of the second entry point; the kernels are
// prefill.cu's).
//
// The sequence is cut into chunks of at most T tokens (the last T tokens of a
// longer sequence as quarters) and pipelined over three streams:
//   copy-in  (internal):  H2D of chunk c's x, z, B, C, dt_raw into slot c % 2;
//   compute  (caller's):  the prefill kernel of chunk c on slot c % 2, its
//                         caches chained from chunk c - 1 (conv_cache_out and
//                         ssm_state_out are the carry; the kernels read a
//                         channel's caches before writing them);
//   copy-out (internal):  D2H of chunk c's y from slot c % 2.
// Events order the three: the copy-in of chunk c waits for the kernel of
// chunk c - 2 (same input slot), the kernel of chunk c waits for its inputs
// and for the copy-out of chunk c - 2 (same y slot), the copy-out waits for the
// kernel. The first copy waits for the work already on the caller's stream and
// the caller's stream waits for the last copy-out. Because chunked prefill
// with carried caches runs the same arithmetic in the same order per token,
// the result is bit-identical to one launch over the whole sequence.
//
// ssm_prefill_host takes the two chunk slots from a caller-owned workspace and
// creates its events per call. ssm_prefill_host_static allocates nothing: its
// slots live in a file-scope static device array (one per device, address
// taken with cudaGetSymbolAddress once per device), and its events, like the
// internal streams, are created on the first call per device and reused.
// Successive static calls are ordered on that scratch by a per-device event.
#include <cuda_runtime.h>

#include <mutex>

#include "ssm.h"
#include "ssm_internal.h"

namespace {

constexpr int64_t kDefaultChunk = 4096;        // ssm_prefill_host's chunk (chunk_tokens 0)
constexpr int64_t kStaticChunkCap = 2048;      // the static variant's largest automatic chunk
constexpr size_t kAlign = 256;
constexpr size_t kStaticScratchBytes = SSM_HOST_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Chunk buffers of ssm_prefill_host_static, one copy per device.
static __device__ __align__(256) unsigned char g_host_prefill_scratch[kStaticScratchBytes];

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

int64_t clip_chunk(int64_t T, int64_t L) { return L > 0 && T > L ? L : T; }

// Byte layout of one chunk slot (dense [b][T][...] buffers).
struct SlotLayout {
  size_t x, z, y, B, C, dt, bytes;
};

SlotLayout slot_layout(int64_t b, int64_t T, int64_t E, size_t es) {
  SlotLayout s{};
  size_t off = 0;
  s.x = off, off = align_up(off + static_cast<size_t>(b * T * E) * es);
  s.z = off, off = align_up(off + static_cast<size_t>(b * T * E) * es);
  s.y = off, off = align_up(off + static_cast<size_t>(b * T * E) * es);
  s.B = off, off = align_up(off + static_cast<size_t>(b * T * 16) * 4);
  s.C = off, off = align_up(off + static_cast<size_t>(b * T * 16) * 4);
  s.dt = off, off = align_up(off + static_cast<size_t>(b * T) * 4);
  s.bytes = off;
  return s;
}

size_t io_size(const ssm_dims* d) { return d->io_dtype == SSM_BF16 ? 2 : 4; }

// Pipeline events: start (on the caller's stream), per slot: inputs ready,
// kernel done, copy-out done; end (on the copy-in stream).
struct PipelineEvents {
  cudaEvent_t start = nullptr, in[2] = {}, comp[2] = {}, out[2] = {}, end = nullptr;
  cudaEvent_t* all[8] = {&start, &in[0], &in[1], &comp[0], &comp[1], &out[0], &out[1], &end};
};

cudaError_t create_events(PipelineEvents* ev) {
  for (cudaEvent_t* e : ev->all) {
    const cudaError_t r = cudaEventCreateWithFlags(e, cudaEventDisableTiming);
    if (r != cudaSuccess) return r;
  }
  return cudaSuccess;
}

// Destroying a recorded event that has not completed is legal: its resources
// are released when it completes.
void destroy_events(PipelineEvents* ev) {
  for (cudaEvent_t* e : ev->all)
    if (*e) cudaEventDestroy(*e), *e = nullptr;
}

// Per-device state, created on first use and kept for the process.
struct DeviceState {
  cudaStream_t in = nullptr, out = nullptr;  // internal copy streams
  bool static_ready = false;                 // the static entry point's members below are set
  PipelineEvents static_ev;
  cudaEvent_t scratch_free = nullptr;  // recorded when a static call has finished with the scratch
  char* scratch = nullptr;             // device address of g_host_prefill_scratch
};
std::mutex g_mutex;  // guards the table and serialises enqueueing
DeviceState g_dev[kMaxDevices];

cudaError_t device_state(DeviceState** out, bool with_static) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceState& d = g_dev[dev];
  if (!d.in && (e = cudaStreamCreateWithFlags(&d.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if (!d.out && (e = cudaStreamCreateWithFlags(&d.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if (with_static && !d.static_ready) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_host_prefill_scratch)) != cudaSuccess) return e;
    if ((e = create_events(&d.static_ev)) != cudaSuccess) {
      destroy_events(&d.static_ev);
      return e;
    }
    if ((e = cudaEventCreateWithFlags(&d.scratch_free, cudaEventDisableTiming)) != cudaSuccess) {
      destroy_events(&d.static_ev);
      return e;
    }
    d.scratch = static_cast<char*>(p);
    d.static_ready = true;
  }
  *out = &d;
  return cudaSuccess;
}

// Copies `rows` rows of `width` bytes for each of `nseq` sequences. The rows
// of one sequence are `src_row` / `dst_row` bytes apart and the sequences
// `src_seq` / `dst_seq` apart. One 2-D copy covers the common case of each
// sequence's rows forming one contiguous run; otherwise one 2-D copy per
// sequence.
cudaError_t copy_rows(char* dst, size_t dst_row, size_t dst_seq, const char* src, size_t src_row, size_t src_seq,
                      size_t width, int64_t rows, int64_t nseq, cudaMemcpyKind kind, cudaStream_t st) {
  if (rows <= 0 || nseq <= 0 || width == 0) return cudaSuccess;
  const size_t run = width * static_cast<size_t>(rows);
  if (src_row == width && dst_row == width && src_seq >= run && dst_seq >= run)
    return cudaMemcpy2DAsync(dst, dst_seq, src, src_seq, run, static_cast<size_t>(nseq), kind, st);
  for (int64_t s = 0; s < nseq; ++s) {
    cudaError_t e = cudaMemcpy2DAsync(dst + s * dst_seq, dst_row, src + s * src_seq, src_row, width,
                                      static_cast<size_t>(rows), kind, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The arguments of one host prefill, validated.
struct HostPrefill {
  const ssm_dims* dims;
  const ssm_weights* w;
  const void *x, *z;
  const float *B, *C, *dt;
  const void* cin;
  const float* sin;
  void* y;
  void* cout;
  float* sout;
  ssm::Strides s;
};

// Checks shared by both entry points, all before any CUDA call.
ssm_status validate(HostPrefill& hp, int64_t chunk_tokens) {
  ssm_status st = ssm::check_dims(hp.dims, true, &hp.s);
  if (st != SSM_OK) return st;
  if (chunk_tokens < 0) return ssm::fail(SSM_ERR_INVALID_ARG, "chunk_tokens=%lld must be >= 0", (long long)chunk_tokens);
  if ((st = ssm::check_weights(hp.w)) != SSM_OK) return st;
  if ((st = ssm::check_prefill_caches(hp.cin, hp.sin, hp.cout, hp.sout)) != SSM_OK) return st;
  if (hp.dims->seqlen == 0) return SSM_OK;  // the token tensors are not read
  const void* host_in[5] = {hp.x, hp.z, hp.B, hp.C, hp.dt};
  const char* names[5] = {"x", "z", "B", "C", "dt_raw"};
  for (int i = 0; i < 5; ++i)
    if (!host_in[i]) return ssm::fail(SSM_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (!hp.y) return ssm::fail(SSM_ERR_INVALID_ARG, "y is NULL");
  if (hp.y == hp.x || hp.y == hp.z) return ssm::fail(SSM_ERR_INVALID_ARG, "y must not alias x or z");
  return SSM_OK;
}

// x, z, B, C, dt_raw and y must be page-locked host memory. A copy from or
// to pageable memory makes the calling thread wait for it (for the kernels
// queued before it on its stream, too) while this library's enqueue mutex is
// held, which would stall every other thread and could deadlock one whose
// stream waits on work queued through this library.
ssm_status check_page_locked(const HostPrefill& hp) {
  const void* p[6] = {hp.x, hp.z, hp.B, hp.C, hp.dt, hp.y};
  const char* names[6] = {"x", "z", "B", "C", "dt_raw", "y"};
  for (int i = 0; i < 6; ++i) {
    cudaPointerAttributes at{};
    const cudaError_t e = cudaPointerGetAttributes(&at, p[i]);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return ssm::fail(SSM_ERR_CUDA, "pointer attributes of %s: %s", names[i], cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeHost)
      return ssm::fail(SSM_ERR_INVALID_ARG, "%s must be page-locked host memory, got %s", names[i],
                       at.type == cudaMemoryTypeUnregistered ? "pageable host memory"
                       : at.type == cudaMemoryTypeDevice   ? "device memory"
                                                           : "managed memory");
  }
  return SSM_OK;
}

// Enqueues the chunk pipeline. `after` (may be NULL) is an event the first
// copy also waits for. On return the caller's stream waits for every copy
// and kernel enqueued here, on success and on failure.
ssm_status enqueue(const HostPrefill& hp, char* ws, int64_t T, cudaStream_t cs, DeviceState* ds,
                   const PipelineEvents& ev, cudaEvent_t after) {
  const ssm_dims* dims = hp.dims;
  const ssm::Strides& s = hp.s;
  const int64_t b = dims->batch, L = dims->seqlen, E = dims->d_inner;
  const size_t es = io_size(dims);
  const SlotLayout lay = slot_layout(b, T, E, es);
  char* slot_base[2] = {ws, ws + lay.bytes};

  // Chunk dims: dense device buffers, sequence pitch T tokens.
  ssm_dims cd = *dims;
  cd.x_tok_stride = cd.z_tok_stride = cd.y_tok_stride = E;
  cd.x_seq_stride = cd.z_seq_stride = cd.y_seq_stride = T * E;
  cd.bc_tok_stride = 16;
  cd.bc_seq_stride = T * 16;
  cd.dt_seq_stride = T;

  // Chunk lengths: T tokens at a time, except that a sequence longer than one
  // chunk sends its last T tokens as quarters, so the pipeline drains after a
  // short kernel and copy-out (the caches carry across any cut, so the result
  // does not depend on where the chunks fall).
  const int64_t quarter = (T + 3) / 4;
  auto chunk_len = [&](int64_t t0) -> int64_t {
    const int64_t rem = L - t0;
    if (L <= T) return rem;
    if (rem > 2 * T) return T;
    if (rem > T) return rem - T;  // leaves exactly T tokens for the quarters
    return rem < quarter ? rem : quarter;
  };
  ssm_status result = SSM_OK;
  cudaError_t e = cudaSuccess;
  int64_t last_out = -1;  // the last chunk whose copy-out was enqueued
  auto cuda_fail = [&](const char* what) { result = ssm::fail(SSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e)); };
  do {
    if ((e = cudaEventRecord(ev.start, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(ds->in, ev.start, 0)) ||
        (e = cudaStreamWaitEvent(ds->out, ev.start, 0)) || (after && (e = cudaStreamWaitEvent(ds->in, after, 0)))) {
      cuda_fail("start");
      break;
    }
    int64_t t0 = 0, Tc = 0;
    for (int64_t c = 0; t0 < L; ++c, t0 += Tc) {
      const int k = static_cast<int>(c & 1);
      Tc = chunk_len(t0);
      char* base = slot_base[k];
      // copy-in of chunk c (slot k was last read by the kernel of chunk c - 2)
      if (c >= 2 && (e = cudaStreamWaitEvent(ds->in, ev.comp[k], 0)) != cudaSuccess) {
        cuda_fail("wait");
        break;
      }
      const char* hx = static_cast<const char*>(hp.x) + static_cast<size_t>(t0 * s.x_tok) * es;
      const char* hz = static_cast<const char*>(hp.z) + static_cast<size_t>(t0 * s.z_tok) * es;
      const char* hB = reinterpret_cast<const char*>(hp.B + t0 * s.bc_tok);
      const char* hC = reinterpret_cast<const char*>(hp.C + t0 * s.bc_tok);
      const char* hd = reinterpret_cast<const char*>(hp.dt + t0);
      const size_t row = static_cast<size_t>(E) * es, dseq = static_cast<size_t>(T * E) * es;
      const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
      if ((e = copy_rows(base + lay.x, row, dseq, hx, s.x_tok * es, s.x_seq * es, row, Tc, b, h2d, ds->in)) ||
          (e = copy_rows(base + lay.z, row, dseq, hz, s.z_tok * es, s.z_seq * es, row, Tc, b, h2d, ds->in)) ||
          (e = copy_rows(base + lay.B, 64, T * 64, hB, s.bc_tok * 4, s.bc_seq * 4, 64, Tc, b, h2d, ds->in)) ||
          (e = copy_rows(base + lay.C, 64, T * 64, hC, s.bc_tok * 4, s.bc_seq * 4, 64, Tc, b, h2d, ds->in)) ||
          (e = copy_rows(base + lay.dt, 4, T * 4, hd, 4, s.dt_seq * 4, 4, Tc, b, h2d, ds->in)) ||
          (e = cudaEventRecord(ev.in[k], ds->in))) {
        cuda_fail("copy-in");
        break;
      }
      // kernel of chunk c (y slot k was last read by the copy-out of chunk c - 2)
      if ((e = cudaStreamWaitEvent(cs, ev.in[k], 0)) || (c >= 2 && (e = cudaStreamWaitEvent(cs, ev.out[k], 0)))) {
        cuda_fail("wait");
        break;
      }
      cd.seqlen = Tc;
      const ssm_status ks = ssm_prefill(
          &cd, hp.w, base + lay.x, base + lay.z, reinterpret_cast<const float*>(base + lay.B),
          reinterpret_cast<const float*>(base + lay.C), reinterpret_cast<const float*>(base + lay.dt),
          c == 0 ? hp.cin : hp.cout, c == 0 ? hp.sin : hp.sout, base + lay.y, hp.cout, hp.sout, nullptr, 0, cs);
      if (ks != SSM_OK) {
        result = ks;  // ssm_prefill has set the message
        break;
      }
      if ((e = cudaEventRecord(ev.comp[k], cs)) != cudaSuccess) {
        cuda_fail("record");
        break;
      }
      // copy-out of chunk c
      char* hy = static_cast<char*>(hp.y) + static_cast<size_t>(t0 * s.y_tok) * es;
      if ((e = cudaStreamWaitEvent(ds->out, ev.comp[k], 0)) ||
          (e = copy_rows(hy, s.y_tok * es, s.y_seq * es, base + lay.y, row, dseq, row, Tc, b, cudaMemcpyDeviceToHost,
                         ds->out)) ||
          (e = cudaEventRecord(ev.out[k], ds->out))) {
        cuda_fail("copy-out");
        break;
      }
      last_out = c;
    }
  } while (false);
  // The caller's stream waits for everything enqueued, on success and on failure.
  if (last_out >= 0) cudaStreamWaitEvent(cs, ev.out[last_out & 1], 0);
  if (cudaEventRecord(ev.end, ds->in) == cudaSuccess) cudaStreamWaitEvent(cs, ev.end, 0);
  if (result == SSM_OK) ssm::fail(SSM_OK, "");
  return result;
}

// Largest chunk (at most kStaticChunkCap tokens, at most L) whose two slots fit
// `bytes`; 0 if not even one token fits.
int64_t largest_fitting_chunk(const ssm_dims* d, size_t bytes) {
  const size_t es = io_size(d);
  const int64_t b = d->batch, E = d->d_inner;
  const size_t per_token = 2 * static_cast<size_t>(b) * (3 * static_cast<size_t>(E) * es + 2 * 64 + 4);
  int64_t T = clip_chunk(kStaticChunkCap, d->seqlen);
  const int64_t est = static_cast<int64_t>(bytes / per_token);
  if (est < T) T = est;
  while (T > 0 && 2 * slot_layout(b, T, E, es).bytes > bytes) --T;
  return T;
}

}  // namespace

extern "C" {

size_t ssm_prefill_host_workspace_bytes(const ssm_dims* dims, int64_t chunk_tokens) {
  ssm::Strides s;
  if (chunk_tokens < 0 || ssm::check_dims(dims, true, &s) != SSM_OK) return 0;
  const int64_t T = clip_chunk(chunk_tokens > 0 ? chunk_tokens : kDefaultChunk, dims->seqlen);
  return 2 * slot_layout(dims->batch, T, dims->d_inner, io_size(dims)).bytes;
}

ssm_status ssm_prefill_host(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                            const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                            void* y, void* conv_cache_out, float* ssm_state_out, void* workspace,
                            size_t workspace_bytes, int64_t chunk_tokens, void* stream) {
  HostPrefill hp{dims, w, x, z, B, C, dt_raw, conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out, {}};
  ssm_status st = validate(hp, chunk_tokens);
  if (st != SSM_OK) return st;
  if (dims->seqlen == 0)  // nothing to stream: the caches-only path of ssm_prefill
    return ssm_prefill(dims, w, nullptr, nullptr, nullptr, nullptr, nullptr, conv_cache_in, ssm_state_in, nullptr,
                       conv_cache_out, ssm_state_out, nullptr, 0, stream);
  if (!workspace || !ssm::aligned(workspace, kAlign))
    return ssm::fail(SSM_ERR_INVALID_ARG, "workspace is NULL or not %zu-byte aligned", kAlign);
  const size_t need = ssm_prefill_host_workspace_bytes(dims, chunk_tokens);
  if (workspace_bytes < need)
    return ssm::fail(SSM_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, need);
  const int64_t T = clip_chunk(chunk_tokens > 0 ? chunk_tokens : kDefaultChunk, dims->seqlen);
  if ((st = check_page_locked(hp)) != SSM_OK) return st;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* ds = nullptr;
  cudaError_t e = device_state(&ds, false);
  if (e != cudaSuccess) return ssm::fail(SSM_ERR_CUDA, "internal streams: %s", cudaGetErrorString(e));
  PipelineEvents ev;
  if ((e = create_events(&ev)) != cudaSuccess) {
    destroy_events(&ev);
    return ssm::fail(SSM_ERR_CUDA, "events: %s", cudaGetErrorString(e));
  }
  st = enqueue(hp, static_cast<char*>(workspace), T, static_cast<cudaStream_t>(stream), ds, ev, nullptr);
  destroy_events(&ev);
  return st;
}

ssm_status ssm_prefill_host_static(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z,
                                   const float* B, const float* C, const float* dt_raw, const void* conv_cache_in,
                                   const float* ssm_state_in, void* y, void* conv_cache_out, float* ssm_state_out,
                                   int64_t chunk_tokens, void* stream) {
  HostPrefill hp{dims, w, x, z, B, C, dt_raw, conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out, {}};
  ssm_status st = validate(hp, chunk_tokens);
  if (st != SSM_OK) return st;
  if (dims->seqlen == 0)
    return ssm_prefill(dims, w, nullptr, nullptr, nullptr, nullptr, nullptr, conv_cache_in, ssm_state_in, nullptr,
                       conv_cache_out, ssm_state_out, nullptr, 0, stream);
  int64_t T = 0;
  if (chunk_tokens > 0) {
    T = clip_chunk(chunk_tokens, dims->seqlen);
    if (2 * slot_layout(dims->batch, T, dims->d_inner, io_size(dims)).bytes > kStaticScratchBytes)
      return ssm::fail(SSM_ERR_INVALID_ARG, "chunk of %lld tokens does not fit the %zu-byte static scratch",
                       (long long)T, kStaticScratchBytes);
  } else if ((T = largest_fitting_chunk(dims, kStaticScratchBytes)) == 0) {
    return ssm::fail(SSM_ERR_UNSUPPORTED, "batch * d_inner too large for the %zu-byte static scratch",
                     kStaticScratchBytes);
  }
  if ((st = check_page_locked(hp)) != SSM_OK) return st;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* ds = nullptr;
  cudaError_t e = device_state(&ds, true);
  if (e != cudaSuccess) return ssm::fail(SSM_ERR_CUDA, "static scratch / streams / events: %s", cudaGetErrorString(e));
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The first copy waits until the previous static call on this device (on
  // any stream) has finished with the scratch; this call marks its own end.
  st = enqueue(hp, ds->scratch, T, cs, ds, ds->static_ev, ds->scratch_free);
  if ((e = cudaEventRecord(ds->scratch_free, cs)) != cudaSuccess && st == SSM_OK)
    st = ssm::fail(SSM_ERR_CUDA, "record: %s", cudaGetErrorString(e));
  return st;
}

}  // extern "C"
