// stream_prefill.cu -- ssm_prefill_host: prefill from and to host memory with
// the copies overlapped (host code only; the kernels are prefill.cu's).
//
// The sequence is cut into chunks of T tokens and pipelined over three streams:
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
#include <cuda_runtime.h>

#include <mutex>

#include "ssm.h"
#include "ssm_internal.h"

namespace {

constexpr int64_t kDefaultChunk = 2048;
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

int64_t chunk_of(int64_t chunk_tokens, int64_t L) {
  const int64_t T = chunk_tokens > 0 ? chunk_tokens : kDefaultChunk;
  return L > 0 && T > L ? L : T;
}

// Byte layout of one chunk slot in the workspace (dense [b][T][...] buffers).
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

// Per-device internal streams, created on first use.
struct DeviceStreams {
  cudaStream_t in = nullptr, out = nullptr;
};
std::mutex g_mutex;  // guards the table and serialises enqueueing
DeviceStreams g_streams[64];

cudaError_t streams_for_current_device(DeviceStreams** ds) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DeviceStreams& d = g_streams[dev];
  if (!d.in && (e = cudaStreamCreateWithFlags(&d.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if (!d.out && (e = cudaStreamCreateWithFlags(&d.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  *ds = &d;
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

}  // namespace

extern "C" {

size_t ssm_prefill_host_workspace_bytes(const ssm_dims* dims, int64_t chunk_tokens) {
  ssm::Strides s;
  if (chunk_tokens < 0 || ssm::check_dims(dims, true, &s) != SSM_OK) return 0;
  const int64_t T = chunk_of(chunk_tokens, dims->seqlen);
  const size_t es = dims->io_dtype == SSM_BF16 ? 2 : 4;
  return 2 * slot_layout(dims->batch, T, dims->d_inner, es).bytes;
}

ssm_status ssm_prefill_host(const ssm_dims* dims, const ssm_weights* w, const void* x, const void* z, const float* B,
                            const float* C, const float* dt_raw, const void* conv_cache_in, const float* ssm_state_in,
                            void* y, void* conv_cache_out, float* ssm_state_out, void* workspace,
                            size_t workspace_bytes, int64_t chunk_tokens, void* stream) {
  ssm::Strides s;
  ssm_status st = ssm::check_dims(dims, true, &s);
  if (st != SSM_OK) return st;
  if (chunk_tokens < 0) return ssm::fail(SSM_ERR_INVALID_ARG, "chunk_tokens=%lld must be >= 0", (long long)chunk_tokens);
  if ((st = ssm::check_weights(w)) != SSM_OK) return st;
  if ((st = ssm::check_prefill_caches(conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out)) != SSM_OK) return st;
  const int64_t b = dims->batch, L = dims->seqlen, E = dims->d_inner;
  if (L == 0)  // nothing to stream: the caches-only path of ssm_prefill
    return ssm_prefill(dims, w, nullptr, nullptr, nullptr, nullptr, nullptr, conv_cache_in, ssm_state_in, nullptr,
                       conv_cache_out, ssm_state_out, nullptr, 0, stream);
  const void* host_in[5] = {x, z, B, C, dt_raw};
  const char* names[5] = {"x", "z", "B", "C", "dt_raw"};
  for (int i = 0; i < 5; ++i)
    if (!host_in[i]) return ssm::fail(SSM_ERR_INVALID_ARG, "%s is NULL", names[i]);
  if (!y) return ssm::fail(SSM_ERR_INVALID_ARG, "y is NULL");
  if (y == x || y == z) return ssm::fail(SSM_ERR_INVALID_ARG, "y must not alias x or z");
  if (!workspace || !ssm::aligned(workspace, kAlign))
    return ssm::fail(SSM_ERR_INVALID_ARG, "workspace is NULL or not %zu-byte aligned", kAlign);
  const size_t need = ssm_prefill_host_workspace_bytes(dims, chunk_tokens);
  if (workspace_bytes < need)
    return ssm::fail(SSM_ERR_INVALID_ARG, "workspace of %zu bytes, need %zu", workspace_bytes, need);

  const int64_t T = chunk_of(chunk_tokens, L);
  const size_t es = dims->io_dtype == SSM_BF16 ? 2 : 4;
  const SlotLayout lay = slot_layout(b, T, E, es);
  char* slot_base[2] = {static_cast<char*>(workspace), static_cast<char*>(workspace) + lay.bytes};

  // Chunk dims: dense device buffers, sequence pitch T tokens.
  ssm_dims cd = *dims;
  cd.x_tok_stride = cd.z_tok_stride = cd.y_tok_stride = E;
  cd.x_seq_stride = cd.z_seq_stride = cd.y_seq_stride = T * E;
  cd.bc_tok_stride = 16;
  cd.bc_seq_stride = T * 16;
  cd.dt_seq_stride = T;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceStreams* ds = nullptr;
  cudaError_t e = streams_for_current_device(&ds);
  if (e != cudaSuccess) return ssm::fail(SSM_ERR_CUDA, "internal streams: %s", cudaGetErrorString(e));
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);

  // Events: start (on the caller's stream), per slot: inputs ready, kernel
  // done, copy-out done. Destroying a recorded event that has not completed
  // is legal; its resources are released when it completes.
  cudaEvent_t ev_start, ev_in[2], ev_comp[2], ev_out[2];
  cudaEvent_t* all[7] = {&ev_start, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
  int created = 0;
  for (; created < 7; ++created)
    if ((e = cudaEventCreateWithFlags(all[created], cudaEventDisableTiming)) != cudaSuccess) break;
  auto destroy_events = [&]() {
    for (int i = 0; i < created; ++i) cudaEventDestroy(*all[i]);
  };
  if (e != cudaSuccess) {
    destroy_events();
    return ssm::fail(SSM_ERR_CUDA, "events: %s", cudaGetErrorString(e));
  }

  const int64_t n_chunks = (L + T - 1) / T;
  ssm_status result = SSM_OK;
  int64_t last_out = -1;  // index of the last chunk whose copy-out was enqueued
  auto cuda_fail = [&](const char* what) {
    result = ssm::fail(SSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  };
  do {
    if ((e = cudaEventRecord(ev_start, cs)) != cudaSuccess) { cuda_fail("record"); break; }
    if ((e = cudaStreamWaitEvent(ds->in, ev_start, 0)) != cudaSuccess) { cuda_fail("wait"); break; }
    if ((e = cudaStreamWaitEvent(ds->out, ev_start, 0)) != cudaSuccess) { cuda_fail("wait"); break; }
    for (int64_t c = 0; c < n_chunks && result == SSM_OK; ++c) {
      const int k = static_cast<int>(c & 1);
      const int64_t t0 = c * T, Tc = (L - t0 < T) ? L - t0 : T;
      char* base = slot_base[k];
      // copy-in of chunk c (slot k was last read by the kernel of chunk c - 2)
      if (c >= 2 && (e = cudaStreamWaitEvent(ds->in, ev_comp[k], 0)) != cudaSuccess) { cuda_fail("wait"); break; }
      const char* hx = static_cast<const char*>(x) + static_cast<size_t>(t0 * s.x_tok) * es;
      const char* hz = static_cast<const char*>(z) + static_cast<size_t>(t0 * s.z_tok) * es;
      const char* hB = reinterpret_cast<const char*>(B + t0 * s.bc_tok);
      const char* hC = reinterpret_cast<const char*>(C + t0 * s.bc_tok);
      const char* hd = reinterpret_cast<const char*>(dt_raw + t0);
      const size_t row = static_cast<size_t>(E) * es, dseq = static_cast<size_t>(T * E) * es;
      if ((e = copy_rows(base + lay.x, row, dseq, hx, s.x_tok * es, s.x_seq * es, row, Tc, b, cudaMemcpyHostToDevice,
                         ds->in)) != cudaSuccess ||
          (e = copy_rows(base + lay.z, row, dseq, hz, s.z_tok * es, s.z_seq * es, row, Tc, b, cudaMemcpyHostToDevice,
                         ds->in)) != cudaSuccess ||
          (e = copy_rows(base + lay.B, 64, T * 64, hB, s.bc_tok * 4, s.bc_seq * 4, 64, Tc, b, cudaMemcpyHostToDevice,
                         ds->in)) != cudaSuccess ||
          (e = copy_rows(base + lay.C, 64, T * 64, hC, s.bc_tok * 4, s.bc_seq * 4, 64, Tc, b, cudaMemcpyHostToDevice,
                         ds->in)) != cudaSuccess ||
          (e = copy_rows(base + lay.dt, 4, T * 4, hd, 4, s.dt_seq * 4, 4, Tc, b, cudaMemcpyHostToDevice, ds->in)) !=
              cudaSuccess ||
          (e = cudaEventRecord(ev_in[k], ds->in)) != cudaSuccess) {
        cuda_fail("copy-in");
        break;
      }
      // kernel of chunk c (y slot k was last read by the copy-out of chunk c - 2)
      if ((e = cudaStreamWaitEvent(cs, ev_in[k], 0)) != cudaSuccess ||
          (c >= 2 && (e = cudaStreamWaitEvent(cs, ev_out[k], 0)) != cudaSuccess)) {
        cuda_fail("wait");
        break;
      }
      cd.seqlen = Tc;
      const ssm_status ks = ssm_prefill(
          &cd, w, base + lay.x, base + lay.z, reinterpret_cast<const float*>(base + lay.B),
          reinterpret_cast<const float*>(base + lay.C), reinterpret_cast<const float*>(base + lay.dt),
          c == 0 ? conv_cache_in : conv_cache_out, c == 0 ? ssm_state_in : ssm_state_out, base + lay.y,
          conv_cache_out, ssm_state_out, nullptr, 0, stream);
      if (ks != SSM_OK) {
        result = ks;  // ssm_prefill has set the message
        break;
      }
      if ((e = cudaEventRecord(ev_comp[k], cs)) != cudaSuccess) { cuda_fail("record"); break; }
      // copy-out of chunk c
      char* hy = static_cast<char*>(y) + static_cast<size_t>(t0 * s.y_tok) * es;
      if ((e = cudaStreamWaitEvent(ds->out, ev_comp[k], 0)) != cudaSuccess ||
          (e = copy_rows(hy, s.y_tok * es, s.y_seq * es, base + lay.y, row, dseq, row, Tc, b,
                         cudaMemcpyDeviceToHost, ds->out)) != cudaSuccess ||
          (e = cudaEventRecord(ev_out[k], ds->out)) != cudaSuccess) {
        cuda_fail("copy-out");
        break;
      }
      last_out = c;
    }
  } while (false);
  // The caller's stream waits for everything enqueued, on success and on failure.
  if (last_out >= 0) cudaStreamWaitEvent(cs, ev_out[last_out & 1], 0);
  cudaEvent_t ev_end;
  if (cudaEventCreateWithFlags(&ev_end, cudaEventDisableTiming) == cudaSuccess) {
    if (cudaEventRecord(ev_end, ds->in) == cudaSuccess) cudaStreamWaitEvent(cs, ev_end, 0);
    cudaEventDestroy(ev_end);
  }
  destroy_events();
  if (result == SSM_OK) ssm::fail(SSM_OK, "");
  return result;
}

}  // extern "C"
