/*
 * ssm.h -- C ABI of the B200 (sm_100a) selective state-space block core.
 *
 * The block core computes, per channel e of every sequence (Mamba-style,
 * diagonal A, one B/C group shared by all channels):
 *
 *   c_t   = conv_b[e] + sum_{k<4} conv_w[e,k] * xh[t+k]    causal depthwise conv,
 *           xh = [3 history rows, x_0 .. x_{L-1}]           weight 3 = current token
 *   u_t   = SiLU(c_t)
 *   dt_t  = clip(softplus(dt_raw_t * w_dt[e] + dt_bias[e]), dt_min, dt_max)
 *   A_n   = -exp(A_log[e,n])
 *   h_n   <- exp(dt_t A_n) h_n + dt_t B_{t,n} u_t          (Euler-B, default)
 *            exp(dt_t A_n) h_n + (exp(dt_t A_n)-1)/A_n B_{t,n} u_t   (ZOH)
 *   y_t   = (sum_n C_{t,n} h_n + D[e] u_t) * SiLU(z_t)
 *
 * Sources: "Axon-SSM: selective state space model" (Bit-Axon docs), the block
 * diagram under "Algorithm" (conv1d causal kernel=4 groups=E, SiLU, x_proj to
 * B, C, dt_raw, dt_proj 1->E with softplus and clip, scan, y*SiLU(z)),
 * "State initialization" (A = -exp(A_log)), "JIT-compiled kernels"
 * (_ssm_fma: dA*h + dB*x_t; _compute_dt: clip(softplus(dt+dt_bias),lo,hi)) and
 * "Autoregressive decoding" (prefill from cache=None with a zero state that
 * builds conv_cache from the last K-1 positions; decode = one scan step that
 * carries [conv_cache, ssm_state]). The zero-order-hold option follows "Mamba/
 * SSM basics" (molayo insights), "Technical details"; the D skip on the scan
 * input follows "What is the Mamba model?" (velog), "chunkscan". Two entry
 * points, one per mode, as "Understanding the selective state space model from
 * the implementation side" (molayo insights) recommends in its reading
 * checklist (separate full-sequence scan and incremental update).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory and keeps no per-call state.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = the
 *    legacy default stream); nothing synchronises the host. Launch failures
 *    return SSM_ERR_CUDA; faults during execution surface at the caller's next
 *    synchronisation.
 *  - Argument checks happen on the host before any launch: a NULL required
 *    pointer, a non-positive size, a misaligned pointer or stride returns
 *    SSM_ERR_INVALID_ARG; d_state != 16 or d_conv != 4 returns
 *    SSM_ERR_UNSUPPORTED. ssm_last_error() then describes the failure.
 *  - Strides are in elements; 0 selects the dense default. x, z, y and
 *    conv_cache use `io_dtype`; B, C, dt_raw, the parameters and ssm_state are
 *    fp32. Pointers of x, z, y, B, C, dt_raw must be 16-byte aligned and the
 *    non-zero strides of x, z, y multiples of 8 elements (16 bytes at bf16),
 *    those of B, C multiples of 4 elements; d_inner must be a multiple of 8.
 */
#ifndef SSM_B200_H
#define SSM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = 1,
  SSM_ERR_UNSUPPORTED = 2,
  SSM_ERR_CUDA = 3,
  SSM_ERR_DEVICE = 4 /* a kernel reported a failure through the error word */
} ssm_status;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype;

typedef enum { SSM_DISC_EULER_B = 0, SSM_DISC_ZOH = 1 } ssm_discretization;

/* Problem shape, options and tensor strides (elements; 0 = dense default). */
typedef struct {
  int64_t batch;          /* b: independent sequences (> 0) */
  int64_t seqlen;         /* L: tokens per sequence for prefill (>= 0); decode ignores it */
  int64_t d_inner;        /* E: channels (> 0, multiple of 8) */
  int32_t d_state;        /* N: must be 16 */
  int32_t d_conv;         /* K: must be 4 */
  float dt_min, dt_max;   /* clip bounds of dt, 0 < dt_min <= dt_max */
  int32_t io_dtype;       /* ssm_dtype of x, z, y, conv_cache */
  int32_t discretization; /* ssm_discretization */
  /* x, z, y: element (s, t, e) lives at s*seq_stride + t*tok_stride + e.
   * Dense defaults: tok_stride = E, seq_stride = L*tok_stride (prefill) or
   * tok_stride (decode, where t is absent). A fused in_proj buffer [b, L, 2E]
   * passes x = buf, z = buf + E with tok_stride = 2E. */
  int64_t x_tok_stride, x_seq_stride;
  int64_t z_tok_stride, z_seq_stride;
  int64_t y_tok_stride, y_seq_stride;
  /* B, C: element (s, t, n) at s*bc_seq_stride + t*bc_tok_stride + n.
   * Dense: bc_tok_stride = 16, bc_seq_stride = L*16 (decode: 16).
   * dt_raw: element (s, t) at s*dt_seq_stride + t. Dense: L (decode: 1). */
  int64_t bc_tok_stride, bc_seq_stride;
  int64_t dt_seq_stride;
} ssm_dims;

/* Per-channel parameters, fp32, dense, device pointers (all required).
 * conv_w [E][4], conv_b [E], w_dt [E], dt_bias [E], A_log [E][16], D [E].
 * conv_w and A_log must be 16-byte aligned, the others 4-byte aligned. */
typedef struct {
  const float *conv_w, *conv_b, *w_dt, *dt_bias, *A_log, *D;
} ssm_weights;

/* Launch overrides for tests and tuning; pass NULL for the defaults.
 * kernel: 0 = auto; 3 = pipelined state slices (a CTA of 4 warps covers 32
 *   channels, warp j owns states 4j..4j+3 of each, the per-token work of the
 *   next 32-token stage overlaps the scan of the current one), built for three
 *   resident CTAs per SM; 4 = the same code built for two CTAs per SM (a larger
 *   register budget); 5 = warp-specialised: the same state slices in 4 warps
 *   and the per-token work (conv, SiLU, dt, gate) of the next stage in 4 more,
 *   handing over through mbarriers (two CTAs of 8 warps per SM). With
 *   ctas = batch * ceil(d_inner / 32), auto takes 5 when ctas <= SMs; else,
 *   up to 64 * SMs, 5 when every CTA runs per-state exponentials (ZOH, or
 *   decay_path = 1) and 4 otherwise; else 3. Any other value returns
 *   SSM_ERR_INVALID_ARG.
 * decay_path: 0 = auto; 1 = every decay exp(dt A_n) as its own exponential.
 *   Auto: a CTA whose 32 channels all have A_n = (n+1) A_0 within 2^-20
 *   relative (the "State initialization" of "Axon-SSM": diagonals -1..-16)
 *   forms the decays as powers q^(n+1) of q = exp(dt A_0), one exponential per
 *   channel-token instead of 16; every other CTA uses per-state exponentials.
 *   Euler-B only (ZOH always uses per-state exponentials). */
typedef struct {
  int32_t kernel;
  int32_t decay_path;
} ssm_tuning;

/*
 * ssm_prefill -- full-sequence mode ("Autoregressive decoding", first call).
 *
 *   x, z            [b, L, *] io_dtype (strides above)
 *   B, C            [b, L, 16] fp32; dt_raw [b, L] fp32
 *   conv_cache_in   [b, 3, E] io_dtype, dense, or NULL = zero history
 *   ssm_state_in    [b, E, 16] fp32, dense, or NULL = zero state
 *   y               [b, L, *] io_dtype (strides above); must not overlap x or z
 *   conv_cache_out  [b, 3, E] io_dtype: the last 3 raw x rows of [history, x]
 *   ssm_state_out   [b, E, 16] fp32: the state after the last token
 *   workspace       device scratch of ssm_prefill_workspace_bytes() bytes, or
 *                   NULL when that size is 0
 * conv_cache_out may alias conv_cache_in and ssm_state_out may alias
 * ssm_state_in (each channel reads its cache before writing it). The non-NULL
 * *_in pointers let a long sequence be processed in pieces: feeding one call's
 * caches to the next gives the result of one call over the whole sequence.
 * L == 0 copies the incoming caches (or zeros) to the outputs; x, z, B, C,
 * dt_raw and y are then not read and may be NULL.
 */
ssm_status ssm_prefill(const ssm_dims *dims, const ssm_weights *w, const void *x, const void *z,
                       const float *B, const float *C, const float *dt_raw, const void *conv_cache_in,
                       const float *ssm_state_in, void *y, void *conv_cache_out, float *ssm_state_out,
                       void *workspace, size_t workspace_bytes, void *stream);

/* ssm_prefill with launch-shape overrides (tuning may be NULL). */
ssm_status ssm_prefill_ex(const ssm_dims *dims, const ssm_weights *w, const void *x, const void *z,
                          const float *B, const float *C, const float *dt_raw, const void *conv_cache_in,
                          const float *ssm_state_in, void *y, void *conv_cache_out, float *ssm_state_out,
                          void *workspace, size_t workspace_bytes, const ssm_tuning *tuning, void *stream);

/* Device scratch bytes ssm_prefill needs for `dims` (0 for every shape the
 * single-pass kernel covers). Returns 0 for invalid dims as well. */
size_t ssm_prefill_workspace_bytes(const ssm_dims *dims);

/* The prefill kernel (3, 4 or 5; see ssm_tuning) that ssm_prefill launches
 * for `dims` and `tuning` (NULL = defaults) on a GPU of `num_sms` SMs
 * (<= 0: the current device's). Host-only: with num_sms > 0 it makes no CUDA
 * call. Returns 0 where ssm_prefill would reject the dims or the tuning. With
 * seqlen 0 ssm_prefill runs no scan kernel (it only passes the caches on);
 * the value is then the shape the same call would take with tokens. */
int32_t ssm_prefill_kernel(const ssm_dims *dims, const ssm_tuning *tuning, int32_t num_sms);

/*
 * ssm_prefill_host -- ssm_prefill with the token tensors in HOST memory. The
 * block core is the same, from the same pages and sections as ssm_prefill:
 * prefill of "Axon-SSM: selective state space model", "Algorithm".
 *
 * What it does. x, z, B, C and dt_raw are read from host buffers, and y is
 * written to a host buffer. L is processed in chunks of chunk_tokens tokens
 * (when L is longer than one chunk, its last chunk_tokens tokens go as four
 * quarter chunks, so that the pipeline drains after a short kernel and
 * copy-out), and three kinds of work overlap chunk by chunk:
 *  - the host->device copies of chunk c + 1, on an internal copy-in stream;
 *  - the kernel of chunk c, on `stream`;
 *  - the device->host copy of chunk c - 1's y, on an internal copy-out stream.
 * The caches carry from chunk to chunk on the device: conv_cache_out and
 * ssm_state_out serve as the carry. The result therefore equals one
 * ssm_prefill over the whole sequence, bit for bit.
 *
 * Arguments.
 *   x, z, B, C, dt_raw, y   HOST pointers, laid out as in ssm_prefill. The
 *                           token and sequence strides of dims apply to them.
 *                           They must be page-locked host memory (cudaHostAlloc,
 *                           cudaHostRegister, torch pin_memory); pageable,
 *                           device or managed memory returns
 *                           SSM_ERR_INVALID_ARG. (A copy from or to pageable
 *                           memory blocks the calling thread, and the enqueue
 *                           below holds a library-wide lock.)
 *   conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out
 *                           device pointers, as in ssm_prefill.
 *   workspace               device scratch of at least
 *                           ssm_prefill_host_workspace_bytes(dims, chunk_tokens)
 *                           bytes, 256-byte aligned. It holds two chunk buffers.
 *   chunk_tokens            tokens per chunk, >= 1; 0 selects 4096.
 *
 * Ordering. The call returns once every copy and kernel is enqueued. The first
 * copy waits for the work already queued on `stream`, and `stream` waits for
 * the last copy. A synchronisation of `stream` therefore makes y complete on
 * the host. The host buffers and the workspace must stay valid until then.
 * Enqueueing from several host threads is serialised inside the library.
 *
 * Errors. Argument errors return SSM_ERR_INVALID_ARG before any work is
 * queued. A CUDA error while enqueueing returns SSM_ERR_CUDA. Chunks already
 * enqueued then still run, and `stream` is left waiting for them.
 */
ssm_status ssm_prefill_host(const ssm_dims *dims, const ssm_weights *w, const void *x, const void *z,
                            const float *B, const float *C, const float *dt_raw, const void *conv_cache_in,
                            const float *ssm_state_in, void *y, void *conv_cache_out, float *ssm_state_out,
                            void *workspace, size_t workspace_bytes, int64_t chunk_tokens, void *stream);

/* Device scratch bytes ssm_prefill_host needs for `dims` and `chunk_tokens`
 * (0 selects 4096): two chunk buffers of x, z, y, B, C and dt_raw. Returns 0
 * for invalid dims. */
size_t ssm_prefill_host_workspace_bytes(const ssm_dims *dims, int64_t chunk_tokens);

/* Bytes of the device scratch that ssm_prefill_host_static owns: a static
 * device array of the library, one per device. It is reserved on a device
 * when the library's device code is loaded there (at context creation under
 * CUDA_MODULE_LOADING=EAGER, else at the first use of any of the library's
 * kernels), whichever entry points the process calls, and held until exit:
 * every process that loads libssm.so pays these bytes on each device it
 * uses the library on. */
#define SSM_HOST_STATIC_SCRATCH_BYTES ((size_t)128 << 20)

/*
 * ssm_prefill_host_static -- ssm_prefill_host without a workspace and without
 * any allocation. The computation, arguments, result (bit-identical to one
 * ssm_prefill), ordering with `stream` and host-buffer lifetime are those of
 * ssm_prefill_host.
 *
 * Scratch. The two chunk buffers live in the library's static device scratch
 * of SSM_HOST_STATIC_SCRATCH_BYTES per device; its address is looked up once
 * per device. The internal streams and events are created on the first call
 * on a device and reused by every later call, so steady-state calls create
 * nothing and allocate no memory.
 *
 * Chunk size. chunk_tokens 0 selects the largest chunk of at most 2048 tokens
 * whose two buffers fit the scratch. A nonzero chunk_tokens whose buffers do
 * not fit returns SSM_ERR_INVALID_ARG. If not even one token fits
 * (batch * d_inner too large), the call returns SSM_ERR_UNSUPPORTED.
 *
 * Sharing. Calls on one device share the scratch, whatever their streams:
 * each call's first copy waits until the previous call has finished with it,
 * so such calls run one after another on the device.
 */
ssm_status ssm_prefill_host_static(const ssm_dims *dims, const ssm_weights *w, const void *x, const void *z,
                                   const float *B, const float *C, const float *dt_raw, const void *conv_cache_in,
                                   const float *ssm_state_in, void *y, void *conv_cache_out, float *ssm_state_out,
                                   int64_t chunk_tokens, void *stream);

/*
 * ssm_decode_step -- one-token mode ("Autoregressive decoding", later calls):
 * concatenates conv_cache with the new token, runs the conv for that token and
 * exactly one scan step from ssm_state, and updates both caches IN PLACE.
 *
 *   x, z        [b, *] io_dtype, token of sequence s at s*x_seq_stride (dense: E)
 *   B, C        [b, 16] fp32 at s*bc_seq_stride (dense: 16); dt_raw [b] at s*dt_seq_stride (dense: 1)
 *   y           [b, *] io_dtype at s*y_seq_stride (dense: E)
 *   conv_cache  [b, 3, E] io_dtype, dense, in-out
 *   ssm_state   [b, E, 16] fp32, dense, in-out, 16-byte aligned
 * dims->seqlen is ignored. Consecutive calls on one stream continue the
 * sequence: prefill(L) followed by k calls equals prefill(L + k).
 * The state of (sequence, 128 channels) moves between HBM and shared memory
 * as one 8 KB TMA tile in each direction; a thread owns one channel.
 */
ssm_status ssm_decode_step(const ssm_dims *dims, const ssm_weights *w, const void *x, const void *z,
                           const float *B, const float *C, const float *dt_raw, void *y, void *conv_cache,
                           float *ssm_state, void *stream);

/*
 * ssm_block_forward -- the whole AxonSSMBlock forward of "Axon-SSM: selective
 * state space model", "Algorithm" diagram, for a prefill:
 *
 *   x, z         = split(hidden @ W_in^T)          in_proj  (D -> 2E), x first
 *   u            = SiLU(conv1d(x))                  causal depthwise conv, K = 4
 *   B, C, dt_raw = split(u @ W_x^T)                 x_proj   (E -> 2N + 1), in that order
 *   y            = the block core of ssm_prefill    (dt_proj, softplus, clip, scan, D skip, y * SiLU(z))
 *   out          = y @ W_out^T                      out_proj (E -> D)
 *
 * Implementation. in_proj and out_proj are this library's tcgen05 GEMM
 * (ssm_proj_gemm: bf16 operands, fp32 accumulation in TMEM, bf16 out).
 * x_proj is one fused kernel: it computes u from x tile by tile straight into
 * tensor-core operand tiles (tcgen05 MMA, TMEM accumulator), so u never
 * reaches memory. The core is ssm_prefill's kernel, reading x and z in place
 * from the in_proj output; out_proj reads the core's gated output as its A
 * operand. No projection has a bias. No library GEMM is called.
 *
 * Arguments.
 *   dims      batch, seqlen, d_model (D, a multiple of 8), d_inner (E, a
 *             multiple of 8), d_state 16, d_conv 4, dt_min / dt_max,
 *             discretization. io_dtype must be SSM_BF16 (SSM_ERR_UNSUPPORTED
 *             otherwise).
 *   w         the core's per-channel parameters, as for ssm_prefill.
 *   proj      W_in [2E, D], W_x [2N + 1, E], W_out [D, E]: row-major
 *             [out_features, in_features], bf16, 16-byte aligned, on the device.
 *   hidden    [b, L, D] bf16, dense;  out [b, L, D] bf16, dense.
 *   conv_cache_in, ssm_state_in, conv_cache_out, ssm_state_out
 *             as for ssm_prefill. The conv cache holds raw x rows (in_proj
 *             output), so chained calls equal one call over the whole sequence.
 *   workspace device scratch of ssm_block_workspace_bytes(dims) bytes,
 *             256-byte aligned. It holds the in_proj output (b L 2E bf16),
 *             B / C / dt_raw (b L 33 fp32), the gated core output
 *             (b L E bf16) and the projections' cut-tile scratch (see
 *             ssm_proj_gemm).
 *
 * Ordering and errors. Everything is enqueued on `stream`, with no host
 * synchronisation: a memset of the projections' tile counters (when a tile is
 * cut), then in_proj, x_proj, the core and out_proj. Each of the last three is
 * launched overlapped with the kernel before it (programmatic dependent
 * launch), and reads nothing that kernel writes before it has finished.
 * Argument errors return before any work is queued.
 */
typedef struct {
  int64_t batch, seqlen, d_model, d_inner;
  int32_t d_state, d_conv;
  float dt_min, dt_max;
  ssm_dtype io_dtype;
  ssm_discretization discretization;
} ssm_block_dims;

typedef struct {
  const void *w_in;  /* [2E, D] */
  const void *w_x;   /* [2N + 1, E] */
  const void *w_out; /* [D, E] */
} ssm_block_weights;

ssm_status ssm_block_forward(const ssm_block_dims *dims, const ssm_weights *w, const ssm_block_weights *proj,
                             const void *hidden, const void *conv_cache_in, const float *ssm_state_in, void *out,
                             void *conv_cache_out, float *ssm_state_out, void *workspace, size_t workspace_bytes,
                             void *stream);

/* Workspace bytes of ssm_block_forward for `dims` (0 for invalid dims). */
size_t ssm_block_workspace_bytes(const ssm_block_dims *dims);

/*
 * ssm_proj_gemm -- one projection of the block, C = A . W^T: in_proj (A =
 * hidden [M, D], W = W_in [2E, D]) and out_proj (A = the core's gated output
 * [M, E], W = W_out [D, E]) of "Axon-SSM: selective state space model",
 * "Algorithm" diagram, as ssm_block_forward runs them.
 *   A  [M, K] bf16, row-major;  W  [N, K] bf16, row-major;  C  [M, N] bf16
 * Device pointers, 16-byte aligned; K and N multiples of 8; 0 < M, N, K <=
 * 2^31; C must not alias A or W. fp32 accumulation, C rounded to bf16 (RNE).
 * One persistent kernel of CTA pairs (two-SM tcgen05 MMAs into TMEM, TMA
 * operand rings, TMA stores) enqueued on `stream`, after a memset of the
 * workspace's tile counters when some tile is cut between pairs.
 *   workspace  ssm_proj_gemm_workspace_bytes(M, N, K) bytes of device scratch,
 *              256-byte aligned, or NULL when that is 0. Whole 256 x 256 output
 *              tiles go round-robin to the pairs. Where a last wave would leave
 *              most pairs idle, the final one to two tiles a pair are instead
 *              cut along K into equal runs, one per pair; a counter per tile
 *              (first) and the fp32 partials of the cut tiles (512 KB a pair)
 *              live here. The partials of a cut tile are summed in a fixed
 *              order, so results do not depend on timing. Calls that overlap
 *              on the GPU need separate workspaces.
 */
size_t ssm_proj_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
ssm_status ssm_proj_gemm(const void *A, const void *W, void *C, int64_t M, int64_t N, int64_t K, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * ssm_ssd_chunk_scan -- the output of the Mamba-2 (SSD) chunk scan, "What is
 * the Mamba model?" (velog, Texnee), "chunkscan" section. For batch b, chunk c,
 * head h (group g = h / (nheads / ngroups)) and position l of the chunk:
 *
 *   out[l] = sum_{s <= l} cb[l, s] exp(dA[l] - dA[s]) dt[s] x[s]
 *          + exp(dA[l]) C[l] . prev_states
 *          + D[h] x[l]
 *
 * Arguments. Dense row-major device tensors; bf16 = SSM_BF16 storage.
 *   cb           [b, nchunks, ngroups, cs, cs] bf16   (the chunk's C B^T scores)
 *   x            [b, L, nheads, headdim] bf16
 *   dt           [b, nheads, nchunks, cs] fp32
 *   dA_cumsum    [b, nheads, nchunks, cs] fp32        (within-chunk cumulative sum of dt A)
 *   C            [b, L, ngroups, dstate] bf16
 *   prev_states  [b, nchunks, nheads, headdim, dstate] bf16
 *   D            [nheads] fp32, or NULL for no skip
 *   out          [b, L, nheads, headdim] bf16; must not overlap the inputs
 * L = nchunks * cs. The built shapes are cs = 64, 128 or 256, headdim = 64
 * and dstate = 64 or 128 (SSM_ERR_UNSUPPORTED otherwise); at most 32767
 * chunks. nheads must be a multiple of ngroups, and every pointer 16-byte
 * aligned.
 *
 * Computation. Per (b, h) and 128 positions -- one chunk of 128, two
 * consecutive chunks of 64 on the diagonal of one 128 x 128 score tile, or
 * one half of a chunk of 256 (the second half contracting over all 256
 * positions) -- one CTA:
 *  - scores = masked cb * exp(dA[l] - dA[s]) * dt[s] in bf16, times x;
 *  - C[l] in bf16, times prev_states^T;
 * as tcgen05 MMAs into two fp32 TMEM accumulators, combined as
 * acc_scores + exp(dA[l]) acc_state + D x and stored as bf16.
 *
 * Range. Each decay exp(dA[l] - dA[s]) is formed as the product of
 * exp(dA[l] - dA[s1]) and exp(dA[s1] - dA[s]), s1 the last position of s's
 * 8-position group (in the group that holds l, when dA falls by more than 80
 * across that group: one exponential per element).
 * When dA_cumsum does not increase along a chunk (dt >= 0 and A <= 0, what a
 * cumulative sum of dt A gives), every exponent is <= 0: no factor exceeds 1
 * however strong the decay, a decayed term that underflows fp32 is 0, and
 * exp(dA[l]) <= 1 as long as dA_cumsum starts at or below 0. Any other
 * dA_cumsum is computed by the same formula, exactly while each of those
 * exponents and dA[l] stays below about 80 (fp32 exp range); beyond that the
 * output may hold inf or NaN.
 */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, ngroups, dstate, chunk_size;
} ssm_ssd_dims;

ssm_status ssm_ssd_chunk_scan(const ssm_ssd_dims *dims, const void *cb, const void *x, const float *dt,
                              const float *dA_cumsum, const void *C, const void *prev_states, const float *D,
                              void *out, void *stream);

/*
 * Sequence-parallel prefill -- one sequence split into segments that are
 * computed at the same time (one per GPU, or pieces of one long context), in
 * the three steps of "What is the Mamba model?" (velog, Texnee), "chunkscan",
 * with a segment as the chunk:
 *  1. ssm_segment_summary on every segment (but the last), independently:
 *     its final state from a zero start, h_zero, and its dt sum, dtsum;
 *  2. the summaries are exchanged (an all-gather across GPUs; the library
 *     does not communicate), and ssm_segment_carry folds those of segments
 *     0..r-1 into the state entering segment r:
 *         h <- exp(A_n dtsum_j) h + h_zero_j,   j = 0 .. r-1, from ssm_state_in,
 *     the closed form of "Mamba/SSM basics" (molayo insights), "Technical
 *     details" (h_t = A_t...A_1 h_0 + sum_j A_t...A_{j+1} B_j x_j), a segment
 *     at a time;
 *  3. ssm_prefill of segment r with ssm_state_in = that state and
 *     conv_cache_in = the last 3 raw x rows before the segment.
 * The result equals ssm_prefill of the whole sequence up to fp32 rounding
 * order; the last segment's conv_cache_out and ssm_state_out are the whole
 * sequence's.
 *
 * ssm_segment_summary. dims describe the segment (seqlen = its token count T,
 * may be 0; io_dtype, discretization, dt clip and the strides of x, B and
 * dt_raw as for ssm_prefill; z, C and y are not read).
 *   x              [b, T, *] io_dtype          B [b, T, 16] fp32; dt_raw [b, T] fp32
 *   conv_cache_in  [b, 3, E] io_dtype, dense: raw x rows before the segment;
 *                  NULL = zeros (the first segment of a fresh sequence)
 *   summary        [b, 17, E] fp32, dense: rows 0..15 h_zero (state n of
 *                  channel e at [s][n][e]), row 16 dtsum; 16-byte aligned
 *   workspace      ssm_segment_summary_workspace_bytes(dims) bytes of device
 *                  scratch (b * ceil(T / 256) * 17 * E floats), 16-byte aligned
 * Two launches: 256-token blocks reduce in parallel to (state contribution,
 * dt total) rows, then the blocks are folded in order.
 *
 * ssm_segment_carry. dims give batch, d_inner and the checks of ssm_prefill
 * (seqlen is not used).
 *   summaries      [count, b, 17, E] fp32: the summaries of segments 0..count-1
 *   ssm_state_in   [b, E, 16] fp32: state before segment 0, or NULL = zeros
 *   ssm_state_out  [b, E, 16] fp32: state entering segment `count`; may alias
 *                  ssm_state_in
 * count = 0 copies ssm_state_in (or writes zeros).
 */
size_t ssm_segment_summary_workspace_bytes(const ssm_dims *dims);
ssm_status ssm_segment_summary(const ssm_dims *dims, const ssm_weights *w, const void *x, const float *B,
                               const float *dt_raw, const void *conv_cache_in, float *summary, void *workspace,
                               size_t workspace_bytes, void *stream);
ssm_status ssm_segment_carry(const ssm_dims *dims, const ssm_weights *w, const float *summaries, int64_t count,
                             const float *ssm_state_in, float *ssm_state_out, void *stream);

/* Reads and clears the device error word that kernels set when a bounded
 * wait gives up (synchronises `stream` first). SSM_OK if no kernel failed;
 * SSM_ERR_DEVICE with the code in ssm_last_error() otherwise. Codes: 1 the
 * prefill's TMA ring, 2 the hand-overs of prefill kernel 5, 3-6 the block's x_proj kernel, 7-11 the chunk scan's
 * operand and MMA waits, 11 the decode's state ring, 21-29 the projection
 * GEMM (21 ring slot free, 22 accumulator free, 23 operands landed, 24
 * accumulator full, 25 and 29 drains, 27-28 the cut-tile handshake),
 * SSM_SELFTEST_WAIT_CODE the self-test below. Every kernel's waits give up
 * after about 2 s. */
ssm_status ssm_check_device_error(void *stream);

/* Error-word code written by ssm_selftest_bounded_wait. */
#define SSM_SELFTEST_WAIT_CODE 99

/*
 * ssm_selftest_bounded_wait -- exercises the failure path the kernels use
 * when a wait cannot complete (the failure detection of the bounded mbarrier
 * waits): one CTA arms an mbarrier that can never complete its phase, waits
 * for at most limit_ns (1e3 .. 2e9 ns), writes SSM_SELFTEST_WAIT_CODE to the
 * device error word and returns. Nothing faults or hangs; the context stays
 * usable. A following ssm_check_device_error on `stream` returns
 * SSM_ERR_DEVICE and clears the word. Enqueued on `stream`; out-of-range
 * limit_ns returns SSM_ERR_INVALID_ARG. Not part of the computation (the
 * pages have no counterpart): a check a caller can run on its own device.
 */
ssm_status ssm_selftest_bounded_wait(int64_t limit_ns, void *stream);

/* Static description of a status code. */
const char *ssm_status_string(ssm_status s);

/* Message of the last failure on the calling host thread ("" if none). */
const char *ssm_last_error(void);

/* Library version as "major.minor.patch". */
const char *ssm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_B200_H */
