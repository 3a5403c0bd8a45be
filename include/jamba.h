/*
 * jamba.h — C ABI of the B200 (sm_100a) Jamba Mamba-mixer / MoE library.
 *
 * The computation follows "Jamba: A Hybrid Transformer-Mamba Language Model"
 * (paper summary page): section 2 (Mamba layers with RMSNorm inside them, no
 * positional encoding, SwiGLU MLPs, MoE with n experts and top-K routing),
 * section 3.1 (n = 16 experts, K = 2), section 6.4 / figure 9 (RMSNorm on the
 * Mamba layer's inner activations).  The Mamba layer itself is the selective
 * state-space layer the paper cites (section 2, ref [17]):
 *
 *   xz = u W_in^T;  x, z = split(xz)
 *   xc = SiLU(causal depthwise conv1d(x) + conv_b)
 *   dt_low, B, C = split(xc W_x^T)         (RMSNorm on each when enabled)
 *   dt = softplus(dt_low W_dt^T + dt_bias)
 *   h_t = exp(dt_t A) h_{t-1} + dt_t B_t x_t,   y_t = (C_t . h_t + D x_t) SiLU(z_t)
 *   out = y W_out^T (+ residual)
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *    contiguous unless a leading dimension is given, 16-byte aligned.  The
 *    library never frees caller memory and keeps no pointer to activations
 *    after a call returns.
 *  - "dtype" tensors are bf16 (JAMBA_BF16) or fp32 (JAMBA_F32) as configured;
 *    states, dt_bias, A, D and norm weights are always fp32.
 *  - Work is enqueued on the given stream (a cudaStream_t; NULL = legacy
 *    default stream) and runs asynchronously; calls never synchronize unless
 *    documented.  Arguments are validated before anything is launched: on an
 *    error status nothing was enqueued.
 *  - Asynchronous device errors (a bounded wait inside a kernel that ran out
 *    of time) are latched in a per-device error word; read it with
 *    jamba_device_status().
 *  - No function throws; jamba_last_error() describes the last failure of
 *    the calling thread.
 */
#ifndef JAMBA_H_
#define JAMBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum jamba_status {
  JAMBA_OK = 0,
  JAMBA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size        */
  JAMBA_ERR_UNSUPPORTED = 2, /* shape or dtype outside what the kernels handle    */
  JAMBA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than *_workspace_size */
  JAMBA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed                 */
  JAMBA_ERR_TIMEOUT = 5,     /* a device-side bounded wait gave up                */
  JAMBA_ERR_OOM = 6,         /* host allocation failed                            */
  JAMBA_ERR_BOUNDS = 7       /* checked build: an index read from device data was
                                out of range (the access was skipped)             */
} jamba_status;

typedef enum jamba_dtype { JAMBA_F32 = 0, JAMBA_BF16 = 1, JAMBA_INT8 = 2 } jamba_dtype;

typedef struct CUstream_st* jamba_stream_t; /* same type as cudaStream_t */

/* Last error message of the calling thread (static storage, never NULL). */
const char* jamba_last_error(void);

/* 1 in the checked build of the library (libjamba_checked.so, compiled with
 * -DJAMBA_CHECKS), 0 otherwise.  The checked build tests on the device every
 * index that kernels read from device data before using it: routed-row
 * positions (permutation and its inverse), expert group offsets, channel
 * permutations of the reordered caches, cache lengths of the attention step.
 * A failed test latches JAMBA_ERR_BOUNDS in the device error word and skips
 * the access; nothing traps.  Group offsets are clamped into range in both
 * builds. */
int jamba_checked_build(void);

/* Synchronizes `stream`, then returns and clears the device error word of the
 * current device: JAMBA_OK, JAMBA_ERR_TIMEOUT, JAMBA_ERR_BOUNDS (checked build
 * only), or JAMBA_ERR_CUDA when the stream itself reports an error.  The word latches: once a wait has given
 * up, later kernels that share the word stop early (writing nothing) until
 * this call clears it.  It also reads and clears the word that
 * jamba_selective_scan_static uses when called with status == NULL. */
jamba_status jamba_device_status(jamba_stream_t stream);

/* ------------------------------------------------------------------ Mamba */

typedef struct jamba_mamba_config {
  int d_model;       /* block width (4096 in Jamba)                              */
  int d_inner;       /* mixer width, multiple of 8 (8192)                        */
  int d_state;       /* SSM state size: must be 16                               */
  int d_conv;        /* conv taps: must be 4                                     */
  int dt_rank;       /* rank of the dt projection, multiple of 8 (256)           */
  int dtype;         /* jamba_dtype of weights and activations                   */
  int inner_rmsnorm; /* 1: RMSNorm on dt_low, B and C (Jamba section 6.4)        */
  float eps;         /* epsilon of the inner RMSNorms                            */
} jamba_mamba_config;

typedef struct jamba_mamba_weights {
  const void* in_proj;   /* [2*d_inner, d_model] dtype; rows [0,d_inner) give x, the rest z */
  const void* conv_w;    /* [d_inner, d_conv] dtype; tap d_conv-1 multiplies the current token */
  const void* conv_b;    /* [d_inner] dtype */
  const void* x_proj;    /* [dt_rank + 2*d_state, d_inner] dtype; rows: dt_low | B | C */
  const void* dt_proj;   /* [d_inner, dt_rank] dtype */
  const float* dt_bias;  /* [d_inner] */
  const float* A;        /* [d_inner, d_state], any finite values (negative for a stable layer) */
  const float* D;        /* [d_inner] */
  const void* out_proj;  /* [d_model, d_inner] dtype */
  const float* norm_dt;  /* [dt_rank]  (read only when inner_rmsnorm) */
  const float* norm_B;   /* [d_state] */
  const float* norm_C;   /* [d_state] */
} jamba_mamba_weights;

typedef struct jamba_mamba* jamba_mamba_t;

/* Creates a mixer handle on the current CUDA device.  The weight pointers are
 * borrowed: they must stay valid and unchanged until destroy.
 * bf16 mixers (d_inner up to 16384) also keep, in device memory the handle
 * owns, a copy of the channel-indexed weights with the channels reordered by
 * how long they carry state (softplus(dt_bias) * min |A| of each channel,
 * slowest first) for the prefill: the selective scan's groups of 256
 * channels then hold channels of like speed and each group gets its own
 * number of time chunks.  The reordering is internal: inputs, outputs and
 * both caches keep the caller's channel order, and decode steps use the
 * caller's weights.  create is synchronous for bf16 (it reads dt_bias and A
 * back and builds the copy).
 * Errors: INVALID_ARG (null pointers, misalignment), UNSUPPORTED (d_state != 16,
 * d_conv != 4, widths not multiples of 8), OOM (no device memory for the
 * copy), CUDA. */
jamba_status jamba_mamba_create(const jamba_mamba_config* cfg, const jamba_mamba_weights* w,
                                jamba_mamba_t* out);
jamba_status jamba_mamba_destroy(jamba_mamba_t h);

/* Bytes of device workspace that jamba_mamba_prefill needs for `batch` rows of
 * `seqlen` tokens (seqlen = 1 gives the size for jamba_mamba_step). */
jamba_status jamba_mamba_workspace_size(jamba_mamba_t h, int batch, int seqlen, size_t* bytes);

/* Mixer forward over whole sequences (prefill).
 *   u        [batch, seqlen, d_model] dtype       input (already block-normed)
 *   residual [batch, seqlen, d_model] dtype|NULL  added to the output when given
 *   out      [batch, seqlen, d_model] dtype       may alias residual, not u
 *   conv_state_in / ssm_state_in [batch, d_inner, d_conv-1] / [batch, d_inner, d_state]
 *            fp32 or NULL: state to continue from (NULL = zeros)
 *   conv_state_out / ssm_state_out: same shapes, fp32 or NULL: the caches after
 *            the last token (conv: the last d_conv-1 pre-conv inputs, oldest first)
 *   ws / ws_bytes: device workspace of at least jamba_mamba_workspace_size bytes
 * The states may alias (in == out) for in-place continuation (the conv cache
 * is copied to the workspace first; the scan orders its own in-place update),
 * but may not overlap otherwise. */
jamba_status jamba_mamba_prefill(jamba_mamba_t h, const void* u, const void* residual, void* out,
                                 int batch, int seqlen, const float* conv_state_in,
                                 const float* ssm_state_in, float* conv_state_out,
                                 float* ssm_state_out, void* ws, size_t ws_bytes,
                                 jamba_stream_t stream);

/* Prefill from and to HOST memory, pipelined: the sequence is cut into time
 * chunks of `chunk` tokens (0 = 16384); the copy of chunk i+1 to the device,
 * the prefill of chunk i (continuing the caches) and the copy of chunk i-1
 * back overlap on two internal copy streams, so the transfers hide behind the
 * compute.  The result equals jamba_mamba_prefill of the whole sequence up to
 * rounding order at the chunk boundaries.
 *   u_host / residual_host (or NULL) / out_host: [batch, seqlen, d_model] dtype in
 *            page-locked host memory (cudaHostAlloc / cudaHostRegister);
 *            out_host may alias residual_host, not u_host
 *   conv_state_in / ssm_state_in: device, as in jamba_mamba_prefill (NULL = zeros)
 *   conv_state_out / ssm_state_out: device, required (they carry the chunks);
 *            may alias the inputs
 *   ws / ws_bytes: device workspace of at least jamba_mamba_host_workspace_size
 * The call is stream-ordered on `stream`: work queued on it afterwards sees the
 * finished output in out_host.  Errors: INVALID_ARG (host buffers not
 * page-locked, null states), WORKSPACE, CUDA. */
jamba_status jamba_mamba_host_workspace_size(jamba_mamba_t h, int batch, int chunk, size_t* bytes);
jamba_status jamba_mamba_prefill_host(jamba_mamba_t h, const void* u_host, const void* residual_host,
                                      void* out_host, int batch, int seqlen, int chunk,
                                      const float* conv_state_in, const float* ssm_state_in,
                                      float* conv_state_out, float* ssm_state_out, void* ws,
                                      size_t ws_bytes, jamba_stream_t stream);

/* One-token decode step for every batch row, updating both caches in place.
 *   u [batch, d_model], residual [batch, d_model] or NULL, out [batch, d_model]
 *   conv_state [batch, d_inner, d_conv-1] fp32, ssm_state [batch, d_inner, d_state] fp32
 * Workspace: jamba_mamba_workspace_size(h, batch, 1). */
jamba_status jamba_mamba_step(jamba_mamba_t h, const void* u, const void* residual, void* out,
                              int batch, float* conv_state, float* ssm_state, void* ws,
                              size_t ws_bytes, jamba_stream_t stream);

/* -------------------------------------------- tensor-parallel prefill */

/* Prefill with the mixer's d_inner channels split over ranks (tensor
 * parallelism; the summary page lists tensor parallelism among its training
 * parallelisms, appendix on training infrastructure, without a scheme).
 * Each rank creates its handle with d_inner = its channel count and its share
 * of the channel-indexed weights: in_proj rows of its x channels followed by
 * the rows of its z channels, conv weight and bias, x_proj columns, dt_proj
 * rows, dt_bias, A, D and out_proj columns of its channels (norm weights
 * whole).  Conv, the norms' inputs aside, dt_proj and the scan are per
 * channel; the two contractions over d_inner (x_proj and out_proj) give
 * per-rank partial sums that the caller all-reduces (sum) between the calls:
 *   begin  -> xproj_part [batch*seqlen, dt_rank + 2*d_state] fp32
 *   (all-reduce: xproj_sum)
 *   finish -> out_part [batch*seqlen, d_model] fp32
 *   (all-reduce: out_sum)
 *   end    -> out = out_sum (+ residual), in the model dtype
 * begin and finish take the same workspace (jamba_mamba_workspace_size of
 * the handle), unchanged in between: it carries the slice's activations.
 * Caches are this rank's channels: conv [batch, d_inner_r, 3], ssm
 * [batch, d_inner_r, 16], as in jamba_mamba_prefill.  Errors: INVALID_ARG,
 * WORKSPACE, UNSUPPORTED, CUDA. */
jamba_status jamba_mamba_prefill_tp_begin(jamba_mamba_t h, const void* u, int batch, int seqlen,
                                          const float* conv_state_in, float* conv_state_out,
                                          float* xproj_part, void* ws, size_t ws_bytes,
                                          jamba_stream_t stream);
jamba_status jamba_mamba_prefill_tp_finish(jamba_mamba_t h, const float* xproj_sum, int batch, int seqlen,
                                           const float* ssm_state_in, float* ssm_state_out, float* out_part,
                                           void* ws, size_t ws_bytes, jamba_stream_t stream);
jamba_status jamba_mamba_prefill_tp_end(jamba_mamba_t h, const float* out_sum, const void* residual,
                                        void* out, int batch, int seqlen, jamba_stream_t stream);

/* ------------------------------------------- context-parallel prefill */

/* Prefill of sequences split over ranks by time (context parallelism): rank r
 * holds tokens [t_r, t_r+1) of every batch row.  The Jamba summary page
 * names sequence parallelism among its training-infrastructure parallelisms
 * (appendix on training infrastructure) and the news article names MoE
 * parallelism and a faster Mamba as future speed-ups; the pages give no
 * scheme.  Here the split follows the scan's associativity: the state after
 * a slice is P (.) h_in + h_loc, with P the product of the slice's decays
 * exp(dt A) and h_loc the slice's end state from zero, so each rank scans
 * its slice once without the state entering it and once with it, and only
 * these [batch, d_inner, d_state] carries (plus a 3-token conv halo) cross
 * between ranks.  The exchanges are the caller's (two small collectives):
 *   1. before begin: the d_conv - 1 = 3 input rows preceding the slice (the
 *      last 3 rows of rank r-1's u) reach rank r as u_halo;
 *   2. between begin and finish: every rank's (carry_p, carry_h) gathered in
 *      rank order.
 *
 * Bytes of workspace the two calls need (the same workspace must be passed,
 * unchanged, to both: it carries the slice's activations between them). */
jamba_status jamba_mamba_cp_workspace_size(jamba_mamba_t h, int batch, int seqlen, size_t* bytes);

/* in_proj, causal conv + SiLU, x_proj, inner RMSNorms and dt_proj of the
 * slice, then a state-only scan of it from zero:
 *   u       [batch, seqlen, d_model] dtype, this rank's tokens
 *   u_halo  [batch, 3, d_model] dtype: the 3 input rows before the slice
 *           (ranks > 0), or NULL
 *   conv_state_in  [batch, d_inner, 3] fp32 or NULL: the conv cache before
 *           the first slice (rank 0; NULL = zeros).  At most one of u_halo
 *           and conv_state_in.
 *   ssm_state_in   [batch, d_inner, 16] fp32 or NULL: the state before the
 *           first slice (rank 0 only; it seeds rank 0's carry_h, so the
 *           other ranks never need it)
 *   conv_state_out [batch, d_inner, 3] fp32: the slice's last 3 pre-conv
 *           inputs (the global conv cache on the last rank)
 *   carry_p [batch, d_inner, 16] fp32 out: the slice's decay product per state
 *   carry_h [batch, d_inner, 16] fp32 out: the slice's end state from zero
 *           (rank 0: from ssm_state_in)
 * Errors: INVALID_ARG (null / misaligned, both halo sources), WORKSPACE,
 * UNSUPPORTED (too many tokens), CUDA. */
jamba_status jamba_mamba_prefill_cp_begin(jamba_mamba_t h, const void* u, const void* u_halo, int batch,
                                          int seqlen, const float* conv_state_in, const float* ssm_state_in,
                                          float* conv_state_out, float* carry_p, float* carry_h, void* ws,
                                          size_t ws_bytes, jamba_stream_t stream);

/* The state entering the slice, h_in = fold over j < rank of
 * P_j (.) h + h_j starting from zero (rank 0: h_in = ssm_state_in), then the
 * selective scan of the slice from h_in with D skip and SiLU(z) gate, and
 * out_proj.
 *   carries_p, carries_h [world][batch][d_inner][16] fp32: every rank's
 *           carry_p / carry_h in rank order (entries 0 .. rank-1 are read;
 *           may be NULL on rank 0)
 *   ssm_state_in  [batch, d_inner, 16] fp32 or NULL: rank 0 only, as in begin
 *           (INVALID_ARG on other ranks)
 *   ssm_state_out [batch, d_inner, 16] fp32: state after this rank's slice
 *           (the global final state on the last rank)
 *   out [batch, seqlen, d_model] dtype; residual as in jamba_mamba_prefill
 * Errors: INVALID_ARG, WORKSPACE, CUDA. */
jamba_status jamba_mamba_prefill_cp_finish(jamba_mamba_t h, const void* residual, void* out, int batch,
                                           int seqlen, int rank, const float* carries_p,
                                           const float* carries_h, const float* ssm_state_in,
                                           float* ssm_state_out, void* ws, size_t ws_bytes,
                                           jamba_stream_t stream);

/* ------------------------------------------------------- selective scan */

/* Bytes of workspace jamba_selective_scan needs (chunk 0 = automatic). */
jamba_status jamba_selective_scan_workspace_size(int batch, int seqlen, int d_inner, int d_state,
                                                 int chunk, size_t* bytes);

/* The selective scan with D skip and SiLU(z) gate alone (the recurrence
 * stated in the file header), batch x d_inner channels, fp32 state.
 *   x, z   [batch, seqlen, *] dtype, row strides ld_x / ld_z elements (>= d_inner)
 *   dt     [batch, seqlen, *] fp32, row stride ld_dt
 *   B, C   [batch, seqlen, *] bc_dtype, row strides ld_b / ld_c (>= d_state)
 *   A      [d_inner, d_state] fp32, D [d_inner] fp32
 *   h0     [batch, d_inner, d_state] fp32 or NULL (zeros)
 *   y      [batch, seqlen, *] dtype, row stride ld_y (a multiple of 4)
 *   h_out  [batch, d_inner, d_state] fp32 or NULL: state after the last step;
 *          may be h0 itself (in-place update: the last time chunk writes only
 *          after the first has published that it read h0), but may not
 *          overlap it otherwise
 *   chunk  time steps per chunk (multiple of 16), 0 = automatic
 * Time is split into chunks scanned concurrently; the state entering each
 * chunk is passed between chunks with a decoupled look-back, which folds the
 * carries in the order they become available: repeated calls agree up to
 * that rounding order (last bits), not bit for bit.  Errors:
 * UNSUPPORTED for d_state != 16, INVALID_ARG for strides/alignment or an
 * h_out that overlaps h0 without being it. */
jamba_status jamba_selective_scan(const void* x, int ld_x, const void* z, int ld_z, const float* dt,
                                  int ld_dt, const void* B, int ld_b, const void* C, int ld_c,
                                  int bc_dtype, const float* A, const float* D, const float* h0,
                                  void* y, int ld_y, float* h_out, int batch, int seqlen,
                                  int d_inner, int d_state, int dtype, int chunk, void* ws,
                                  size_t ws_bytes, jamba_stream_t stream);

/* jamba_selective_scan without a workspace argument, for callers that must
 * not allocate device memory.  Some callers cannot call cudaMalloc on their
 * execution path: a kernel library plugged into another framework runs inside
 * that framework's memory plan, whose allocator already owns the device
 * memory, so an extra allocation may fail or stall everything else on the
 * GPU.  This entry point allocates nothing: the scratch the scan needs (chunk
 * records, flags, tickets) is a static device array of 32 MiB that every GPU
 * loading the library holds until the process exits.  The caller still passes
 * all inputs and outputs, exactly as for jamba_selective_scan.
 *  - The paper has no counterpart to this entry point; it exists for the
 *    callers described above.
 *  - The first call on each device looks up the array's device address with
 *    that device current (a host-side runtime query, no allocation); make
 *    that first call before any stream capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; each call clears the part that must start at zero.  Calls whose
 *    execution overlaps on the GPU (different streams, no ordering between
 *    them) race on the array and give undefined results: order them.
 *  - Limit: batch * ceil(d_inner / 256) channel groups times the number of
 *    time chunks must fit the array (48 KiB per chunk record).  The automatic
 *    time chunk gives at most one record per CTA resident on the GPU, which
 *    always fits; beyond that the call takes one chunk per group, and
 *    JAMBA_ERR_UNSUPPORTED is returned (nothing launched) when even that
 *    does not fit: more than 682 groups, e.g. batch 22 at d_inner 8192
 *    (batch 21 is accepted).
 *  - status: a device int the kernel sets to JAMBA_ERR_TIMEOUT if one of its
 *    bounded waits gives up (never cleared by the library; while it is set,
 *    later calls given the same word stop early), or NULL to use a static
 *    word of the library that jamba_device_status() reads and clears.
 * Other arguments, layouts and errors: as jamba_selective_scan. */
jamba_status jamba_selective_scan_static(const void* x, int ld_x, const void* z, int ld_z, const float* dt,
                                         int ld_dt, const void* B, int ld_b, const void* C, int ld_c,
                                         int bc_dtype, const float* A, const float* D, const float* h0,
                                         void* y, int ld_y, float* h_out, int batch, int seqlen, int d_inner,
                                         int d_state, int dtype, int* status, jamba_stream_t stream);

/* Test support for the host-side planner of the bf16 prefill's scan (no GPU
 * needed): the per-group time chunks jamba_mamba_prefill gives `groups`
 * channel groups of 256 for `batch` rows of `seqlen` steps when the channels
 * of group g keep a carried state for about head[g] steps (groups ordered
 * slowest first) and `slots` CTAs fit on the device at once.  On return
 * *planned is the number of groups planned (0: the uniform chunking of
 * jamba_selective_scan is used instead), chunks[g] and lens[g] (caller
 * arrays of `groups` ints) their chunk count and length (a multiple of 16)
 * for g < *planned.  Not part of the method. */
jamba_status jamba_test_scan_plan(int batch, int seqlen, int groups, const float* head, int slots, int* chunks,
                                  int* lens, int* planned);

/* Test support for the host-side k-split choices (no GPU needed; the SM count
 * is the current device's, 148 without one): *splits is the k-split count of
 * a dense M x N x K GEMM with N-wide tiles keeping at least min_k_tiles
 * 64-deep steps per split (x_proj and out_proj at decode sizes), and
 * *i8w_splits_out that of the ExpertsInt8 fp32 expert GEMM over num_groups
 * experts whose weights take the M side.  Not part of the method. */
jamba_status jamba_test_gemm_splits(int M, int N, int K, int bn, int min_k_tiles, int num_groups, int* splits,
                                    int* i8w_splits_out);

/* Test support for jamba_mamba_prefill_host (no GPU needed): the time-chunk
 * lengths it cuts a sequence of `seqlen` steps into for a given chunk (chunk
 * above seqlen counts as seqlen), written to lens (capacity ints); *count is
 * their number (JAMBA_ERR_INVALID_ARG when above capacity).  Not part of the
 * method. */
jamba_status jamba_test_host_chunks(int seqlen, int chunk, int* lens, int capacity, int* count);

/* Test support for the bounded device waits (failure detection without a GPU
 * fault).  Runs jamba_selective_scan (same arguments, chunk > 0 and at least
 * two chunks) but launches no CTA for the first time chunk, so the flags of
 * chunk 0 are never published: every CTA whose look-back reaches chunk 0
 * gives up after wait_ns nanoseconds, latches JAMBA_ERR_TIMEOUT in the device
 * error word (read and cleared by jamba_device_status) and returns.  Every
 * load and store stays inside the caller's tensors and the workspace; y and
 * h_out hold unspecified values afterwards.  Not part of the method. */
jamba_status jamba_test_scan_missing_predecessor(const void* x, int ld_x, const void* z, int ld_z,
                                                 const float* dt, int ld_dt, const void* B, int ld_b,
                                                 const void* C, int ld_c, int bc_dtype, const float* A,
                                                 const float* D, void* y, int ld_y, float* h_out, int batch,
                                                 int seqlen, int d_inner, int d_state, int dtype, int chunk,
                                                 unsigned long long wait_ns, void* ws, size_t ws_bytes,
                                                 jamba_stream_t stream);

/* ------------------------------------------------------- building blocks */

/* out = RMSNorm(x) * w over rows of `cols` elements (block norm of the layer pair).
 * x, out [rows, cols] dtype; w [cols] fp32. */
jamba_status jamba_rmsnorm(const void* x, const float* w, void* out, int rows, int cols, float eps,
                           int dtype, jamba_stream_t stream);

/* Causal depthwise conv1d + SiLU over [batch, seqlen] tokens.
 *   x [batch, seqlen, *] dtype row stride ld_x; w [channels, 4] dtype; b [channels] dtype
 *   out [batch, seqlen, channels] dtype (contiguous)
 *   state_in / state_out [batch, channels, 3] fp32 or NULL (see jamba_mamba_prefill) */
jamba_status jamba_causal_conv1d(const void* x, int ld_x, const void* w, const void* b, void* out,
                                 const float* state_in, float* state_out, int batch, int seqlen,
                                 int channels, int dtype, jamba_stream_t stream);

/* in_proj with the causal conv1d + SiLU in its epilogue (bf16): the first step
 * of jamba_mamba_prefill on a bf16 handle, as its own call (Jamba section 2's
 * Mamba layer: in_proj, then the conv over the x half).  Two launches: the
 * tcgen05 GEMM, whose epilogue runs the conv over each 32-token slab it
 * holds, and a small kernel for the rows 0-2 of each slab whose window reaches
 * the slab above.
 *   u [batch * seqlen, d_model] bf16; w_in [2 * d_inner, d_model] bf16 (x rows, then z rows)
 *   conv_w [d_inner, 4], conv_b [d_inner] bf16, 16-byte aligned
 *   xz [batch * seqlen, 2 * d_inner] bf16: z in columns d_inner.. (its x
 *      columns are scratch: raw x of six rows in every 32)
 *   xc [batch * seqlen, d_inner] bf16: SiLU(conv(x)), x the bf16 in_proj output
 *   state_in / state_out [batch, d_inner, 3] fp32 or NULL, not aliased (as in
 *      jamba_mamba_prefill)
 * JAMBA_ERR_UNSUPPORTED unless seqlen >= 3 and d_inner is a multiple of 32 of
 * at least 128 (jamba_gemm then jamba_causal_conv1d compute the same). */
jamba_status jamba_in_proj_conv1d(const void* u, const void* w_in, const void* conv_w, const void* conv_b,
                                  void* xz, void* xc, const float* state_in, float* state_out, int batch,
                                  int seqlen, int d_model, int d_inner, jamba_stream_t stream);

/* Dense GEMM out = a @ b^T (+ residual) on the sm_100a tensor cores (bf16) or
 * the CUDA cores (fp32).  a [m, k], b [n, k] row-major; out [m, n] row stride
 * ld_out; residual NULL or [m, n] with the same stride.  out_dtype may differ
 * from dtype only as fp32 output of bf16 inputs. */
jamba_status jamba_gemm(const void* a, const void* b, void* out, int ld_out, const void* residual,
                        int m, int n, int k, int dtype, int out_dtype, jamba_stream_t stream);

/* -------------------------------------------------------------------- MoE */

typedef struct jamba_moe_config {
  int d_model;      /* 4096 */
  int d_ff;         /* expert hidden width (14336), multiple of 128 */
  int n_experts;    /* n (16 in Jamba section 3.1), at most 64 */
  int top_k;        /* K (2 in Jamba section 3.1), 1 or 2 */
  int dtype;        /* JAMBA_BF16: activations and router */
  int expert_dtype; /* JAMBA_BF16: w_gate / w_up / w_down in bf16;
                       JAMBA_INT8: ExpertsInt8 (Jamba-1.5 article, section on
                       ExpertsInt8): the three expert matrices hold int8 codes
                       q with one fp32 scale per output row (see
                       jamba_quantize_int8_rows); the weight is q * scale and
                       is widened to bf16 inside the expert GEMM kernels, the
                       scale applied to the fp32 accumulator.  Activations and
                       the router stay bf16. */
} jamba_moe_config;

typedef struct jamba_moe_weights {
  const void* router; /* [n_experts, d_model] dtype */
  const void* w_gate; /* [n_experts, d_ff, d_model] expert_dtype */
  const void* w_up;   /* [n_experts, d_ff, d_model] expert_dtype */
  const void* w_down; /* [n_experts, d_model, d_ff] expert_dtype */
  const float* s_gate; /* JAMBA_INT8 only: [n_experts, d_ff] row scales of w_gate (else NULL) */
  const float* s_up;   /* JAMBA_INT8 only: [n_experts, d_ff] row scales of w_up */
  const float* s_down; /* JAMBA_INT8 only: [n_experts, d_model] row scales of w_down */
} jamba_moe_weights;

/* Per-row symmetric INT8 quantisation, the ExpertsInt8 weight format (no
 * calibration data: every row is quantised from its own values).
 *   w     [rows, cols] dtype (JAMBA_BF16 or JAMBA_F32), row-major, contiguous
 *   q     [rows, cols] int8 out
 *   scale [rows] fp32 out
 * For each row, in fp32 with IEEE division: scale = max|w| / 127 and
 * q = round-half-even(w / scale), an integer in [-127, 127]; an all-zero row
 * gives scale = 0 and q = 0.  cols must be a multiple of 8 and every pointer
 * 16-byte aligned; JAMBA_ERR_INVALID_ARG otherwise.  Deterministic: the
 * output depends only on w. */
jamba_status jamba_quantize_int8_rows(const void* w, int dtype, long long rows, int cols, int8_t* q,
                                      float* scale, jamba_stream_t stream);

jamba_status jamba_moe_workspace_size(const jamba_moe_config* cfg, int tokens, size_t* bytes);

/* Top-K-of-n SwiGLU mixture of experts on `tokens` rows (Jamba section 2).
 *   x        [tokens, d_model] dtype (already block-normed)
 *   residual [tokens, d_model] dtype or NULL, added to the output
 *   y        [tokens, d_model] dtype
 *   topk_idx [tokens, top_k] int32 out: experts by descending logit, ties to the lower index
 *   topk_w   [tokens, top_k] fp32 out: their softmax probabilities (not renormalised)
 *   expert_offsets [n_experts + 1] int32 out: routed-row ranges per expert
 *   perm     [tokens * top_k] int32 out: routed row p holds pair (token, slot) = perm[p]
 *            as token * top_k + slot, rows sorted by (expert, token, slot)
 * Router logits are accumulated in fp64 from the bf16 inputs, so the expert
 * choice is the exact-arithmetic one except for ties closer than 1e-13. */
jamba_status jamba_moe_forward(const jamba_moe_config* cfg, const jamba_moe_weights* w,
                               const void* x, const void* residual, void* y, int tokens,
                               int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                               int32_t* perm, void* ws, size_t ws_bytes, jamba_stream_t stream);

/* ------------------------------------------------- expert-parallel MoE */

/* The top-K MoE with its experts split over ranks (expert parallelism; the
 * news article names MoE parallelism as a future speed-up, the summary page
 * expert parallelism among its training parallelisms; no scheme is given).
 * Each rank routes its own tokens, sends every routed row to the rank that
 * owns its expert, runs its share of the experts on what it receives, and
 * gets the results back; the caller does the two all-to-alls (and one of the
 * per-expert row counts) between the calls.  Rank r owns experts
 * [r E / world, (r + 1) E / world); a rank's routed rows are already in
 * (expert, token, slot) order, so the rows for rank r are one contiguous
 * range: expert_offsets[r E / world] .. expert_offsets[(r + 1) E / world].
 *
 * dispatch (cfg: the whole MoE, n_experts = E; router [E, d_model]):
 *   routing as in jamba_moe_forward, and send_rows [tokens * top_k, d_model]
 *   dtype, the routed rows in that order.  ws: jamba_moe_workspace_size(cfg,
 *   tokens); it keeps the inverse permutation for combine: pass it unchanged.
 * experts (cfg: this rank's share, n_experts = E / world; w: its w_gate /
 *   w_up / w_down [and scales]; router unused):
 *   rows_in [rows, d_model] dtype: the rows received, grouped by source rank
 *   and, within one source, by local expert; group_counts [world * E_local]
 *   int32 on the device: rows of (source s, local expert e) at s * E_local + e.
 *   rows_out [rows, d_model] fp32: the expert outputs, same order.
 *   ws: jamba_moe_ep_experts_workspace_size(cfg, rows, world).
 * combine (cfg: the whole MoE): rows_back [tokens * top_k, d_model] fp32, the
 *   expert outputs of this rank's routed rows in routed order; y = the
 *   top-K weighted sum (+ residual), as jamba_moe_forward.
 * Errors: INVALID_ARG, UNSUPPORTED (as jamba_moe_forward), WORKSPACE, CUDA. */
jamba_status jamba_moe_ep_dispatch(const jamba_moe_config* cfg, const void* router, const void* x, int tokens,
                                   int32_t* topk_idx, float* topk_w, int32_t* expert_offsets, int32_t* perm,
                                   void* send_rows, void* ws, size_t ws_bytes, jamba_stream_t stream);
jamba_status jamba_moe_ep_experts_workspace_size(const jamba_moe_config* cfg, int rows, int world,
                                                 size_t* bytes);
jamba_status jamba_moe_ep_experts(const jamba_moe_config* cfg, const jamba_moe_weights* w, const void* rows_in,
                                  int rows, const int32_t* group_counts, int world, float* rows_out, void* ws,
                                  size_t ws_bytes, jamba_stream_t stream);
jamba_status jamba_moe_ep_combine(const jamba_moe_config* cfg, const float* rows_back, const float* topk_w,
                                  int tokens, const void* residual, void* y, void* ws, size_t ws_bytes,
                                  jamba_stream_t stream);


/* ------------------------------------------------------------- attention */

/* The Jamba block's attention layer ("Jamba: A Hybrid Transformer-Mamba
 * Language Model", section 2: one layer in eight; standard details including
 * grouped-query attention; no explicit positional information, so no
 * positional embedding or RoPE).  Query head h reads KV head
 * h / (n_heads / n_kv_heads); causal softmax of q . k / sqrt(head_dim);
 * projections without bias. */
typedef struct jamba_attn_config {
  int d_model;    /* 4096 */
  int n_heads;    /* query heads (32 at Jamba width) */
  int n_kv_heads; /* key/value heads, divides n_heads (8 at Jamba width) */
  int head_dim;   /* 128 (the only width supported) */
  int dtype;      /* JAMBA_BF16 */
} jamba_attn_config;

typedef struct jamba_attn_weights {
  const void* w_qkv; /* [(n_heads + 2 n_kv_heads) * head_dim, d_model]: W_q rows, then W_k, then W_v */
  const void* w_o;   /* [d_model, n_heads * head_dim] */
} jamba_attn_weights;

jamba_status jamba_attn_prefill_workspace_size(const jamba_attn_config* cfg, int batch, int seqlen, size_t* bytes);

/* Causal attention over `seqlen` tokens of each of `batch` sequences.
 *   x        [batch, seqlen, d_model] dtype (already block-normed)
 *   residual [batch, seqlen, d_model] or NULL, added to the output
 *   out      [batch, seqlen, d_model] (may not alias x)
 *   k_cache, v_cache  NULL, or [batch, n_kv_heads, max_len, head_dim] dtype:
 *            positions 0..seqlen-1 are written (max_len >= seqlen)
 * The workspace holds the fused q|k|v rows, V transposed and the attention
 * output before out_proj.  seqlen >= 1; no other limit than the workspace. */
jamba_status jamba_attn_prefill(const jamba_attn_config* cfg, const jamba_attn_weights* w, const void* x,
                                const void* residual, void* out, int batch, int seqlen, void* k_cache,
                                void* v_cache, int max_len, void* ws, size_t ws_bytes, jamba_stream_t stream);

jamba_status jamba_attn_step_workspace_size(const jamba_attn_config* cfg, int batch, int max_len, size_t* bytes);

/* One decode token per sequence (at most 8 query heads per KV head;
 * JAMBA_ERR_UNSUPPORTED otherwise).
 *   x [batch, d_model]; residual [batch, d_model] or NULL; out [batch, d_model]
 *   k_cache, v_cache [batch, n_kv_heads, max_len, head_dim]
 *   lengths [batch] int32 device array: tokens already cached per sequence.
 *            The new token's k and v are written at position lengths[b], the
 *            token attends to positions 0..lengths[b], and lengths[b] is then
 *            incremented (so a captured CUDA graph can be replayed step after
 *            step).  Lengths are device data, so the host cannot check them:
 *            for a sequence whose length is outside [0, max_len) nothing is
 *            appended, no cache position at or past max_len is read, and its
 *            output row is unspecified; the caller keeps lengths < max_len. */
jamba_status jamba_attn_step(const jamba_attn_config* cfg, const jamba_attn_weights* w, const void* x,
                             const void* residual, void* out, int batch, void* k_cache, void* v_cache,
                             int max_len, int32_t* lengths, void* ws, size_t ws_bytes, jamba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* JAMBA_H_ */
