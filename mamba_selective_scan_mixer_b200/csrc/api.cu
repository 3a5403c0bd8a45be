// C ABI: argument checks, workspace layout and the launch sequences of the
// Mamba mixer (prefill, decode step), the selective scan alone, the building
// blocks and the MoE.  See include/jamba.h for the contract of each call.
#include <algorithm>
#include <cmath>
#include <new>
#include <numeric>
#include <string>
#include <vector>

#include "gemm_tc.cuh"
#include "host.hpp"

using namespace jb;

struct jamba_mamba {
  jamba_mamba_config cfg;
  jamba_mamba_weights w;
  int device;
  int a_form;   // ScanAForm of A, read once at create: picks the one scan kernel to launch
  // bf16 mixers, prefill only: the channels reordered by how long they carry
  // state (slowest decay first) so that the scan's channel groups hold
  // channels of like speed.  wp holds the reordered weights (in `own`), perm
  // maps a reordered channel to its cache row (the caller's channel), head[g]
  // is the number of steps after which group g's slowest channel has lost the
  // carried state.  Decode steps use the caller's weights and order.
  jamba_mamba_weights wp;
  void* own = nullptr;
  int* perm = nullptr;
  std::vector<float> head;
  // host-buffer prefill pipeline: two copy streams and the events that order
  // the double-buffered chunks (created on first use)
  cudaStream_t io_in = nullptr, io_out = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
};

namespace {

constexpr size_t kAlign = 256;
inline size_t al(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// Sequential carve-out of a workspace; with a null base it only measures.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(reinterpret_cast<uint8_t*>(b)) {}
  template <typename T = void>
  T* take(size_t bytes) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += al(bytes);
    return p;
  }
};

inline int esize(int dtype) { return dtype == JAMBA_BF16 ? 2 : 4; }
inline cudaStream_t cs(jamba_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

struct PrefillWs {
  void* xz; void* xc; float* xpart; void* dtlow; float* bc; float* dt; void* y; float* conv_tmp; void* scan;
  size_t scan_bytes;
  int splits, chunk;
  // context-parallel prefill only: in_proj rows of the 3 input tokens before
  // the slice, the conv cache they make, and the state entering the slice
  void* xz_halo; float* conv_halo; float* h_in;
  ScanSchedule sched;   // the scan's per-group time chunks (n == 0: uniform chunks of `chunk`)
  size_t total;
};

// The scan's time chunks for one prefill call: per channel group when the
// handle has reordered its channels, else uniform.
void plan_scan(const jamba_mamba* h, int batch, int L, ScanSchedule* out) {
  out->n = 0;
  if (h->perm) {
    const int groups = (int)h->head.size();
    scan_plan(batch, L, groups, h->head.data(), scan_slots(h->cfg.dtype, JAMBA_F32), out);
  }
}

PrefillWs carve_prefill(const jamba_mamba* h, int batch, int L, void* ws, bool cp = false) {
  const jamba_mamba_config& c = h->cfg;
  PrefillWs p;
  const size_t T = (size_t)batch * L;
  const int es = esize(c.dtype);
  const int W = c.dt_rank + 2 * c.d_state;
  p.splits = c.dtype == JAMBA_BF16 ? choose_splits((int)T, W, c.d_inner, 144, 8) : 1;
  p.chunk = scan_auto_chunk(batch, L, c.d_inner, c.dtype, JAMBA_F32);
  Carver cv(ws);
  p.xz = cv.take(T * 2 * c.d_inner * es);
  p.xc = cv.take(T * c.d_inner * es);
  p.xpart = cv.take<float>((size_t)p.splits * T * W * 4);
  p.dtlow = cv.take(T * c.dt_rank * es);
  p.bc = cv.take<float>(T * 2 * c.d_state * 4);
  p.dt = cv.take<float>(T * c.d_inner * 4);
  p.y = cv.take(T * c.d_inner * es);
  p.conv_tmp = cv.take<float>((size_t)batch * c.d_inner * (c.d_conv - 1) * 4);
  plan_scan(h, batch, L, &p.sched);
  if (h->perm) {
    // a per-group plan never exceeds the resident CTAs; sized for that bound
    // so that shorter calls (the host pipeline's ramp chunks) always fit
    const size_t uni = scan_records(batch, L, c.d_inner, p.chunk, nullptr);
    const size_t cap = (size_t)scan_slots(c.dtype, JAMBA_F32);
    p.scan_bytes = scan_records_bytes(uni > cap ? uni : cap);
  } else {
    p.scan_bytes = scan_workspace_bytes(batch, L, c.d_inner, p.chunk);
  }
  p.scan = cv.take(p.scan_bytes);
  p.xz_halo = p.conv_halo = p.h_in = nullptr;
  if (cp) {
    p.xz_halo = cv.take((size_t)batch * (c.d_conv - 1) * 2 * c.d_inner * es);
    p.conv_halo = cv.take<float>((size_t)batch * c.d_inner * (c.d_conv - 1) * 4);
    p.h_in = cv.take<float>((size_t)batch * c.d_inner * c.d_state * 4);
  }
  p.total = cv.off;
  return p;
}


struct StepWs {
  void* xz; void* xc; float* xpart; void* dtlow; float* bc; float* dt; void* y; float* opart;
  int x_splits, o_splits;
  size_t total;
};

StepWs carve_step(const jamba_mamba_config& c, int batch, void* ws) {
  StepWs p;
  const int es = esize(c.dtype);
  const int W = c.dt_rank + 2 * c.d_state;
  const bool tc = c.dtype == JAMBA_BF16;
  p.x_splits = tc ? choose_splits(W, batch, c.d_inner, 64, 4) : 1;
  p.o_splits = tc ? choose_splits(c.d_model, batch, c.d_inner, 64, 8) : 1;
  Carver cv(ws);
  p.xz = cv.take((size_t)batch * 2 * c.d_inner * es);
  p.xc = cv.take((size_t)batch * c.d_inner * es);
  p.xpart = cv.take<float>((size_t)p.x_splits * batch * W * 4);
  p.dtlow = cv.take((size_t)batch * c.dt_rank * es);
  p.bc = cv.take<float>((size_t)batch * 2 * c.d_state * 4);
  p.dt = cv.take<float>((size_t)batch * c.d_inner * 4);
  p.y = cv.take((size_t)batch * c.d_inner * es);
  p.opart = cv.take<float>((size_t)p.o_splits * batch * c.d_model * 4);
  p.total = cv.off;
  return p;
}

GemmDesc gdesc(const void* a, long long lda, const void* b, long long ldb, int M, int N, int K, int epi, void* out,
               long long ldo) {
  GemmDesc g = {};
  g.a = a; g.lda = lda; g.b = b; g.ldb = ldb; g.M = M; g.N = N; g.K = K; g.epi = epi; g.out = out; g.ldo = ldo;
  g.splits = 1;
  return g;
}

jamba_status gemm_any(int dtype, const GemmDesc& g, cudaStream_t s) {
  return dtype == JAMBA_BF16 ? gemm_bf16(g, s) : gemm_f32(g, s);
}

jamba_status check_dtype(int d) {
  return (d == JAMBA_BF16 || d == JAMBA_F32) ? JAMBA_OK : fail(JAMBA_ERR_UNSUPPORTED, "dtype must be JAMBA_F32 or JAMBA_BF16");
}

jamba_status check_ptr(const void* p, const char* name, bool required = true) {
  if (!p) return required ? fail(JAMBA_ERR_INVALID_ARG, std::string(name) + " is null") : JAMBA_OK;
  if (!aligned16(p)) return fail(JAMBA_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  return JAMBA_OK;
}

jamba_status check_device(const jamba_mamba* h) {
  int dev = -1;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev != h->device) return fail(JAMBA_ERR_INVALID_ARG, "handle was created on another device");
  return JAMBA_OK;
}

// Sort the channels by their slowest decay, softplus(dt_bias[c]) *
// min_n |A[c, n]| (the decay rate when dt sits at its bias), slowest first,
// and keep a copy of every channel-indexed weight in that order for the
// prefill: in_proj rows (x and z halves), conv weight and bias, x_proj
// columns, dt_proj rows and bias, A, D and out_proj columns (the norm weights
// are not channel-indexed).  Caches stay in the caller's channel order (the
// prefill kernels index them through perm).  Synchronous: it reads dt_bias
// and A back to the host.
jamba_status reorder_channels(jamba_mamba* h) {
  const jamba_mamba_config& c = h->cfg;
  const jamba_mamba_weights w = h->w;
  const int di = c.d_inner, dm = c.d_model, R = c.dt_rank, N = c.d_state, W = R + 2 * N;
  const size_t es = 2;   // bf16 weights
  std::vector<float> bias(di), A((size_t)di * N);
  JB_CUDA(cudaMemcpy(bias.data(), w.dt_bias, sizeof(float) * di, cudaMemcpyDeviceToHost));
  JB_CUDA(cudaMemcpy(A.data(), w.A, sizeof(float) * A.size(), cudaMemcpyDeviceToHost));
  std::vector<double> rate(di);
  for (int ch = 0; ch < di; ++ch) {
    const double b = bias[ch];
    const double dt = b > 30.0 ? b : std::log1p(std::exp(b));
    double amin = INFINITY;
    for (int n = 0; n < N; ++n) amin = std::min(amin, std::fabs((double)A[(size_t)ch * N + n]));
    rate[ch] = std::isfinite(dt * amin) ? dt * amin : 0.0;
  }
  std::vector<int> perm(di);
  std::iota(perm.begin(), perm.end(), 0);
  std::stable_sort(perm.begin(), perm.end(), [&](int a, int b) { return rate[a] < rate[b]; });
  // steps until a group's slowest channel has decayed the carried state below the scan's drop threshold (2^-32)
  const int groups = (di + SCAN_GROUP_CHANNELS - 1) / SCAN_GROUP_CHANNELS;
  h->head.assign(groups, 0.f);
  for (int g = 0; g < groups; ++g) {
    const double r = rate[perm[(size_t)g * SCAN_GROUP_CHANNELS]];
    h->head[g] = r > 0.0 ? (float)std::min(32.0 * std::log(2.0) / r, 1e9) : 1e9f;
  }

  Carver cv(nullptr);
  const size_t o_in = (size_t)cv.off; cv.take((size_t)2 * di * dm * es);
  const size_t o_cw = cv.off; cv.take((size_t)di * 4 * es);
  const size_t o_cb = cv.off; cv.take((size_t)di * es);
  const size_t o_x = cv.off; cv.take((size_t)W * di * es);
  const size_t o_dtp = cv.off; cv.take((size_t)di * R * es);
  const size_t o_dtb = cv.off; cv.take((size_t)di * 4);
  const size_t o_A = cv.off; cv.take((size_t)di * N * 4);
  const size_t o_D = cv.off; cv.take((size_t)di * 4);
  const size_t o_out = cv.off; cv.take((size_t)dm * di * es);
  const size_t o_p = cv.off; cv.take((size_t)di * 4);
  void* buf = nullptr;
  if (cudaMalloc(&buf, cv.off) != cudaSuccess) {
    cudaGetLastError();
    return fail(JAMBA_ERR_OOM, "create: no device memory for the reordered weights");
  }
  h->own = buf;
  uint8_t* base = reinterpret_cast<uint8_t*>(buf);
  int* dperm = reinterpret_cast<int*>(base + o_p);
  JB_CUDA(cudaMemcpy(dperm, perm.data(), sizeof(int) * di, cudaMemcpyHostToDevice));
  cudaStream_t s = 0;
  const uint8_t* in = reinterpret_cast<const uint8_t*>(w.in_proj);
  JB_TRY(gather_rows(in, base + o_in, dperm, di, (int)(dm * es), s));
  JB_TRY(gather_rows(in + (size_t)di * dm * es, base + o_in + (size_t)di * dm * es, dperm, di, (int)(dm * es), s));
  JB_TRY(gather_rows(w.conv_w, base + o_cw, dperm, di, (int)(4 * es), s));
  JB_TRY(gather_rows(w.conv_b, base + o_cb, dperm, di, (int)es, s));
  JB_TRY(gather_cols(w.x_proj, base + o_x, dperm, W, di, (int)es, s));
  JB_TRY(gather_rows(w.dt_proj, base + o_dtp, dperm, di, (int)(R * es), s));
  JB_TRY(gather_rows(w.dt_bias, base + o_dtb, dperm, di, 4, s));
  JB_TRY(gather_rows(w.A, base + o_A, dperm, di, N * 4, s));
  JB_TRY(gather_rows(w.D, base + o_D, dperm, di, 4, s));
  JB_TRY(gather_cols(w.out_proj, base + o_out, dperm, dm, di, (int)es, s));
  JB_CUDA(cudaStreamSynchronize(s));
  jamba_mamba_weights& o = h->wp;
  o = h->w;
  o.in_proj = base + o_in;
  o.conv_w = base + o_cw;
  o.conv_b = base + o_cb;
  o.x_proj = base + o_x;
  o.dt_proj = base + o_dtp;
  o.dt_bias = reinterpret_cast<const float*>(base + o_dtb);
  o.A = reinterpret_cast<const float*>(base + o_A);
  o.D = reinterpret_cast<const float*>(base + o_D);
  o.out_proj = base + o_out;
  h->perm = dperm;
  return JAMBA_OK;
}

// The weights the prefill runs on: the reordered copy when the handle has one.
const jamba_mamba_weights& prefill_weights(const jamba_mamba& h) { return h.perm ? h.wp : h.w; }

// bf16 in_proj with the conv + SiLU in its epilogue, then the slab rows it
// deferred: z into xz (its x columns are scratch), SiLU(conv(x)) into xc.
jamba_status in_proj_conv(const void* u, const void* w_in, const void* conv_w, const void* conv_b, void* xz, void* xc,
                          const float* cin, float* cout, const int* perm, int T, int seqlen, int dm, int di,
                          cudaStream_t s) {
  GemmDesc g = gdesc(u, dm, w_in, dm, T, 2 * di, dm, EPI_CONVP, xz, 2 * di);
  g.conv_w = conv_w; g.conv_b = conv_b; g.xc_out = xc; g.conv_c = di;
  g.conv_in = cin; g.conv_out = cout; g.conv_perm = perm; g.conv_L = seqlen;
  JB_TRY(gemm_bf16(g, s));
  NvtxRange r("conv1d_slab_rows");
  return conv_fixup(xz, 2 * di, conv_w, conv_b, xc, cin, T, seqlen, di, perm, s);
}

// The prefill's first steps: in_proj, conv + SiLU (cache in -> out), x_proj
// into split-K partials (p.xpart, p.splits of them).
jamba_status prefill_front_a(const jamba_mamba& h, const PrefillWs& p, const void* u, int batch, int seqlen,
                             const float* conv_state_in, float* conv_state_out, cudaStream_t s) {
  const jamba_mamba_config& c = h.cfg;
  const jamba_mamba_weights& w = prefill_weights(h);
  const int T = batch * seqlen, di = c.d_inner, dm = c.d_model, R = c.dt_rank, N = c.d_state;
  const int W = R + 2 * N;
  NvtxSteps nv;
  // the conv cache in: an aliased one is copied first (the new cache is
  // written while the old one is still read)
  const float* cin = conv_state_in;
  if (cin && cin == conv_state_out) {
    JB_CUDA(cudaMemcpyAsync(p.conv_tmp, cin, sizeof(float) * (size_t)batch * di * 3, cudaMemcpyDeviceToDevice, s));
    cin = p.conv_tmp;
  }
  if (c.dtype == JAMBA_BF16 && seqlen >= 3 && di % 32 == 0 && di >= 128 && aligned16(w.conv_w) &&
      aligned16(w.conv_b)) {
    // in_proj with the conv + SiLU in its epilogue: z into xz, xc directly;
    // the few rows whose window crosses a 32-row slab are finished after it
    nv.next("in_proj_conv1d");
    JB_TRY(in_proj_conv(u, w.in_proj, w.conv_w, w.conv_b, p.xz, p.xc, cin, conv_state_out, h.perm, T, seqlen, dm,
                        di, s));
  } else {
    // in_proj: xz = u W_in^T, then conv + SiLU (cache in -> out)
    nv.next("in_proj");
    JB_TRY(gemm_any(c.dtype, gdesc(u, dm, w.in_proj, dm, T, 2 * di, dm, c.dtype == JAMBA_BF16 ? EPI_BF16 : EPI_F32,
                                   p.xz, 2 * di), s));
    nv.next("conv1d");
    JB_TRY(conv_prefill(p.xz, 2 * di, w.conv_w, w.conv_b, p.xc, cin, conv_state_out, batch, seqlen, di, c.dtype,
                        h.perm, s));
  }
  // x_proj (split-K partials) -> sum + inner RMSNorms
  nv.next("x_proj");
  GemmDesc gx = gdesc(p.xc, di, w.x_proj, di, T, W, di, EPI_F32, p.xpart, W);
  gx.splits = p.splits;
  gx.split_stride = (long long)T * W;
  if (c.dtype == JAMBA_BF16) gx.bn = 144;
  return gemm_any(c.dtype, gx, s);
}

// Then: the x_proj sum (`splits` fp32 partials of [T, R + 2N] at `part`) through
// the inner RMSNorms into dt_low and B|C, and dt = softplus(dt_low W_dt^T + dt_bias).
jamba_status prefill_front_b(const jamba_mamba& h, const PrefillWs& p, const float* part, int splits, int batch,
                             int seqlen, cudaStream_t s) {
  const jamba_mamba_config& c = h.cfg;
  const jamba_mamba_weights& w = prefill_weights(h);
  const int T = batch * seqlen, di = c.d_inner, R = c.dt_rank, N = c.d_state;
  const int W = R + 2 * N;
  NvtxSteps nv;
  nv.next("x_proj_sum_norms");
  JB_TRY(xproj_norm(part, splits, (long long)T * W, T, R, N, w.norm_dt, w.norm_B, w.norm_C, c.inner_rmsnorm, c.eps,
                    p.dtlow, p.bc, c.dtype, s));
  nv.next("dt_proj_softplus");
  GemmDesc gd = gdesc(p.dtlow, R, w.dt_proj, R, T, di, R, EPI_SOFTPLUS, p.dt, di);
  gd.bias = w.dt_bias;
  return gemm_any(c.dtype, gd, s);
}

// The prefill up to the scan's inputs: in_proj, conv + SiLU (cache in -> out),
// x_proj, inner RMSNorms, dt_proj + softplus.
jamba_status prefill_front(const jamba_mamba& h, const PrefillWs& p, const void* u, int batch, int seqlen,
                           const float* conv_state_in, float* conv_state_out, cudaStream_t s) {
  JB_TRY(prefill_front_a(h, p, u, batch, seqlen, conv_state_in, conv_state_out, s));
  return prefill_front_b(h, p, p.xpart, p.splits, batch, seqlen, s);
}

// The scan's arguments over the front's outputs.
ScanCall scan_call(const jamba_mamba& h, const PrefillWs& p, int batch, int seqlen) {
  const jamba_mamba_config& c = h.cfg;
  const int di = c.d_inner, N = c.d_state;
  ScanCall sc = {};
  sc.x = p.xc; sc.ld_x = di;
  sc.z = reinterpret_cast<const uint8_t*>(p.xz) + (size_t)di * esize(c.dtype); sc.ld_z = 2 * di;
  sc.dt = p.dt; sc.ld_dt = di;
  sc.B = p.bc; sc.ld_b = 2 * N;
  sc.C = p.bc + N; sc.ld_c = 2 * N;
  sc.bc_dtype = JAMBA_F32;
  sc.A = prefill_weights(h).A; sc.D = prefill_weights(h).D;
  sc.y = p.y; sc.ld_y = di;
  sc.batch = batch; sc.L = seqlen; sc.di = di; sc.dtype = c.dtype; sc.chunk = p.chunk;
  sc.ws = p.scan; sc.ws_bytes = p.scan_bytes;
  sc.a_form = h.a_form;
  sc.sched = &p.sched;
  sc.perm = h.perm;
  return sc;
}

// The prefill from the scan on: selective scan + D skip + SiLU(z) gate, out_proj (+ residual).
jamba_status prefill_back(const jamba_mamba& h, const PrefillWs& p, int batch, int seqlen, const float* ssm_state_in,
                          float* ssm_state_out, const void* residual, void* out, cudaStream_t s) {
  const jamba_mamba_config& c = h.cfg;
  const int T = batch * seqlen, di = c.d_inner, dm = c.d_model;
  NvtxSteps nv;
  nv.next("selective_scan");
  ScanCall sc = scan_call(h, p, batch, seqlen);
  sc.h0 = ssm_state_in;   // may be ssm_state_out itself: the scan orders the in-place update
  sc.h_out = ssm_state_out;
  JB_TRY(scan_run(sc, s));
  nv.next("out_proj");
  GemmDesc go = gdesc(p.y, di, prefill_weights(h).out_proj, di, T, dm, di, c.dtype == JAMBA_BF16 ? EPI_BF16 : EPI_F32, out, dm);
  go.residual = residual;
  go.ldr = dm;
  return gemm_any(c.dtype, go, s);
}

}  // namespace

extern "C" {

const char* jamba_last_error(void) { return jb::last_error(); }

int jamba_checked_build(void) {
#ifdef JAMBA_CHECKS
  return 1;
#else
  return 0;
#endif
}

jamba_status jamba_device_status(jamba_stream_t stream) {
  JB_CUDA(cudaStreamSynchronize(cs(stream)));
  int* w = device_error_word();
  if (!w) return fail(JAMBA_ERR_CUDA, "could not allocate the device status word");
  int v = 0;
  JB_CUDA(cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) JB_CUDA(cudaMemset(w, 0, sizeof(int)));
  int vs = 0;   // the word of jamba_selective_scan_static calls made without a status argument
  JB_TRY(jb::static_scan_status_take(&vs));
  if (v == 0) v = vs;
  if (v != 0) return fail((jamba_status)v, "a device-side wait gave up");
  return JAMBA_OK;
}

// ------------------------------------------------------------------ Mamba

jamba_status jamba_mamba_create(const jamba_mamba_config* cfg, const jamba_mamba_weights* w, jamba_mamba_t* out) {
  JB_RANGE("jamba_mamba_create");
  if (!cfg || !w || !out) return fail(JAMBA_ERR_INVALID_ARG, "create: null argument");
  *out = nullptr;
  const jamba_mamba_config& c = *cfg;
  JB_TRY(check_dtype(c.dtype));
  if (c.d_state != 16) return fail(JAMBA_ERR_UNSUPPORTED, "d_state must be 16");
  if (c.d_conv != 4) return fail(JAMBA_ERR_UNSUPPORTED, "d_conv must be 4");
  if (c.d_model <= 0 || c.d_inner <= 0 || c.dt_rank <= 0) return fail(JAMBA_ERR_INVALID_ARG, "widths must be positive");
  if (c.d_model % 8 || c.d_inner % 8) return fail(JAMBA_ERR_UNSUPPORTED, "d_model and d_inner must be multiples of 8");
  if (c.dtype == JAMBA_BF16 && c.dt_rank % 8) return fail(JAMBA_ERR_UNSUPPORTED, "bf16 needs dt_rank % 8 == 0");
  if (c.dt_rank + 2 * c.d_state > 512) return fail(JAMBA_ERR_UNSUPPORTED, "dt_rank + 2 d_state above 512");
  if (!(c.eps >= 0.f)) return fail(JAMBA_ERR_INVALID_ARG, "eps must be >= 0");
  JB_TRY(check_ptr(w->in_proj, "in_proj"));
  JB_TRY(check_ptr(w->conv_w, "conv_w"));
  JB_TRY(check_ptr(w->conv_b, "conv_b"));
  JB_TRY(check_ptr(w->x_proj, "x_proj"));
  JB_TRY(check_ptr(w->dt_proj, "dt_proj"));
  JB_TRY(check_ptr(w->dt_bias, "dt_bias"));
  JB_TRY(check_ptr(w->A, "A"));
  JB_TRY(check_ptr(w->D, "D"));
  JB_TRY(check_ptr(w->out_proj, "out_proj"));
  if (c.inner_rmsnorm) {
    JB_TRY(check_ptr(w->norm_dt, "norm_dt"));
    JB_TRY(check_ptr(w->norm_B, "norm_B"));
    JB_TRY(check_ptr(w->norm_C, "norm_C"));
  }
  jamba_mamba* h = new (std::nothrow) jamba_mamba;
  if (!h) return fail(JAMBA_ERR_OOM, "create: out of host memory");
  h->cfg = c;
  h->w = *w;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return fail(JAMBA_ERR_CUDA, "create: no CUDA device");
  }
  // A decides which scan kernel owns the channels: the power form when
  // A[c, n] == (n + 1) A[c, 0] for every channel (bf16 only), else the general one
  h->a_form = jb::SCAN_A_GENERAL;
  if (c.dtype == JAMBA_BF16) {
    std::vector<float> A((size_t)c.d_inner * c.d_state);
    if (cudaMemcpy(A.data(), w->A, A.size() * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) {
      delete h;
      return fail(JAMBA_ERR_CUDA, "create: could not read A");
    }
    bool power = true;
    for (int ch = 0; ch < c.d_inner && power; ++ch)
      for (int n = 0; n < c.d_state; ++n)
        power = power && A[(size_t)ch * c.d_state + n] == (float)(n + 1) * A[(size_t)ch * c.d_state];
    h->a_form = power ? jb::SCAN_A_POWER : jb::SCAN_A_GENERAL;
  }
  if (c.dtype == JAMBA_BF16 && (c.d_inner + SCAN_GROUP_CHANNELS - 1) / SCAN_GROUP_CHANNELS <= SCAN_MAX_GROUPS) {
    const jamba_status st = reorder_channels(h);
    if (st != JAMBA_OK) {
      jamba_mamba_destroy(h);
      return st;
    }
  }
  *out = h;
  return JAMBA_OK;
}

jamba_status jamba_mamba_destroy(jamba_mamba_t h) {
  if (h) {
    if (h->own) cudaFree(h->own);
    if (h->io_in) cudaStreamDestroy(h->io_in);
    if (h->io_out) cudaStreamDestroy(h->io_out);
    for (int i = 0; i < 2; ++i) {
      if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
      if (h->ev_comp[i]) cudaEventDestroy(h->ev_comp[i]);
      if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    }
  }
  delete h;
  return JAMBA_OK;
}

jamba_status jamba_mamba_workspace_size(jamba_mamba_t h, int batch, int seqlen, size_t* bytes) {
  if (!h || !bytes || batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "workspace_size: bad argument");
  size_t a = carve_prefill(h, batch, seqlen, nullptr).total;
  if (seqlen == 1) {
    const size_t b = carve_step(h->cfg, batch, nullptr).total;
    a = a > b ? a : b;
  }
  *bytes = a;
  return JAMBA_OK;
}

jamba_status jamba_mamba_prefill(jamba_mamba_t h, const void* u, const void* residual, void* out, int batch,
                                 int seqlen, const float* conv_state_in, const float* ssm_state_in,
                                 float* conv_state_out, float* ssm_state_out, void* ws, size_t ws_bytes,
                                 jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "prefill: null handle");
  if (batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "prefill: batch and seqlen must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(u, "u"));
  JB_TRY(check_ptr(out, "out"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(conv_state_in, "conv_state_in", false));
  JB_TRY(check_ptr(ssm_state_in, "ssm_state_in", false));
  JB_TRY(check_ptr(conv_state_out, "conv_state_out", false));
  JB_TRY(check_ptr(ssm_state_out, "ssm_state_out", false));
  JB_TRY(check_ptr(ws, "workspace"));
  if (u == out) return fail(JAMBA_ERR_INVALID_ARG, "prefill: out may not alias u");
  if ((long long)batch * seqlen > (1LL << 31) / 2) return fail(JAMBA_ERR_UNSUPPORTED, "prefill: too many tokens");
  PrefillWs p = carve_prefill(h, batch, seqlen, ws);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "prefill: workspace too small");
  cudaStream_t s = cs(stream);
  JB_TRY(prefill_front(*h, p, u, batch, seqlen, conv_state_in, conv_state_out, s));
  return prefill_back(*h, p, batch, seqlen, ssm_state_in, ssm_state_out, residual, out, s);
}

// ------------------------------------------------- tensor-parallel prefill

jamba_status jamba_mamba_prefill_tp_begin(jamba_mamba_t h, const void* u, int batch, int seqlen,
                                          const float* conv_state_in, float* conv_state_out, float* xproj_part,
                                          void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_tp_begin");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "tp begin: null handle");
  if (batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "tp begin: batch and seqlen must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(u, "u"));
  JB_TRY(check_ptr(conv_state_in, "conv_state_in", false));
  JB_TRY(check_ptr(conv_state_out, "conv_state_out", false));
  JB_TRY(check_ptr(xproj_part, "xproj_part"));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_mamba_config& c = h->cfg;
  if ((long long)batch * seqlen > (1LL << 31) / 2) return fail(JAMBA_ERR_UNSUPPORTED, "tp begin: too many tokens");
  PrefillWs p = carve_prefill(h, batch, seqlen, ws);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "tp begin: workspace too small");
  cudaStream_t s = cs(stream);
  const long long T = (long long)batch * seqlen, W = c.dt_rank + 2 * c.d_state;
  JB_TRY(prefill_front_a(*h, p, u, batch, seqlen, conv_state_in, conv_state_out, s));
  // this rank's share of x_proj: its split-K partials summed (fp32)
  return splitk_reduce(p.xpart, p.splits, T * W, T * W, nullptr, xproj_part, JAMBA_F32, s);
}

jamba_status jamba_mamba_prefill_tp_finish(jamba_mamba_t h, const float* xproj_sum, int batch, int seqlen,
                                           const float* ssm_state_in, float* ssm_state_out, float* out_part,
                                           void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_tp_finish");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "tp finish: null handle");
  if (batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "tp finish: batch and seqlen must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(xproj_sum, "xproj_sum"));
  JB_TRY(check_ptr(ssm_state_in, "ssm_state_in", false));
  JB_TRY(check_ptr(ssm_state_out, "ssm_state_out", false));
  JB_TRY(check_ptr(out_part, "out_part"));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_mamba_config& c = h->cfg;
  PrefillWs p = carve_prefill(h, batch, seqlen, ws);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "tp finish: workspace too small");
  cudaStream_t s = cs(stream);
  const int T = batch * seqlen, di = c.d_inner, dm = c.d_model;
  JB_TRY(prefill_front_b(*h, p, xproj_sum, 1, batch, seqlen, s));
  ScanCall sc = scan_call(*h, p, batch, seqlen);
  sc.h0 = ssm_state_in;
  sc.h_out = ssm_state_out;
  JB_TRY(scan_run(sc, s));
  // this rank's share of out_proj (its d_inner columns), fp32
  GemmDesc go = gdesc(p.y, di, prefill_weights(*h).out_proj, di, T, dm, di, EPI_F32, out_part, dm);
  return gemm_any(c.dtype, go, s);
}

jamba_status jamba_mamba_prefill_tp_end(jamba_mamba_t h, const float* out_sum, const void* residual, void* out,
                                        int batch, int seqlen, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_tp_end");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "tp end: null handle");
  if (batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "tp end: batch and seqlen must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(out_sum, "out_sum"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(out, "out"));
  const long long n = (long long)batch * seqlen * h->cfg.d_model;
  return splitk_reduce(out_sum, 1, n, n, residual, out, h->cfg.dtype, cs(stream));
}

// ------------------------------------------------- context-parallel prefill

jamba_status jamba_mamba_cp_workspace_size(jamba_mamba_t h, int batch, int seqlen, size_t* bytes) {
  if (!h || !bytes || batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "cp workspace_size: bad argument");
  *bytes = carve_prefill(h, batch, seqlen, nullptr, true).total;
  return JAMBA_OK;
}

jamba_status jamba_mamba_prefill_cp_begin(jamba_mamba_t h, const void* u, const void* u_halo, int batch, int seqlen,
                                          const float* conv_state_in, const float* ssm_state_in,
                                          float* conv_state_out, float* carry_p, float* carry_h, void* ws,
                                          size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_cp_begin");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "cp begin: null handle");
  if (batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "cp begin: batch and seqlen must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(u, "u"));
  JB_TRY(check_ptr(u_halo, "u_halo", false));
  JB_TRY(check_ptr(conv_state_in, "conv_state_in", false));
  JB_TRY(check_ptr(ssm_state_in, "ssm_state_in", false));
  JB_TRY(check_ptr(conv_state_out, "conv_state_out"));
  JB_TRY(check_ptr(carry_p, "carry_p"));
  JB_TRY(check_ptr(carry_h, "carry_h"));
  JB_TRY(check_ptr(ws, "workspace"));
  if (u_halo && conv_state_in) return fail(JAMBA_ERR_INVALID_ARG, "cp begin: pass u_halo or conv_state_in, not both");
  if (conv_state_in && conv_state_in == conv_state_out)
    return fail(JAMBA_ERR_INVALID_ARG, "cp begin: conv_state_out may not alias conv_state_in");
  if (ssm_state_in && (ssm_state_in == carry_h || ssm_state_in == carry_p))
    return fail(JAMBA_ERR_INVALID_ARG, "cp begin: the carries may not alias ssm_state_in");
  const jamba_mamba_config& c = h->cfg;
  if ((long long)batch * seqlen > (1LL << 31) / 2) return fail(JAMBA_ERR_UNSUPPORTED, "cp begin: too many tokens");
  PrefillWs p = carve_prefill(h, batch, seqlen, ws, true);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "cp begin: workspace too small");
  cudaStream_t s = cs(stream);
  const int di = c.d_inner, dm = c.d_model, K1 = c.d_conv - 1;
  const float* cin = conv_state_in;
  if (u_halo) {
    // the conv cache entering the slice: in_proj of the d_conv - 1 input rows before it
    JB_TRY(gemm_any(c.dtype, gdesc(u_halo, dm, h->w.in_proj, dm, batch * K1, 2 * di, dm,
                                   c.dtype == JAMBA_BF16 ? EPI_BF16 : EPI_F32, p.xz_halo, 2 * di), s));
    JB_TRY(conv_halo_state(p.xz_halo, 2 * di, p.conv_halo, batch, di, c.dtype, s));
    cin = p.conv_halo;
  }
  JB_TRY(prefill_front(*h, p, u, batch, seqlen, cin, conv_state_out, s));
  // the slice's summary: its end state from ssm_state_in (or zero) and its decay product
  ScanCall sc = scan_call(*h, p, batch, seqlen);
  sc.h0 = ssm_state_in;
  sc.z = nullptr;
  sc.y = nullptr;
  sc.summary = 1;
  sc.h_out = carry_h;
  sc.p_out = carry_p;
  return scan_run(sc, s);
}

jamba_status jamba_mamba_prefill_cp_finish(jamba_mamba_t h, const void* residual, void* out, int batch, int seqlen,
                                           int rank, const float* carries_p, const float* carries_h,
                                           const float* ssm_state_in, float* ssm_state_out, void* ws, size_t ws_bytes,
                                           jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_cp_finish");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "cp finish: null handle");
  if (batch <= 0 || seqlen <= 0 || rank < 0) return fail(JAMBA_ERR_INVALID_ARG, "cp finish: bad sizes or rank");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(out, "out"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(ssm_state_in, "ssm_state_in", false));
  JB_TRY(check_ptr(ssm_state_out, "ssm_state_out"));
  JB_TRY(check_ptr(carries_p, "carries_p", rank > 0));
  JB_TRY(check_ptr(carries_h, "carries_h", rank > 0));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_mamba_config& c = h->cfg;
  PrefillWs p = carve_prefill(h, batch, seqlen, ws, true);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "cp finish: workspace too small");
  cudaStream_t s = cs(stream);
  if (rank == 0) return prefill_back(*h, p, batch, seqlen, ssm_state_in, ssm_state_out, residual, out, s);
  if (ssm_state_in) return fail(JAMBA_ERR_INVALID_ARG, "cp finish: ssm_state_in is rank 0's (it is in its carry)");
  JB_TRY(carry_combine(carries_p, carries_h, rank, nullptr, p.h_in, (long long)batch * c.d_inner * c.d_state, s));
  return prefill_back(*h, p, batch, seqlen, p.h_in, ssm_state_out, residual, out, s);
}

jamba_status jamba_mamba_step(jamba_mamba_t h, const void* u, const void* residual, void* out, int batch,
                              float* conv_state, float* ssm_state, void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_step");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "step: null handle");
  if (batch <= 0) return fail(JAMBA_ERR_INVALID_ARG, "step: batch must be positive");
  JB_TRY(check_device(h));
  JB_TRY(check_ptr(u, "u"));
  JB_TRY(check_ptr(out, "out"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(conv_state, "conv_state"));
  JB_TRY(check_ptr(ssm_state, "ssm_state"));
  JB_TRY(check_ptr(ws, "workspace"));
  if (u == out) return fail(JAMBA_ERR_INVALID_ARG, "step: out may not alias u");
  const jamba_mamba_config& c = h->cfg;
  const jamba_mamba_weights& w = h->w;
  StepWs p = carve_step(c, batch, ws);
  if (ws_bytes < p.total) return fail(JAMBA_ERR_WORKSPACE, "step: workspace too small");
  cudaStream_t s = cs(stream);
  const int di = c.d_inner, dm = c.d_model, R = c.dt_rank, N = c.d_state, W = R + 2 * N;
  NvtxSteps nv;
  if (c.dtype == JAMBA_BF16) {
    // weights stream through the tensor cores as the 128-row side; the token batch is the N side
    // in_proj with the conv step in its epilogue: x rows -> conv cache shift + SiLU -> xc, z rows -> xz
    nv.next("in_proj_conv");
    GemmDesc g1 = gdesc(w.in_proj, dm, u, dm, 2 * di, batch, dm, EPI_CONV, p.xz, 2 * di);
    g1.transpose_out = 1;
    g1.bn = 64;
    g1.conv_w = w.conv_w;
    g1.conv_b = w.conv_b;
    g1.conv_state = conv_state;
    g1.xc_out = p.xc;
    g1.conv_c = di;
    JB_TRY(gemm_bf16(g1, s));
    nv.next("x_proj");
    GemmDesc g2 = gdesc(w.x_proj, di, p.xc, di, W, batch, di, EPI_F32, p.xpart, W);
    g2.transpose_out = 1;
    g2.bn = 64;
    g2.splits = p.x_splits;
    g2.split_stride = (long long)batch * W;
    JB_TRY(gemm_bf16(g2, s));
    nv.next("x_proj_sum_norms");
    JB_TRY(xproj_norm(p.xpart, p.x_splits, (long long)batch * W, batch, R, N, w.norm_dt, w.norm_B, w.norm_C,
                      c.inner_rmsnorm, c.eps, p.dtlow, p.bc, c.dtype, s));
    nv.next("dt_proj_softplus");
    GemmDesc g3 = gdesc(w.dt_proj, R, p.dtlow, R, di, batch, R, EPI_SOFTPLUS, p.dt, di);
    g3.transpose_out = 1;
    g3.bn = 64;
    g3.bias = w.dt_bias;
    JB_TRY(gemm_bf16(g3, s));
    nv.next("state_update");
    JB_TRY(ssm_step(p.xc, reinterpret_cast<const uint8_t*>(p.xz) + (size_t)di * 2, 2 * di, p.dt, p.bc, 2 * N, w.A,
                    w.D, ssm_state, p.y, batch, di, c.dtype, s));
    nv.next("out_proj");
    GemmDesc g4 = gdesc(w.out_proj, di, p.y, di, dm, batch, di, EPI_F32, p.opart, dm);
    g4.transpose_out = 1;
    g4.bn = 64;
    g4.splits = p.o_splits;
    g4.split_stride = (long long)batch * dm;
    JB_TRY(gemm_bf16(g4, s));
    JB_TRY(splitk_reduce(p.opart, p.o_splits, (long long)batch * dm, (long long)batch * dm, residual, out, c.dtype, s));
  } else {
    JB_TRY(gemm_f32(gdesc(u, dm, w.in_proj, dm, batch, 2 * di, dm, EPI_F32, p.xz, 2 * di), s));
    JB_TRY(conv_step(p.xz, 2 * di, w.conv_w, w.conv_b, p.xc, conv_state, batch, di, c.dtype, s));
    JB_TRY(gemm_f32(gdesc(p.xc, di, w.x_proj, di, batch, W, di, EPI_F32, p.xpart, W), s));
    JB_TRY(xproj_norm(p.xpart, 1, 0, batch, R, N, w.norm_dt, w.norm_B, w.norm_C, c.inner_rmsnorm, c.eps, p.dtlow,
                      p.bc, c.dtype, s));
    GemmDesc g3 = gdesc(p.dtlow, R, w.dt_proj, R, batch, di, R, EPI_SOFTPLUS, p.dt, di);
    g3.bias = w.dt_bias;
    JB_TRY(gemm_f32(g3, s));
    JB_TRY(ssm_step(p.xc, reinterpret_cast<const uint8_t*>(p.xz) + (size_t)di * 4, 2 * di, p.dt, p.bc, 2 * N, w.A,
                    w.D, ssm_state, p.y, batch, di, c.dtype, s));
    GemmDesc g4 = gdesc(p.y, di, w.out_proj, di, batch, dm, di, EPI_F32, out, dm);
    g4.residual = residual;
    g4.ldr = dm;
    JB_TRY(gemm_f32(g4, s));
  }
  return JAMBA_OK;
}

// --------------------------------------------------------- prefill from host memory

namespace {

constexpr int kHostChunk = 16384;

size_t host_chunk_bytes(const jamba_mamba_config& c, int batch, int chunk) {
  return al((size_t)batch * chunk * c.d_model * esize(c.dtype));
}

jamba_status check_pinned(const void* p, const char* name, bool required) {
  if (!p) return required ? fail(JAMBA_ERR_INVALID_ARG, std::string(name) + " is null") : JAMBA_OK;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(JAMBA_ERR_INVALID_ARG, std::string(name) + ": not page-locked host memory");
  }
  if (at.type != cudaMemoryTypeHost)
    return fail(JAMBA_ERR_INVALID_ARG, std::string(name) + ": not page-locked host memory");
  return JAMBA_OK;
}

jamba_status ensure_io(jamba_mamba* h) {
  if (h->io_in) return JAMBA_OK;
  JB_CUDA(cudaStreamCreateWithFlags(&h->io_in, cudaStreamNonBlocking));
  JB_CUDA(cudaStreamCreateWithFlags(&h->io_out, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    JB_CUDA(cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming));
    JB_CUDA(cudaEventCreateWithFlags(&h->ev_comp[i], cudaEventDisableTiming));
    JB_CUDA(cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming));
  }
  return JAMBA_OK;
}

// columns [t0, t0 + n) of every batch row of a [batch, L, d_model] host tensor
cudaError_t copy_rows(void* dst, const void* src, size_t row_bytes, size_t src_pitch, size_t dst_pitch, int batch,
                      cudaMemcpyKind kind, cudaStream_t s) {
  return cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, row_bytes, (size_t)batch, kind, s);
}

// Time chunks of the host-memory prefill: the first and last chunks ramp
// (chunk/4, chunk/2) so that the copy-in before the first prefill and the
// copy-out after the last one, which nothing overlaps, stay short.
std::vector<int> host_chunk_lengths(int seqlen, int chunk) {
  std::vector<int> lens;
  if (seqlen >= 4 * chunk && chunk >= 64) {
    const int q = chunk / 4, hlf = chunk / 2;
    lens.push_back(q);
    lens.push_back(hlf);
    int rem = seqlen - 2 * (q + hlf);
    while (rem > 0) {
      lens.push_back(rem < chunk ? rem : chunk);
      rem -= lens.back();
    }
    lens.push_back(hlf);
    lens.push_back(q);
  } else {
    for (int t = 0; t < seqlen; t += chunk) lens.push_back(seqlen - t < chunk ? seqlen - t : chunk);
  }
  return lens;
}

}  // namespace

jamba_status jamba_test_host_chunks(int seqlen, int chunk, int* lens, int capacity, int* count) {
  if (!lens || !count || seqlen <= 0 || chunk <= 0 || capacity < 0)
    return fail(JAMBA_ERR_INVALID_ARG, "host chunks: bad argument");
  const std::vector<int> v = host_chunk_lengths(seqlen, chunk < seqlen ? chunk : seqlen);
  *count = (int)v.size();
  if ((int)v.size() > capacity) return fail(JAMBA_ERR_INVALID_ARG, "host chunks: capacity too small");
  for (size_t i = 0; i < v.size(); ++i) lens[i] = v[i];
  return JAMBA_OK;
}

jamba_status jamba_mamba_host_workspace_size(jamba_mamba_t h, int batch, int chunk, size_t* bytes) {
  if (!h || !bytes || batch <= 0 || chunk < 0) return fail(JAMBA_ERR_INVALID_ARG, "host workspace_size: bad argument");
  if (chunk == 0) chunk = kHostChunk;
  size_t pre = 0;
  JB_TRY(jamba_mamba_workspace_size(h, batch, chunk, &pre));
  // prefill workspace, then u, residual and out chunk buffers, two of each
  *bytes = al(pre) + 6 * host_chunk_bytes(h->cfg, batch, chunk);
  return JAMBA_OK;
}

jamba_status jamba_mamba_prefill_host(jamba_mamba_t h, const void* u_host, const void* residual_host, void* out_host,
                                      int batch, int seqlen, int chunk, const float* conv_state_in,
                                      const float* ssm_state_in, float* conv_state_out, float* ssm_state_out,
                                      void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_mamba_prefill_host");
  if (!h) return fail(JAMBA_ERR_INVALID_ARG, "prefill_host: null handle");
  if (batch <= 0 || seqlen <= 0 || chunk < 0)
    return fail(JAMBA_ERR_INVALID_ARG, "prefill_host: batch and seqlen must be positive, chunk >= 0");
  JB_TRY(check_device(h));
  JB_TRY(check_pinned(u_host, "u_host", true));
  JB_TRY(check_pinned(out_host, "out_host", true));
  JB_TRY(check_pinned(residual_host, "residual_host", false));
  if (u_host == out_host) return fail(JAMBA_ERR_INVALID_ARG, "prefill_host: out_host may not alias u_host");
  JB_TRY(check_ptr(conv_state_out, "conv_state_out"));
  JB_TRY(check_ptr(ssm_state_out, "ssm_state_out"));
  JB_TRY(check_ptr(ws, "workspace"));
  if (chunk == 0) chunk = kHostChunk;
  if (chunk > seqlen) chunk = seqlen;
  size_t need = 0;
  JB_TRY(jamba_mamba_host_workspace_size(h, batch, chunk, &need));
  if (ws_bytes < need) return fail(JAMBA_ERR_WORKSPACE, "prefill_host: workspace too small");
  JB_TRY(ensure_io(h));
  const jamba_mamba_config& c = h->cfg;
  const size_t es = (size_t)esize(c.dtype), tok = (size_t)c.d_model * es;   // bytes per token row
  size_t pre = 0;
  JB_TRY(jamba_mamba_workspace_size(h, batch, chunk, &pre));
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  const size_t cb = host_chunk_bytes(c, batch, chunk);
  uint8_t* in_buf[2] = {base + al(pre), base + al(pre) + cb};
  uint8_t* res_buf[2] = {base + al(pre) + 2 * cb, base + al(pre) + 3 * cb};
  uint8_t* out_buf[2] = {base + al(pre) + 4 * cb, base + al(pre) + 5 * cb};
  cudaStream_t s = cs(stream);
  const size_t pitch = (size_t)seqlen * tok;   // host row pitch: one batch row of the whole sequence
  const std::vector<int> lens = host_chunk_lengths(seqlen, chunk);
  const int n_chunks = (int)lens.size();
  // the copy streams start after the work already queued on `stream`
  JB_CUDA(cudaEventRecord(h->ev_comp[1], s));
  JB_CUDA(cudaStreamWaitEvent(h->io_in, h->ev_comp[1], 0));
  JB_CUDA(cudaStreamWaitEvent(h->io_out, h->ev_comp[1], 0));
  for (int i = 0, t0 = 0; i < n_chunks; t0 += lens[i], ++i) {
    const int k = i & 1, n = lens[i];
    const size_t row = (size_t)n * tok;
    // in: the buffer's previous chunk (i - 2) has been consumed by its prefill
    if (i >= 2) JB_CUDA(cudaStreamWaitEvent(h->io_in, h->ev_comp[k], 0));
    JB_CUDA(copy_rows(in_buf[k], reinterpret_cast<const uint8_t*>(u_host) + (size_t)t0 * tok, row, pitch, row, batch,
                      cudaMemcpyHostToDevice, h->io_in));
    if (residual_host)
      JB_CUDA(copy_rows(res_buf[k], reinterpret_cast<const uint8_t*>(residual_host) + (size_t)t0 * tok, row, pitch,
                        row, batch, cudaMemcpyHostToDevice, h->io_in));
    JB_CUDA(cudaEventRecord(h->ev_in[k], h->io_in));
    // compute: chunk i is in, and the out buffer's previous chunk is back on the host
    JB_CUDA(cudaStreamWaitEvent(s, h->ev_in[k], 0));
    if (i >= 2) JB_CUDA(cudaStreamWaitEvent(s, h->ev_out[k], 0));
    JB_TRY(jamba_mamba_prefill(h, in_buf[k], residual_host ? res_buf[k] : nullptr, out_buf[k], batch, n,
                               i == 0 ? conv_state_in : conv_state_out, i == 0 ? ssm_state_in : ssm_state_out,
                               conv_state_out, ssm_state_out, ws, pre, stream));
    JB_CUDA(cudaEventRecord(h->ev_comp[k], s));
    // out
    JB_CUDA(cudaStreamWaitEvent(h->io_out, h->ev_comp[k], 0));
    JB_CUDA(copy_rows(reinterpret_cast<uint8_t*>(out_host) + (size_t)t0 * tok, out_buf[k], row, row, pitch, batch,
                      cudaMemcpyDeviceToHost, h->io_out));
    JB_CUDA(cudaEventRecord(h->ev_out[k], h->io_out));
  }
  // work queued on `stream` afterwards sees every chunk back on the host
  for (int k = 0; k < 2 && k < n_chunks; ++k) JB_CUDA(cudaStreamWaitEvent(s, h->ev_out[k], 0));
  return JAMBA_OK;
}

// --------------------------------------------------------- selective scan

jamba_status jamba_selective_scan_workspace_size(int batch, int seqlen, int d_inner, int d_state, int chunk,
                                                 size_t* bytes) {
  if (!bytes || batch <= 0 || seqlen <= 0 || d_inner <= 0) return fail(JAMBA_ERR_INVALID_ARG, "scan workspace: bad argument");
  if (d_state != 16) return fail(JAMBA_ERR_UNSUPPORTED, "d_state must be 16");
  if (chunk < 0 || chunk % 16) return fail(JAMBA_ERR_INVALID_ARG, "chunk must be a multiple of 16");
  // the automatic chunk does not depend on the dtypes by more than the
  // resident-CTA count; size for the smallest chunk any dtype would pick
  if (chunk == 0) {
    const int a = scan_auto_chunk(batch, seqlen, d_inner, JAMBA_BF16, JAMBA_BF16);
    const int b = scan_auto_chunk(batch, seqlen, d_inner, JAMBA_BF16, JAMBA_F32);
    const int c = scan_auto_chunk(batch, seqlen, d_inner, JAMBA_F32, JAMBA_F32);
    chunk = a < b ? (a < c ? a : c) : (b < c ? b : c);
  }
  *bytes = scan_workspace_bytes(batch, seqlen, d_inner, chunk);
  return JAMBA_OK;
}

jamba_status jamba_selective_scan(const void* x, int ld_x, const void* z, int ld_z, const float* dt, int ld_dt,
                                  const void* B, int ld_b, const void* C, int ld_c, int bc_dtype, const float* A,
                                  const float* D, const float* h0, void* y, int ld_y, float* h_out, int batch,
                                  int seqlen, int d_inner, int d_state, int dtype, int chunk, void* ws,
                                  size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_selective_scan");
  JB_TRY(check_dtype(dtype));
  JB_TRY(check_dtype(bc_dtype));
  if (d_state != 16) return fail(JAMBA_ERR_UNSUPPORTED, "d_state must be 16");
  if (batch <= 0 || seqlen <= 0 || d_inner <= 0) return fail(JAMBA_ERR_INVALID_ARG, "scan: sizes must be positive");
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(z, "z"));
  JB_TRY(check_ptr(dt, "dt"));
  JB_TRY(check_ptr(B, "B"));
  JB_TRY(check_ptr(C, "C"));
  JB_TRY(check_ptr(A, "A"));
  JB_TRY(check_ptr(D, "D"));
  JB_TRY(check_ptr(h0, "h0", false));
  JB_TRY(check_ptr(y, "y"));
  JB_TRY(check_ptr(h_out, "h_out", false));
  if (chunk == 0) chunk = scan_auto_chunk(batch, seqlen, d_inner, dtype, bc_dtype);
  ScanCall sc = {};
  sc.x = x; sc.ld_x = ld_x; sc.z = z; sc.ld_z = ld_z; sc.dt = dt; sc.ld_dt = ld_dt;
  sc.B = B; sc.ld_b = ld_b; sc.C = C; sc.ld_c = ld_c; sc.bc_dtype = bc_dtype;
  sc.A = A; sc.D = D; sc.h0 = h0; sc.y = y; sc.ld_y = ld_y; sc.h_out = h_out;
  sc.batch = batch; sc.L = seqlen; sc.di = d_inner; sc.dtype = dtype; sc.chunk = chunk;
  sc.ws = ws; sc.ws_bytes = ws_bytes;
  return scan_run(sc, cs(stream));
}

jamba_status jamba_test_scan_plan(int batch, int seqlen, int groups, const float* head, int slots, int* chunks,
                                  int* lens, int* planned) {
  if (!head || !chunks || !lens || !planned || groups <= 0 || groups > SCAN_MAX_GROUPS)
    return fail(JAMBA_ERR_INVALID_ARG, "scan plan: bad argument");
  ScanSchedule sch;
  scan_plan(batch, seqlen, groups, head, slots, &sch);
  *planned = sch.n;
  for (int g = 0; g < sch.n; ++g) {
    chunks[g] = sch.chunks[g];
    lens[g] = sch.len[g];
  }
  return JAMBA_OK;
}

jamba_status jamba_test_gemm_splits(int M, int N, int K, int bn, int min_k_tiles, int num_groups, int* splits,
                                    int* i8w_splits_out) {
  if (!splits || !i8w_splits_out || M <= 0 || N <= 0 || K <= 0 || bn <= 0 || num_groups <= 0)
    return fail(JAMBA_ERR_INVALID_ARG, "gemm splits: bad argument");
  *splits = choose_splits(M, N, K, bn, min_k_tiles);
  *i8w_splits_out = i8w_splits(M, num_groups, N, K);
  return JAMBA_OK;
}

jamba_status jamba_test_scan_missing_predecessor(const void* x, int ld_x, const void* z, int ld_z, const float* dt,
                                                 int ld_dt, const void* B, int ld_b, const void* C, int ld_c,
                                                 int bc_dtype, const float* A, const float* D, void* y, int ld_y,
                                                 float* h_out, int batch, int seqlen, int d_inner, int d_state,
                                                 int dtype, int chunk, unsigned long long wait_ns, void* ws,
                                                 size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_test_scan_missing_predecessor");
  JB_TRY(check_dtype(dtype));
  JB_TRY(check_dtype(bc_dtype));
  if (d_state != 16) return fail(JAMBA_ERR_UNSUPPORTED, "d_state must be 16");
  if (batch <= 0 || seqlen <= 0 || d_inner <= 0 || chunk <= 0 || wait_ns == 0)
    return fail(JAMBA_ERR_INVALID_ARG, "scan test: sizes, chunk and wait must be positive");
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(z, "z"));
  JB_TRY(check_ptr(dt, "dt"));
  JB_TRY(check_ptr(B, "B"));
  JB_TRY(check_ptr(C, "C"));
  JB_TRY(check_ptr(A, "A"));
  JB_TRY(check_ptr(D, "D"));
  JB_TRY(check_ptr(y, "y"));
  JB_TRY(check_ptr(h_out, "h_out", false));
  ScanCall sc = {};
  sc.x = x; sc.ld_x = ld_x; sc.z = z; sc.ld_z = ld_z; sc.dt = dt; sc.ld_dt = ld_dt;
  sc.B = B; sc.ld_b = ld_b; sc.C = C; sc.ld_c = ld_c; sc.bc_dtype = bc_dtype;
  sc.A = A; sc.D = D; sc.h0 = nullptr; sc.y = y; sc.ld_y = ld_y; sc.h_out = h_out;
  sc.batch = batch; sc.L = seqlen; sc.di = d_inner; sc.dtype = dtype; sc.chunk = chunk;
  sc.ws = ws; sc.ws_bytes = ws_bytes;
  sc.wait_ns = wait_ns;
  sc.skip_first_chunk = 1;
  return scan_run(sc, cs(stream));
}

// --------------------------------------------------------- building blocks

jamba_status jamba_rmsnorm(const void* x, const float* w, void* out, int rows, int cols, float eps, int dtype,
                           jamba_stream_t stream) {
  JB_RANGE("jamba_rmsnorm");
  JB_TRY(check_dtype(dtype));
  if (rows <= 0 || cols <= 0) return fail(JAMBA_ERR_INVALID_ARG, "rmsnorm: sizes must be positive");
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(w, "w"));
  JB_TRY(check_ptr(out, "out"));
  return rmsnorm(x, w, out, rows, cols, eps, dtype, cs(stream));
}

jamba_status jamba_causal_conv1d(const void* x, int ld_x, const void* w, const void* b, void* out,
                                 const float* state_in, float* state_out, int batch, int seqlen, int channels,
                                 int dtype, jamba_stream_t stream) {
  JB_RANGE("jamba_causal_conv1d");
  JB_TRY(check_dtype(dtype));
  if (batch <= 0 || seqlen <= 0 || channels <= 0 || ld_x < channels)
    return fail(JAMBA_ERR_INVALID_ARG, "conv: bad sizes");
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(w, "w"));
  JB_TRY(check_ptr(b, "b"));
  JB_TRY(check_ptr(out, "out"));
  if (state_in && state_in == state_out)
    return fail(JAMBA_ERR_INVALID_ARG, "conv: state_in and state_out may not alias here");
  return conv_prefill(x, ld_x, w, b, out, state_in, state_out, batch, seqlen, channels, dtype, nullptr, cs(stream));
}

jamba_status jamba_in_proj_conv1d(const void* u, const void* w_in, const void* conv_w, const void* conv_b, void* xz,
                                  void* xc, const float* state_in, float* state_out, int batch, int seqlen,
                                  int d_model, int d_inner, jamba_stream_t stream) {
  JB_RANGE("jamba_in_proj_conv1d");
  if (batch <= 0 || seqlen <= 0 || d_model <= 0 || d_inner <= 0)
    return fail(JAMBA_ERR_INVALID_ARG, "in_proj conv: sizes must be positive");
  JB_TRY(check_ptr(u, "u"));
  JB_TRY(check_ptr(w_in, "w_in"));
  JB_TRY(check_ptr(conv_w, "conv_w"));
  JB_TRY(check_ptr(conv_b, "conv_b"));
  JB_TRY(check_ptr(xz, "xz"));
  JB_TRY(check_ptr(xc, "xc"));
  JB_TRY(check_ptr(state_in, "state_in", false));
  JB_TRY(check_ptr(state_out, "state_out", false));
  if (state_in && state_in == state_out)
    return fail(JAMBA_ERR_INVALID_ARG, "in_proj conv: state_in and state_out may not alias here");
  if ((long long)batch * seqlen > (1LL << 31) / 2) return fail(JAMBA_ERR_UNSUPPORTED, "in_proj conv: too many tokens");
  if (seqlen < 3 || d_inner % 32 || d_inner < 128 || !aligned16(conv_w) || !aligned16(conv_b))
    return fail(JAMBA_ERR_UNSUPPORTED, "in_proj conv: needs seqlen >= 3, d_inner a multiple of 32 (>= 128) and "
                                       "16-byte aligned conv weights");
  return in_proj_conv(u, w_in, conv_w, conv_b, xz, xc, state_in, state_out, nullptr, batch * seqlen, seqlen, d_model,
                      d_inner, cs(stream));
}

jamba_status jamba_gemm(const void* a, const void* b, void* out, int ld_out, const void* residual, int m, int n,
                        int k, int dtype, int out_dtype, jamba_stream_t stream) {
  JB_RANGE("jamba_gemm");
  JB_TRY(check_dtype(dtype));
  JB_TRY(check_dtype(out_dtype));
  if (m <= 0 || n <= 0 || k <= 0 || ld_out < n) return fail(JAMBA_ERR_INVALID_ARG, "gemm: bad sizes");
  if (dtype == JAMBA_F32 && out_dtype != JAMBA_F32) return fail(JAMBA_ERR_UNSUPPORTED, "gemm: fp32 inputs give fp32 output");
  if (residual && out_dtype != dtype) return fail(JAMBA_ERR_UNSUPPORTED, "gemm: residual needs out_dtype == dtype");
  GemmDesc g = gdesc(a, k, b, k, m, n, k, out_dtype == JAMBA_BF16 ? EPI_BF16 : EPI_F32, out, ld_out);
  g.residual = residual;
  g.ldr = ld_out;
  return gemm_any(dtype, g, cs(stream));
}

// -------------------------------------------------------------------- MoE

namespace {
struct MoeWs {
  int* counts; int* inv; void* xperm; void* act; float* Y;
  int y_splits;   // k-split partial outputs of the down GEMM held in Y
  size_t total;
};
MoeWs carve_moe(const jamba_moe_config& c, int T, void* ws) {
  MoeWs m;
  const size_t rows = (size_t)T * c.top_k;
  m.y_splits = c.expert_dtype == JAMBA_INT8 ? i8w_splits((int)rows, c.n_experts, c.d_model, c.d_ff) : 1;
  Carver cv(ws);
  m.counts = cv.take<int>(sizeof(int) * 64);
  m.inv = cv.take<int>(sizeof(int) * rows);
  m.xperm = cv.take(rows * c.d_model * 2);
  m.act = cv.take(rows * c.d_ff * 2);
  m.Y = cv.take<float>(rows * c.d_model * 4 * m.y_splits);
  m.total = cv.off;
  return m;
}
jamba_status check_moe_cfg(const jamba_moe_config* c) {
  if (!c) return fail(JAMBA_ERR_INVALID_ARG, "moe: null config");
  if (c->dtype != JAMBA_BF16) return fail(JAMBA_ERR_UNSUPPORTED, "moe: bf16 only");
  if (c->n_experts < 1 || c->n_experts > 64) return fail(JAMBA_ERR_UNSUPPORTED, "moe: 1..64 experts");
  if (c->top_k < 1 || c->top_k > 2 || c->top_k > c->n_experts) return fail(JAMBA_ERR_UNSUPPORTED, "moe: top_k must be 1 or 2");
  if (c->d_model <= 0 || c->d_model % 256) return fail(JAMBA_ERR_UNSUPPORTED, "moe: d_model must be a multiple of 256");
  if (c->d_ff <= 0 || c->d_ff % 128) return fail(JAMBA_ERR_UNSUPPORTED, "moe: d_ff must be a multiple of 128");
  if (c->expert_dtype != JAMBA_BF16 && c->expert_dtype != JAMBA_INT8)
    return fail(JAMBA_ERR_UNSUPPORTED, "moe: expert_dtype must be JAMBA_BF16 or JAMBA_INT8");
  return JAMBA_OK;
}
}  // namespace

jamba_status jamba_quantize_int8_rows(const void* w, int dtype, long long rows, int cols, int8_t* q, float* scale,
                                      jamba_stream_t stream) {
  JB_RANGE("jamba_quantize_int8_rows");
  JB_TRY(check_dtype(dtype));
  if (rows <= 0 || cols <= 0 || cols % 8) return fail(JAMBA_ERR_INVALID_ARG, "quantize: rows > 0, cols a positive multiple of 8");
  JB_TRY(check_ptr(w, "w"));
  JB_TRY(check_ptr(q, "q"));
  JB_TRY(check_ptr(scale, "scale"));
  return quantize_int8_rows(w, dtype, rows, cols, q, scale, cs(stream));
}

jamba_status jamba_moe_workspace_size(const jamba_moe_config* cfg, int tokens, size_t* bytes) {
  JB_TRY(check_moe_cfg(cfg));
  if (!bytes || tokens <= 0) return fail(JAMBA_ERR_INVALID_ARG, "moe workspace: bad argument");
  *bytes = carve_moe(*cfg, tokens, nullptr).total;
  return JAMBA_OK;
}

jamba_status jamba_moe_forward(const jamba_moe_config* cfg, const jamba_moe_weights* w, const void* x,
                               const void* residual, void* y, int tokens, int32_t* topk_idx, float* topk_w,
                               int32_t* expert_offsets, int32_t* perm, void* ws, size_t ws_bytes,
                               jamba_stream_t stream) {
  JB_RANGE("jamba_moe_forward");
  JB_TRY(check_moe_cfg(cfg));
  if (!w || tokens <= 0) return fail(JAMBA_ERR_INVALID_ARG, "moe: bad argument");
  JB_TRY(check_ptr(w->router, "router"));
  JB_TRY(check_ptr(w->w_gate, "w_gate"));
  JB_TRY(check_ptr(w->w_up, "w_up"));
  JB_TRY(check_ptr(w->w_down, "w_down"));
  const bool q8 = cfg->expert_dtype == JAMBA_INT8;
  JB_TRY(check_ptr(w->s_gate, "s_gate", q8));
  JB_TRY(check_ptr(w->s_up, "s_up", q8));
  JB_TRY(check_ptr(w->s_down, "s_down", q8));
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(y, "y"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(topk_idx, "topk_idx"));
  JB_TRY(check_ptr(topk_w, "topk_w"));
  JB_TRY(check_ptr(expert_offsets, "expert_offsets"));
  JB_TRY(check_ptr(perm, "perm"));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_moe_config& c = *cfg;
  MoeWs m = carve_moe(c, tokens, ws);
  if (ws_bytes < m.total) return fail(JAMBA_ERR_WORKSPACE, "moe: workspace too small");
  cudaStream_t s = cs(stream);
  const int E = c.n_experts, K = c.top_k, dm = c.d_model, dff = c.d_ff;
  const int rows = tokens * K;
  NvtxSteps nv;
  nv.next("router_top_k");
  JB_TRY(moe_route(x, w->router, tokens, dm, E, K, topk_idx, topk_w, m.counts, expert_offsets, perm, m.inv, s));
  nv.next("gather");
  JB_TRY(moe_gather(x, perm, rows, K, dm, m.xperm, s));
  nv.next("experts_gate_up_swiglu");
  // gate | up with SwiGLU: act = SiLU(x W_g^T) * (x W_u^T), per expert
  GemmDesc g1 = gdesc(m.xperm, dm, w->w_gate, dm, rows, dff, dm, EPI_SWIGLU, m.act, dff);
  g1.b2 = w->w_up;
  g1.grouped = 1;
  g1.offsets = expert_offsets;
  g1.num_groups = E;
  g1.b_rows = dff;
  if (q8) {
    g1.b_int8 = 1;
    g1.scale_b = w->s_gate;
    g1.scale_b2 = w->s_up;
  }
  JB_TRY(gemm_bf16(g1, s));
  // down: Y = act W_d^T, fp32 rows in routed order
  nv.next("experts_down");
  GemmDesc g2 = gdesc(m.act, dff, w->w_down, dff, rows, dm, dff, EPI_F32, m.Y, dm);
  g2.grouped = 1;
  g2.offsets = expert_offsets;
  g2.num_groups = E;
  g2.b_rows = dm;
  if (q8) {
    g2.b_int8 = 1;
    g2.scale_b = w->s_down;
    g2.splits = m.y_splits;   // decode batches: k-split partials, summed by the combine
    g2.split_stride = (long long)rows * dm;
  }
  JB_TRY(gemm_bf16(g2, s));
  nv.next("combine");
  JB_TRY(moe_combine(m.Y, m.y_splits, (long long)rows * dm, m.inv, topk_w, tokens, K, dm, residual, y, s));
  return JAMBA_OK;
}

// ------------------------------------------------------ expert-parallel MoE

jamba_status jamba_moe_ep_dispatch(const jamba_moe_config* cfg, const void* router, const void* x, int tokens,
                                   int32_t* topk_idx, float* topk_w, int32_t* expert_offsets, int32_t* perm,
                                   void* send_rows, void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_moe_ep_dispatch");
  JB_TRY(check_moe_cfg(cfg));
  if (tokens <= 0) return fail(JAMBA_ERR_INVALID_ARG, "moe ep dispatch: tokens must be positive");
  JB_TRY(check_ptr(router, "router"));
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(topk_idx, "topk_idx"));
  JB_TRY(check_ptr(topk_w, "topk_w"));
  JB_TRY(check_ptr(expert_offsets, "expert_offsets"));
  JB_TRY(check_ptr(perm, "perm"));
  JB_TRY(check_ptr(send_rows, "send_rows"));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_moe_config& c = *cfg;
  MoeWs m = carve_moe(c, tokens, ws);
  if (ws_bytes < m.total) return fail(JAMBA_ERR_WORKSPACE, "moe ep dispatch: workspace too small");
  cudaStream_t s = cs(stream);
  JB_TRY(moe_route(x, router, tokens, c.d_model, c.n_experts, c.top_k, topk_idx, topk_w, m.counts, expert_offsets,
                   perm, m.inv, s));
  return moe_gather(x, perm, tokens * c.top_k, c.top_k, c.d_model, send_rows, s);
}

jamba_status jamba_moe_ep_experts_workspace_size(const jamba_moe_config* cfg, int rows, int world, size_t* bytes) {
  JB_TRY(check_moe_cfg(cfg));
  if (!bytes || rows < 0 || world <= 0) return fail(JAMBA_ERR_INVALID_ARG, "moe ep workspace: bad argument");
  *bytes = al(sizeof(int) * ((size_t)world * cfg->n_experts + 1)) + al((size_t)(rows > 0 ? rows : 1) * cfg->d_ff * 2);
  return JAMBA_OK;
}

jamba_status jamba_moe_ep_experts(const jamba_moe_config* cfg, const jamba_moe_weights* w, const void* rows_in,
                                  int rows, const int32_t* group_counts, int world, float* rows_out, void* ws,
                                  size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_moe_ep_experts");
  JB_TRY(check_moe_cfg(cfg));
  if (!w || rows < 0 || world <= 0 || world * cfg->n_experts > 4096)
    return fail(JAMBA_ERR_INVALID_ARG, "moe ep experts: bad argument");
  if (rows == 0) return JAMBA_OK;
  JB_TRY(check_ptr(w->w_gate, "w_gate"));
  JB_TRY(check_ptr(w->w_up, "w_up"));
  JB_TRY(check_ptr(w->w_down, "w_down"));
  const bool q8 = cfg->expert_dtype == JAMBA_INT8;
  JB_TRY(check_ptr(w->s_gate, "s_gate", q8));
  JB_TRY(check_ptr(w->s_up, "s_up", q8));
  JB_TRY(check_ptr(w->s_down, "s_down", q8));
  JB_TRY(check_ptr(rows_in, "rows_in"));
  JB_TRY(check_ptr(group_counts, "group_counts"));
  JB_TRY(check_ptr(rows_out, "rows_out"));
  JB_TRY(check_ptr(ws, "workspace"));
  size_t need = 0;
  JB_TRY(jamba_moe_ep_experts_workspace_size(cfg, rows, world, &need));
  if (ws_bytes < need) return fail(JAMBA_ERR_WORKSPACE, "moe ep experts: workspace too small");
  const jamba_moe_config& c = *cfg;
  const int E = c.n_experts, G = world * E, dm = c.d_model, dff = c.d_ff;
  Carver cv(ws);
  int* offsets = cv.take<int>(sizeof(int) * ((size_t)G + 1));
  void* act = cv.take((size_t)rows * dff * 2);
  cudaStream_t s = cs(stream);
  // groups in received order: (source rank, local expert); group g uses local expert g % E
  JB_TRY(group_offsets(group_counts, G, offsets, s));
  GemmDesc g1 = gdesc(rows_in, dm, w->w_gate, dm, rows, dff, dm, EPI_SWIGLU, act, dff);
  g1.b2 = w->w_up;
  g1.grouped = 1;
  g1.offsets = offsets;
  g1.num_groups = G;
  g1.group_mod = E;
  g1.b_rows = dff;
  if (q8) {
    g1.b_int8 = 1;
    g1.scale_b = w->s_gate;
    g1.scale_b2 = w->s_up;
  }
  JB_TRY(gemm_bf16(g1, s));
  GemmDesc g2 = gdesc(act, dff, w->w_down, dff, rows, dm, dff, EPI_F32, rows_out, dm);
  g2.grouped = 1;
  g2.offsets = offsets;
  g2.num_groups = G;
  g2.group_mod = E;
  g2.b_rows = dm;
  if (q8) {
    g2.b_int8 = 1;
    g2.scale_b = w->s_down;
  }
  return gemm_bf16(g2, s);
}

jamba_status jamba_moe_ep_combine(const jamba_moe_config* cfg, const float* rows_back, const float* topk_w,
                                  int tokens, const void* residual, void* y, void* ws, size_t ws_bytes,
                                  jamba_stream_t stream) {
  JB_RANGE("jamba_moe_ep_combine");
  JB_TRY(check_moe_cfg(cfg));
  if (tokens <= 0) return fail(JAMBA_ERR_INVALID_ARG, "moe ep combine: tokens must be positive");
  JB_TRY(check_ptr(rows_back, "rows_back"));
  JB_TRY(check_ptr(topk_w, "topk_w"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(y, "y"));
  JB_TRY(check_ptr(ws, "workspace"));
  const jamba_moe_config& c = *cfg;
  MoeWs m = carve_moe(c, tokens, ws);
  if (ws_bytes < m.total) return fail(JAMBA_ERR_WORKSPACE, "moe ep combine: workspace too small");
  return moe_combine(rows_back, 1, 0, m.inv, topk_w, tokens, c.top_k, c.d_model, residual, y, cs(stream));
}

}  // extern "C"

// -------------------------------------------------------------- attention

namespace {
struct AttnPrefillWs {
  void* qkv; void* vt; void* o;
  long long ldv;
  size_t total;
};
AttnPrefillWs carve_attn_prefill(const jamba_attn_config& c, int B, int L, void* ws) {
  AttnPrefillWs a;
  const long long T = (long long)B * L;
  const int W = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  a.ldv = (L + 7) / 8 * 8;
  Carver cv(ws);
  a.qkv = cv.take((size_t)T * W * 2);
  a.vt = cv.take((size_t)B * c.n_kv_heads * c.head_dim * a.ldv * 2);
  a.o = cv.take((size_t)T * c.n_heads * c.head_dim * 2);
  a.total = cv.off;
  return a;
}
struct AttnStepWs {
  void* qkv; float* part; void* o; float* opart;
  int splits, o_splits;
  size_t total;
};
AttnStepWs carve_attn_step(const jamba_attn_config& c, int B, int max_len, void* ws) {
  AttnStepWs a;
  const int W = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim, HD = c.n_heads * c.head_dim;
  a.splits = attn_decode_splits(B, c.n_kv_heads, max_len);
  a.o_splits = choose_splits(c.d_model, B, HD, 64, 8);
  Carver cv(ws);
  a.qkv = cv.take((size_t)B * W * 2);
  a.part = cv.take<float>((size_t)B * c.n_heads * a.splits * (c.head_dim + 2) * 4);
  a.o = cv.take((size_t)B * HD * 2);
  a.opart = cv.take<float>((size_t)a.o_splits * B * c.d_model * 4);
  a.total = cv.off;
  return a;
}
jamba_status check_attn_cfg(const jamba_attn_config* c) {
  if (!c) return fail(JAMBA_ERR_INVALID_ARG, "attention: null config");
  if (c->dtype != JAMBA_BF16) return fail(JAMBA_ERR_UNSUPPORTED, "attention: bf16 only");
  if (c->head_dim != 128) return fail(JAMBA_ERR_UNSUPPORTED, "attention: head_dim must be 128");
  if (c->n_heads <= 0 || c->n_kv_heads <= 0 || c->n_heads % c->n_kv_heads)
    return fail(JAMBA_ERR_INVALID_ARG, "attention: n_kv_heads must divide n_heads");
  if (c->d_model <= 0 || c->d_model % 64) return fail(JAMBA_ERR_UNSUPPORTED, "attention: d_model must be a multiple of 64");
  return JAMBA_OK;
}
}  // namespace

extern "C" {

jamba_status jamba_attn_prefill_workspace_size(const jamba_attn_config* cfg, int batch, int seqlen, size_t* bytes) {
  JB_TRY(check_attn_cfg(cfg));
  if (!bytes || batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "attention workspace: bad argument");
  *bytes = carve_attn_prefill(*cfg, batch, seqlen, nullptr).total;
  return JAMBA_OK;
}

jamba_status jamba_attn_prefill(const jamba_attn_config* cfg, const jamba_attn_weights* w, const void* x,
                                const void* residual, void* out, int batch, int seqlen, void* k_cache,
                                void* v_cache, int max_len, void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_attn_prefill");
  JB_TRY(check_attn_cfg(cfg));
  if (!w || batch <= 0 || seqlen <= 0) return fail(JAMBA_ERR_INVALID_ARG, "attention prefill: bad argument");
  JB_TRY(check_ptr(w->w_qkv, "w_qkv"));
  JB_TRY(check_ptr(w->w_o, "w_o"));
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(out, "out"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(k_cache, "k_cache", false));
  JB_TRY(check_ptr(v_cache, "v_cache", false));
  JB_TRY(check_ptr(ws, "workspace"));
  if (x == out) return fail(JAMBA_ERR_INVALID_ARG, "attention prefill: out may not alias x");
  if ((k_cache == nullptr) != (v_cache == nullptr))
    return fail(JAMBA_ERR_INVALID_ARG, "attention prefill: give both caches or neither");
  if (k_cache && max_len < seqlen) return fail(JAMBA_ERR_INVALID_ARG, "attention prefill: max_len < seqlen");
  const jamba_attn_config& c = *cfg;
  AttnPrefillWs a = carve_attn_prefill(c, batch, seqlen, ws);
  if (ws_bytes < a.total) return fail(JAMBA_ERR_WORKSPACE, "attention prefill: workspace too small");
  cudaStream_t s = cs(stream);
  const int T = batch * seqlen, dm = c.d_model, HD = c.n_heads * c.head_dim;
  const int W = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  JB_TRY(gemm_bf16(gdesc(x, dm, w->w_qkv, dm, T, W, dm, EPI_BF16, a.qkv, W), s));
  JB_TRY(attn_prefill_core(a.qkv, a.vt, a.ldv, a.o, k_cache, v_cache, max_len, batch, seqlen, c.n_heads,
                           c.n_kv_heads, s));
  GemmDesc go = gdesc(a.o, HD, w->w_o, HD, T, dm, HD, EPI_BF16, out, dm);
  go.residual = residual;
  go.ldr = dm;
  JB_TRY(gemm_bf16(go, s));
  return JAMBA_OK;
}

jamba_status jamba_attn_step_workspace_size(const jamba_attn_config* cfg, int batch, int max_len, size_t* bytes) {
  JB_TRY(check_attn_cfg(cfg));
  if (!bytes || batch <= 0 || max_len <= 0) return fail(JAMBA_ERR_INVALID_ARG, "attention workspace: bad argument");
  *bytes = carve_attn_step(*cfg, batch, max_len, nullptr).total;
  return JAMBA_OK;
}

jamba_status jamba_attn_step(const jamba_attn_config* cfg, const jamba_attn_weights* w, const void* x,
                             const void* residual, void* out, int batch, void* k_cache, void* v_cache,
                             int max_len, int32_t* lengths, void* ws, size_t ws_bytes, jamba_stream_t stream) {
  JB_RANGE("jamba_attn_step");
  JB_TRY(check_attn_cfg(cfg));
  if (!w || batch <= 0 || max_len <= 0) return fail(JAMBA_ERR_INVALID_ARG, "attention step: bad argument");
  JB_TRY(check_ptr(w->w_qkv, "w_qkv"));
  JB_TRY(check_ptr(w->w_o, "w_o"));
  JB_TRY(check_ptr(x, "x"));
  JB_TRY(check_ptr(out, "out"));
  JB_TRY(check_ptr(residual, "residual", false));
  JB_TRY(check_ptr(k_cache, "k_cache"));
  JB_TRY(check_ptr(v_cache, "v_cache"));
  JB_TRY(check_ptr(ws, "workspace"));
  if (!lengths) return fail(JAMBA_ERR_INVALID_ARG, "attention step: lengths is null");
  if (x == out) return fail(JAMBA_ERR_INVALID_ARG, "attention step: out may not alias x");
  const jamba_attn_config& c = *cfg;
  AttnStepWs a = carve_attn_step(c, batch, max_len, ws);
  if (ws_bytes < a.total) return fail(JAMBA_ERR_WORKSPACE, "attention step: workspace too small");
  cudaStream_t s = cs(stream);
  const int dm = c.d_model, HD = c.n_heads * c.head_dim;
  const int W = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  // weights stream through the tensor cores as the 128-row side; the token batch is the N side
  GemmDesc g1 = gdesc(w->w_qkv, dm, x, dm, W, batch, dm, EPI_BF16, a.qkv, W);
  g1.transpose_out = 1;
  g1.bn = 64;
  JB_TRY(gemm_bf16(g1, s));
  JB_TRY(attn_decode_core(a.qkv, k_cache, v_cache, max_len, lengths, a.part, a.splits, a.o, batch, c.n_heads,
                          c.n_kv_heads, s));
  GemmDesc g2 = gdesc(w->w_o, HD, a.o, HD, dm, batch, HD, EPI_F32, a.opart, dm);
  g2.transpose_out = 1;
  g2.bn = 64;
  g2.splits = a.o_splits;
  g2.split_stride = (long long)batch * dm;
  JB_TRY(gemm_bf16(g2, s));
  JB_TRY(splitk_reduce(a.opart, a.o_splits, (long long)batch * dm, (long long)batch * dm, residual, out, JAMBA_BF16, s));
  return JAMBA_OK;
}

}  // extern "C"
