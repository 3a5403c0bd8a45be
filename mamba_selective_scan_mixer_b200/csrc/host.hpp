// Host-side internals shared by the launchers: error reporting, device
// properties, TMA tensor-map encoding, per-device error word.
#pragma once
#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <string>

#include "../../include/jamba.h"

namespace jb {

// NVTX ranges on the host timeline: one around every library call that
// launches work (JB_RANGE, named after the entry point) and one per step of
// the path inside it (NvtxSteps::next, named after the step).  They cost a
// no-op call unless a profiler that collects NVTX is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define JB_RANGE_CAT2(a, b) a##b
#define JB_RANGE_CAT(a, b) JB_RANGE_CAT2(a, b)
#define JB_RANGE(name) ::jb::NvtxRange JB_RANGE_CAT(jb_range_, __LINE__)(name)
struct NvtxSteps {
  bool open = false;
  void next(const char* name) {
    if (open) nvtxRangePop();
    nvtxRangePushA(name);
    open = true;
  }
  ~NvtxSteps() {
    if (open) nvtxRangePop();
  }
};

jamba_status fail(jamba_status st, const std::string& msg);
const char* last_error();
jamba_status cuda_fail(cudaError_t e, const char* what);
#define JB_CUDA(call)                                       \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return ::jb::cuda_fail(e_, #call); \
  } while (0)
#define JB_TRY(expr)                         \
  do {                                       \
    jamba_status s_ = (expr);                \
    if (s_ != JAMBA_OK) return s_;           \
  } while (0)

int num_sms();                 // of the current device

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel of the stream finishes and must call griddep_wait() before it
// touches memory that kernel produces or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
int* device_error_word();      // per-device status word (allocated on first use)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D tensor map over a row-major matrix: `inner` elements per row (the
// extent TMA treats as valid), `rows` rows, `row_stride` bytes between rows.
jamba_status make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t inner, uint64_t rows, uint64_t row_stride, uint32_t box_inner,
                         uint32_t box_rows, CUtensorMapSwizzle sw);
// 3-D tensor map over [outer][rows][inner].
jamba_status make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t inner, uint64_t rows, uint64_t outer, uint64_t row_stride,
                         uint64_t outer_stride, uint32_t box_inner, uint32_t box_rows,
                         CUtensorMapSwizzle sw, uint32_t box_outer = 1);

// ---------------------------------------------------------------- GEMM
struct GemmDesc {
  const void* a;   // [M, K] bf16, row stride lda elements
  long long lda;
  const void* b;   // dense: [N, K] row stride ldb; grouped: [groups, b_rows, K] contiguous
  long long ldb;
  const void* b2;  // SwiGLU "up" weights, same shape as b
  int M, N, K;
  int b_rows;      // grouped: rows of each group's B matrix
  int grouped;
  const int* offsets;
  int num_groups;
  int group_mod;   // grouped: > 0 maps group g to weight set g % group_mod
  int epi;         // EpiKind
  int transpose_out;
  void* out;
  long long ldo, split_stride;
  const void* residual;
  long long ldr;
  const float* bias;
  int splits;      // >= 1; more than one only with fp32 partial outputs
  int bn;          // 0 = automatic
  int b_int8;      // grouped expert GEMMs: b / b2 hold INT8 codes (row stride ldb bytes)
  const float* scale_b;   // with b_int8: per-row scales [groups, b_rows] of b
  const float* scale_b2;  // ... and of b2
  // EPI_CONV (swap-AB only): decode conv fused into in_proj's epilogue
  const void* conv_w; const void* conv_b; float* conv_state; void* xc_out; int conv_c;
  // EPI_CONVP (prefill in_proj, bf16): the conv + SiLU of the x columns in the
  // epilogue (conv_w, conv_b, xc_out, conv_c as above); caches in / out per
  // sequence of conv_L rows, cache row of channel c = conv_perm[c]; rows 0-2
  // of 32-row slabs are completed by conv_fixup
  const float* conv_in; float* conv_out; const int* conv_perm; int conv_L;
};
jamba_status gemm_bf16(const GemmDesc& g, cudaStream_t s);
// k-splits that balance the fp32 expert GEMM with INT8 weights over the SMs
// when every expert holds few rows (1 otherwise); the caller gives the GEMM
// that many fp32 partial outputs, split_stride elements apart.
int i8w_splits(int M, int num_groups, int N, int K);
jamba_status gemm_f32(const GemmDesc& g, cudaStream_t s);

// Splits so that m_tiles * n_tiles * splits fills the SMs, each split keeping
// at least `min_k_tiles` 64-wide k-steps.
int choose_splits(int M, int N, int K, int bn, int min_k_tiles);

// ---------------------------------------------------------------- scan
// Time chunks per channel group of 256 (groups = d_inner / 256 rounded up).
// n == 0: every group takes the uniform chunk length of the call.
constexpr int SCAN_MAX_GROUPS = 64;
constexpr int SCAN_GROUP_CHANNELS = 256;   // channels of one scan CTA
struct ScanSchedule {
  int n;                           // channel groups covered (0 = uniform)
  int chunks[SCAN_MAX_GROUPS];     // time chunks of each group
  int len[SCAN_MAX_GROUPS];        // their length in steps (a multiple of 16)
};
// Per-group chunks for `batch` rows of L steps when the channels of group g
// lose the carried state after about head[g] steps (groups sorted so that
// later ones are no slower): the largest CTA cost (chunk + replayed head) is
// minimised with at most `slots` CTAs in the launch.  Returns n = 0 when
// batch rows alone fill the slots.
void scan_plan(int batch, int L, int groups, const float* head, int slots, ScanSchedule* out);
int scan_slots(int dtype, int bc_dtype);   // CTAs of the scan resident at once on this device

struct ScanCall {
  const void* x; long long ld_x;
  const void* z; long long ld_z;
  const float* dt; long long ld_dt;
  const void* B; long long ld_b;
  const void* C; long long ld_c;
  int bc_dtype;
  const float* A; const float* D; const float* h0;
  void* y; long long ld_y;
  float* h_out;
  int batch, L, di, dtype, chunk;
  const ScanSchedule* sched;   // null or n == 0: uniform chunks of `chunk` steps
  const int* perm;             // null, or [di]: the cache row of internal channel c is perm[c]
  void* ws; size_t ws_bytes;
  int* err;   // device status word; null = the library's per-device word
  int a_form;                    // SCAN_A_*: which kernel owns the channels, when the caller knows
  unsigned long long wait_ns;    // look-back wait limit; 0 = the library default
  int skip_first_chunk;          // test only: launch no CTA for chunk 0 (its flags stay unset)
  int summary;                   // state-only: no y / z; h_out (required) and p_out (decay product) out
  float* p_out;
};
enum ScanAForm { SCAN_A_UNKNOWN = 0, SCAN_A_POWER = 1, SCAN_A_GENERAL = 2 };
jamba_status scan_run(const ScanCall& s, cudaStream_t st);
size_t scan_workspace_bytes(int batch, int L, int di, int chunk_len, const ScanSchedule* sched = nullptr);
size_t scan_records(int batch, int L, int di, int chunk_len, const ScanSchedule* sched);   // CTAs of a launch
size_t scan_records_bytes(size_t recs);                                                   // workspace they use
int scan_auto_chunk(int batch, int L, int di, int dtype, int bc_dtype);
jamba_status static_scan_status_take(int* value);   // static scan's own status word (read and cleared)
// context-parallel prefill: the state entering slice `rank` from the slices' carries
jamba_status carry_combine(const float* P, const float* H, int rank, const float* h_init, float* h_in, long long n,
                           cudaStream_t st);
jamba_status ssm_step(const void* xc, const void* z, long long ld_z, const float* dt, const float* bc,
                      long long ld_bc, const float* A, const float* D, float* state, void* y, int batch, int di,
                      int dtype, cudaStream_t st);

// ---------------------------------------------------------------- conv / norms
// perm (prefill): null, or [C]: the cache row of internal channel c is perm[c]
jamba_status conv_prefill(const void* x, long long ld_x, const void* w, const void* b, void* out,
                          const float* st_in, float* st_out, int batch, int L, int C, int dtype, const int* perm,
                          cudaStream_t s);
jamba_status conv_step(const void* x, long long ld_x, const void* w, const void* b, void* out, float* state,
                       int batch, int C, int dtype, cudaStream_t s);
// After an EPI_CONVP in_proj: rows 0-2 of each 32-row slab whose conv window
// reaches the slab above within their sequence, from the raw x the epilogue
// left in the x columns of xz (row stride ld).
jamba_status conv_fixup(const void* xz, long long ld, const void* w, const void* b, void* xc, const float* st_in,
                        int T, int L, int C, const int* perm, cudaStream_t s);
jamba_status conv_halo_state(const void* xz, long long ld, float* state, int batch, int C, int dtype,
                             cudaStream_t s);
// Row and column gathers for reordering channel-indexed weights:
// dst[r, :] = src[perm[r], :] over rows of row_bytes bytes, and, for a
// [rows, cols] matrix of `esize`-byte elements, dst[:, j] = src[:, perm[j]].
jamba_status gather_rows(const void* src, void* dst, const int* perm, int rows, int row_bytes, cudaStream_t s);
jamba_status gather_cols(const void* src, void* dst, const int* perm, int rows, int cols, int esize,
                         cudaStream_t s);
jamba_status rmsnorm(const void* x, const float* w, void* out, int rows, int cols, float eps, int dtype,
                     cudaStream_t s);
jamba_status xproj_norm(const float* part, int splits, long long split_stride, int T, int R, int N,
                        const float* w_dt, const float* w_B, const float* w_C, int inner_norm, float eps,
                        void* dtlow, float* bc, int dtype, cudaStream_t s);
jamba_status splitk_reduce(const float* part, int splits, long long split_stride, long long n,
                           const void* residual, void* out, int dtype, cudaStream_t s);

// ---------------------------------------------------------------- MoE
jamba_status moe_route(const void* x, const void* W, int T, int dm, int E, int K, int* idx, float* w, int* counts,
                       int* offsets, int* perm, int* inv, cudaStream_t s);
jamba_status moe_gather(const void* x, const int* perm, int rows, int K, int dm, void* out, cudaStream_t s);
jamba_status group_offsets(const int* counts, int n, int* offsets, cudaStream_t s);   // exclusive prefix sum
jamba_status quantize_int8_rows(const void* w, int dtype, long long rows, int cols, int8_t* q, float* scale,
                                cudaStream_t s);
// out[t] = sum over slots k of w[t, k] * (sum over splits of Y[split][inv[t, k]]) (+ residual[t])
jamba_status moe_combine(const float* Y, int splits, long long split_stride, const int* inv, const float* w, int T,
                         int K, int dm, const void* residual, void* out, cudaStream_t s);

// ---------------------------------------------------------------- attention
jamba_status attn_prefill_core(const void* qkv, void* vt, long long ldv, void* o, void* k_cache, void* v_cache,
                               int max_len, int B, int L, int H, int G, cudaStream_t s);
int attn_decode_splits(int B, int G, int max_len);
jamba_status attn_decode_core(const void* qkv, void* k_cache, void* v_cache, int max_len, int* lengths, float* part,
                              int splits, void* o, int B, int H, int G, cudaStream_t s);

}  // namespace jb
