// Selective scan whose scratch lives in a static device array, for callers
// that may not allocate device memory (see jamba_selective_scan_static in
// include/jamba.h).
//
// The scan kernel needs scratch beyond its inputs and outputs: two ticket
// counters, one flag per (batch row, channel group, time chunk) and one
// 48 KiB record per such chunk.  Here that scratch is a file-scope array of
// kStaticScratchBytes that every GPU loading the library holds until the
// process exits.  Host code cannot use the array's name as a device address:
// the first call on each device, with that device current, asks the runtime
// for the address with cudaGetSymbolAddress and caches it.
#include <mutex>
#include <string>

#include "host.hpp"

namespace jb {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 32 MiB per device

static __device__ __align__(256) uint8_t g_scan_scratch[kStaticScratchBytes];
static __device__ int g_scan_status;   // status word used when the caller passes none

namespace {

struct StaticAddrs {
  void* scratch = nullptr;
  int* status = nullptr;
};

constexpr int kMaxDev = 64;

StaticAddrs g_cache[kMaxDev];
std::mutex g_mu;

jamba_status static_addrs(StaticAddrs* out) {
  int dev = -1;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev) return fail(JAMBA_ERR_UNSUPPORTED, "static scan: device index out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  StaticAddrs* cache = g_cache;
  if (!cache[dev].scratch) {
    void* p = nullptr;
    void* q = nullptr;
    JB_CUDA(cudaGetSymbolAddress(&p, g_scan_scratch));
    JB_CUDA(cudaGetSymbolAddress(&q, g_scan_status));
    cache[dev].scratch = p;
    cache[dev].status = reinterpret_cast<int*>(q);
  }
  *out = cache[dev];
  return JAMBA_OK;
}

}  // namespace

// Reads and clears the static status word of the current device: the word
// the static scan latches a timeout in when its caller passes no status.
// Nothing to read (JAMBA_OK) until a static call has run on this device.
jamba_status static_scan_status_take(int* value) {
  *value = 0;
  int dev = -1;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDev) return JAMBA_OK;
  int* w = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    w = g_cache[dev].status;
  }
  if (!w) return JAMBA_OK;
  JB_CUDA(cudaMemcpy(value, w, sizeof(int), cudaMemcpyDeviceToHost));
  if (*value != 0) JB_CUDA(cudaMemset(w, 0, sizeof(int)));
  return JAMBA_OK;
}

}  // namespace jb

using namespace jb;

extern "C" jamba_status jamba_selective_scan_static(const void* x, int ld_x, const void* z, int ld_z,
                                                    const float* dt, int ld_dt, const void* B, int ld_b,
                                                    const void* C, int ld_c, int bc_dtype, const float* A,
                                                    const float* D, const float* h0, void* y, int ld_y,
                                                    float* h_out, int batch, int seqlen, int d_inner,
                                                    int d_state, int dtype, int* status, jamba_stream_t stream) {
  JB_RANGE("jamba_selective_scan_static");
  if ((dtype != JAMBA_BF16 && dtype != JAMBA_F32) || (bc_dtype != JAMBA_BF16 && bc_dtype != JAMBA_F32))
    return fail(JAMBA_ERR_UNSUPPORTED, "static scan: dtype must be JAMBA_F32 or JAMBA_BF16");
  if (d_state != 16) return fail(JAMBA_ERR_UNSUPPORTED, "static scan: d_state must be 16");
  if (batch <= 0 || seqlen <= 0 || d_inner <= 0) return fail(JAMBA_ERR_INVALID_ARG, "static scan: sizes must be positive");
  const void* ptrs[] = {x, z, dt, B, C, A, D, y};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return fail(JAMBA_ERR_INVALID_ARG, "static scan: null or misaligned tensor");
  if ((h0 && !aligned16(h0)) || (h_out && !aligned16(h_out)))
    return fail(JAMBA_ERR_INVALID_ARG, "static scan: misaligned state");

  // The automatic chunk gives at most one record per resident CTA (a few
  // hundred records, well inside the array); should it not fit, one chunk per
  // channel group is the smallest layout there is.
  int chunk = scan_auto_chunk(batch, seqlen, d_inner, dtype, bc_dtype);
  if (scan_workspace_bytes(batch, seqlen, d_inner, chunk) > kStaticScratchBytes) chunk = (seqlen + 15) & ~15;
  if (scan_workspace_bytes(batch, seqlen, d_inner, chunk) > kStaticScratchBytes)
    return fail(JAMBA_ERR_UNSUPPORTED,
                "static scan: batch * ceil(d_inner / 256) = " + std::to_string((long long)batch * ((d_inner + 255) / 256)) +
                    " channel groups need more than the 32 MiB static scratch (at most 682 groups)");

  StaticAddrs sa;
  JB_TRY(static_addrs(&sa));
  ScanCall sc = {};
  sc.x = x; sc.ld_x = ld_x; sc.z = z; sc.ld_z = ld_z; sc.dt = dt; sc.ld_dt = ld_dt;
  sc.B = B; sc.ld_b = ld_b; sc.C = C; sc.ld_c = ld_c; sc.bc_dtype = bc_dtype;
  sc.A = A; sc.D = D; sc.h0 = h0; sc.y = y; sc.ld_y = ld_y; sc.h_out = h_out;
  sc.batch = batch; sc.L = seqlen; sc.di = d_inner; sc.dtype = dtype; sc.chunk = chunk;
  sc.ws = sa.scratch;
  sc.ws_bytes = kStaticScratchBytes;
  sc.err = status ? status : sa.status;
  return scan_run(sc, reinterpret_cast<cudaStream_t>(stream));
}
