// Host-side internals: error strings, device queries, tensor-map encoding.
#include <mutex>
#include <string>

#include "host.hpp"

namespace jb {

static thread_local std::string t_last_error = "no error";

jamba_status fail(jamba_status st, const std::string& msg) {
  t_last_error = msg;
  return st;
}

const char* last_error() { return t_last_error.c_str(); }

jamba_status cuda_fail(cudaError_t e, const char* what) {
  t_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return JAMBA_ERR_CUDA;
}

static constexpr int kMaxDevices = 64;

int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int* device_error_word() {
  static int* words[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!words[dev]) {
    int* w = nullptr;
    if (cudaMalloc(&w, sizeof(int)) != cudaSuccess) return nullptr;
    if (cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return nullptr;
    words[dev] = w;
  }
  return words[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

jamba_status make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t inner, uint64_t rows, uint64_t row_stride, uint32_t box_inner,
                         uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto enc = encoder();
  if (!enc) return fail(JAMBA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (!aligned16(base) || (row_stride & 15u) || rows == 0 || inner == 0)
    return fail(JAMBA_ERR_INVALID_ARG, "tensor map: base/stride must be 16-byte aligned and sizes positive");
  (void)elem_bytes;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(JAMBA_ERR_CUDA, "cuTensorMapEncodeTiled (2-D) failed: " + std::to_string((int)r));
  return JAMBA_OK;
}

jamba_status make_map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                         uint64_t inner, uint64_t rows, uint64_t outer, uint64_t row_stride,
                         uint64_t outer_stride, uint32_t box_inner, uint32_t box_rows,
                         CUtensorMapSwizzle sw, uint32_t box_outer) {
  auto enc = encoder();
  if (!enc) return fail(JAMBA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if (!aligned16(base) || (row_stride & 15u) || (outer_stride & 15u))
    return fail(JAMBA_ERR_INVALID_ARG, "tensor map: base/strides must be 16-byte aligned");
  (void)elem_bytes;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {row_stride, outer_stride};
  cuuint32_t box[3] = {box_inner, box_rows, box_outer};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(JAMBA_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed: " + std::to_string((int)r));
  return JAMBA_OK;
}

int choose_splits(int M, int N, int K, int bn, int min_k_tiles) {
  const int tiles = ((M + 127) / 128) * ((N + bn - 1) / bn);
  const int k_tiles = (K + 63) / 64;
  const int sms = num_sms();
  if (tiles >= sms) return 1;
  int s = sms / tiles;  // stay within one wave of CTAs
  if (s < 1) s = 1;
  int max_s = k_tiles / (min_k_tiles > 0 ? min_k_tiles : 1);
  if (max_s < 1) max_s = 1;
  if (s > max_s) s = max_s;
  if (s > 32) s = 32;
  // every split must own at least one k-step
  const int per = (k_tiles + s - 1) / s;
  return (k_tiles + per - 1) / per;
}

}  // namespace jb
