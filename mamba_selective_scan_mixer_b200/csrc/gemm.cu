// GEMM launchers: the tcgen05 kernel for bf16, the INT8-weight grouped expert
// kernel, and a CUDA-core kernel for the fp32 path (fp32 inputs must keep ~1e-5
// accuracy, which TF32 would not).
#include <string>

#include "gemm_i8w.cuh"
#include "gemm_tc.cuh"
#include "host.hpp"

namespace jb {

template <int BN, int STAGES, int EPI, bool TRANS, int EW = GEMM_EPI_WARPS>
static jamba_status launch_tc(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                              const CUtensorMap& mc, const GemmParams& p, int grid, cudaStream_t s) {
  using S = GemmSmem<BN, STAGES, EPI == EPI_SOFTPLUS && !TRANS, EW, gemm_nstg<EW>()>;
  static std::atomic<bool> configured[64];
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN, STAGES, EPI, TRANS, EW>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::BYTES));
    configured[dev] = true;
  }
  JB_CUDA(launch_pdl(gemm_bf16_tc_kernel<BN, STAGES, EPI, TRANS, EW>, dim3(grid), dim3(64 + 32 * EW), S::BYTES, s,
                     ma, mb, mb2, mc, p));
  return JAMBA_OK;
}

template <int EPI, int MT>
static jamba_status launch_i8w(const CUtensorMap& ma, const CUtensorMap& mq, const CUtensorMap& mq2,
                               const GemmParams& p, int grid, cudaStream_t s) {
  using S = I8wSmem<MT>;
  static std::atomic<bool> configured[64];
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(gemm_i8w_kernel<EPI, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)S::BYTES));
    configured[dev] = true;
  }
  JB_CUDA(launch_pdl(gemm_i8w_kernel<EPI, MT>, dim3(grid), dim3(I8W_THREADS), S::BYTES, s, ma, mq, mq2, p));
  return JAMBA_OK;
}

template <int EPI>
static jamba_status launch_i8t(const CUtensorMap& ma, const CUtensorMap& mq, const CUtensorMap& mq2,
                               const GemmParams& p, int grid, cudaStream_t s) {
  using S = I8tSmem<EPI>;
  static std::atomic<bool> configured[64];
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(gemm_i8w_tok_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)S::BYTES));
    configured[dev] = true;
  }
  JB_CUDA(launch_pdl(gemm_i8w_tok_kernel<EPI>, dim3(grid), dim3(i8t_threads<EPI>()), S::BYTES, s, ma, mq, mq2, p));
  return JAMBA_OK;
}

template <int EPI, bool TRANS>
static jamba_status launch_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                              const CUtensorMap& mc, const GemmParams& p, int grid, cudaStream_t s) {
  if constexpr (TRANS) {
    if (bn == 64) return launch_tc<64, 8, EPI, true>(ma, mb, mb2, mc, p, grid, s);
  } else if constexpr (EPI == EPI_SOFTPLUS) {
    // bias + softplus of every output element: sixteen epilogue warps (four per
    // scheduler) keep the epilogue, which bounds this GEMM (K = dt_rank is
    // short), fed; three ring stages and one TMA-store box per epilogue warp
    // share the 227 KB
    if (bn == 256) return launch_tc<256, 3, EPI, false, 16>(ma, mb, mb2, mc, p, grid, s);
  } else if constexpr (EPI == EPI_SWIGLU || EPI == EPI_CONVP) {
    if (bn == 256) return launch_tc<256, 4, EPI, false>(ma, mb, mb2, mc, p, grid, s);
  } else {
    switch (bn) {
      case 64: return launch_tc<64, 8, EPI, false>(ma, mb, mb2, mc, p, grid, s);
      case 128: return launch_tc<128, 6, EPI, false>(ma, mb, mb2, mc, p, grid, s);
      case 144: return launch_tc<144, 6, EPI, false>(ma, mb, mb2, mc, p, grid, s);
      case 256: return launch_tc<256, 4, EPI, false>(ma, mb, mb2, mc, p, grid, s);
      default: break;
    }
  }
  return fail(JAMBA_ERR_UNSUPPORTED, "gemm: no kernel for tile width " + std::to_string(bn) + " with this epilogue");
}

// Grouped expert GEMMs with INT8 weights (see gemm_i8w.cuh), by the average
// number of routed rows per expert: up to 32, the weights take the M side
// (decode batches: bound by streaming the codes); up to 255, 128-row tiles
// with double-buffered accumulators; from 256, two 128-row halves share one
// widened weight tile.
// k-splits for the fp32 (down) expert GEMM with INT8 weights when the weights
// take the M side: the split count (1 to 4, an even number of 64-deep steps
// each) whose last wave of 128-row weight tiles over the SMs leaves the
// fewest idle, assuming every group holds one token tile (decode batches).
int i8w_splits(int M, int num_groups, int N, int K) {
  if (num_groups <= 0 || M / num_groups > I8T_BNT || N % 128 || K % 128) return 1;
  const long long tiles = (long long)(M < num_groups ? M : num_groups) * (N / 128);
  const int k_tiles = K / 64, sms = num_sms();
  int best = 1;
  double best_cost = 1e30;
  for (int sp = 1; sp <= 4; ++sp) {
    if (k_tiles % (2 * sp)) continue;
    const long long units = tiles * sp;
    const double cost = (double)((units + sms - 1) / sms) / sp;   // waves, in whole-tile times
    if (cost < best_cost - 1e-9) { best_cost = cost; best = sp; }
  }
  return best;
}

static jamba_status gemm_i8w(const GemmDesc& g, cudaStream_t s) {
  if (!g.grouped || g.transpose_out || g.residual || (g.epi != EPI_SWIGLU && g.epi != EPI_F32))
    return fail(JAMBA_ERR_UNSUPPORTED, "gemm: INT8 weights only in the grouped SwiGLU / fp32 expert GEMMs");
  if (!g.scale_b || (g.epi == EPI_SWIGLU && (!g.scale_b2 || !g.b2)) || !aligned16(g.scale_b) ||
      (g.scale_b2 && !aligned16(g.scale_b2)) || g.N % 4 || g.ldb % 16 || g.K % 16 || !aligned16(g.b) ||
      (g.b2 && !aligned16(g.b2)))
    return fail(JAMBA_ERR_INVALID_ARG,
                "gemm: INT8 weights need 16-byte aligned codes and scales, N a multiple of 4, K and ldb of 16");
  const int avg_rows = g.M / g.num_groups;
  const bool tok = avg_rows <= I8T_BNT;
  const int bn_out = tok ? 128 : g.epi == EPI_SWIGLU ? I8W_BN / 2 : I8W_BN;
  const uint32_t q_box = (uint32_t)(tok ? 128 : bn_out);
  const uint32_t q_inner = tok ? 128 : 64;   // codes per row per load
  const CUtensorMapSwizzle q_sw = tok ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap ma, mq, mq2;
  JB_TRY(make_map_2d(&ma, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.K, (uint64_t)g.M,
                     (uint64_t)g.lda * 2, 64, tok ? I8T_BNT : 128, CU_TENSOR_MAP_SWIZZLE_128B));
  const uint64_t rs = (uint64_t)g.ldb, os = rs * (uint64_t)g.b_rows;
  JB_TRY(make_map_3d(&mq, g.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)g.K, (uint64_t)g.b_rows,
                     (uint64_t)(g.group_mod > 0 ? g.group_mod : g.num_groups), rs, os, q_inner, q_box, q_sw));
  mq2 = mq;
  if (g.b2)
    JB_TRY(make_map_3d(&mq2, g.b2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)g.K, (uint64_t)g.b_rows,
                       (uint64_t)(g.group_mod > 0 ? g.group_mod : g.num_groups), rs, os, q_inner, q_box, q_sw));
  GemmParams p = {};
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.k_tiles = (g.K + 63) / 64;
  p.splits = g.splits < 1 ? 1 : g.splits;
  if (p.splits > 1 && (!tok || g.epi != EPI_F32 || p.k_tiles % (2 * p.splits) || g.split_stride < (long long)g.M * g.ldo))
    return fail(JAMBA_ERR_INVALID_ARG,
                "gemm: INT8 k-splits only in the few-row fp32 GEMM, an even number of 64-deep steps per split");
  p.k_tiles_per_split = p.k_tiles / p.splits;
  p.split_stride = g.split_stride;
  p.n_tiles = (g.N + bn_out - 1) / bn_out;
  p.grouped = 1;
  p.offsets = g.offsets;
  p.num_groups = g.num_groups;
  p.group_mod = g.group_mod;
  p.out = g.out;
  p.ldo = g.ldo;
  p.scale_b = g.scale_b;
  p.scale_b2 = g.scale_b2;
  p.err = device_error_word();
  if (!p.err) return fail(JAMBA_ERR_CUDA, "could not allocate the device status word");
  if (tok) {
    if (g.N % 128 || g.K % 128)
      return fail(JAMBA_ERR_INVALID_ARG, "gemm: INT8 weights with few rows need N and K multiples of 128");
    const long long tiles = (long long)((g.M + I8T_BNT - 1) / I8T_BNT + g.num_groups) * p.n_tiles * p.splits;
    const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
    return g.epi == EPI_SWIGLU ? launch_i8t<EPI_SWIGLU>(ma, mq, mq2, p, grid, s)
                               : launch_i8t<EPI_F32>(ma, mq, mq2, p, grid, s);
  }
  const bool pairs = avg_rows >= 256;
  const int mh = pairs ? 256 : 128;
  const long long tiles = (long long)((g.M + mh - 1) / mh + g.num_groups) * p.n_tiles;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  if (g.epi == EPI_SWIGLU)
    return pairs ? launch_i8w<EPI_SWIGLU, 2>(ma, mq, mq2, p, grid, s) : launch_i8w<EPI_SWIGLU, 1>(ma, mq, mq2, p, grid, s);
  return pairs ? launch_i8w<EPI_F32, 2>(ma, mq, mq2, p, grid, s) : launch_i8w<EPI_F32, 1>(ma, mq, mq2, p, grid, s);
}

jamba_status gemm_bf16(const GemmDesc& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return fail(JAMBA_ERR_INVALID_ARG, "gemm: sizes must be positive");
  if (!g.a || !g.b || !g.out) return fail(JAMBA_ERR_INVALID_ARG, "gemm: null operand");
  if (g.K % 8 || g.lda % 8 || g.ldb % 8 || !aligned16(g.a) || !aligned16(g.b))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: K and leading dimensions must be multiples of 8, operands 16-byte aligned");
  if (!g.transpose_out && !aligned16(g.out)) return fail(JAMBA_ERR_INVALID_ARG, "gemm: output must be 16-byte aligned");
  if (!g.transpose_out && ((g.epi == EPI_BF16 || g.epi == EPI_SWIGLU || g.epi == EPI_CONVP) ? g.ldo % 8 : g.ldo % 4))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: output leading dimension breaks 16-byte rows");
  if (g.residual && (g.transpose_out || g.epi != EPI_BF16 || g.ldr % 8 || !aligned16(g.residual)))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: residual only with aligned non-transposed bf16 output");
  if (g.splits > 1 && (g.epi != EPI_F32 || (g.grouped && !g.b_int8)))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: split-K writes fp32 partials only");
  if (g.epi == EPI_SWIGLU && (!g.grouped || !g.b2))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: SwiGLU needs grouped gate and up weights");
  if (g.epi == EPI_CONV && (!g.transpose_out || g.splits > 1 || !g.conv_w || !g.conv_b || !g.conv_state ||
                            !g.xc_out || g.conv_c <= 0 || g.conv_c > g.M ||
                            (reinterpret_cast<uintptr_t>(g.conv_w) & 7)))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: the conv epilogue needs a swap-AB GEMM and its conv operands");
  if (g.epi == EPI_CONVP &&
      (g.transpose_out || g.grouped || g.splits > 1 || g.residual || !g.conv_w || !g.conv_b || !g.xc_out ||
       g.conv_c <= 0 || g.conv_c % 32 || g.N != 2 * g.conv_c || g.conv_L < 3 || g.M % g.conv_L ||
       !aligned16(g.conv_w) || (reinterpret_cast<uintptr_t>(g.conv_b) & 3) || !aligned16(g.xc_out) ||
       (g.bn && g.bn != 256)))
    return fail(JAMBA_ERR_INVALID_ARG, "gemm: the prefill conv epilogue needs x|z columns (2 x a multiple of 32), "
                                       "sequences of at least 3 rows and aligned conv operands");
  if (g.b_int8) return gemm_i8w(g, s);
  int bn = g.epi == EPI_CONVP ? 256 : g.bn;
  if (bn == 0) {
    if (g.epi == EPI_SWIGLU || g.epi == EPI_SOFTPLUS) bn = g.transpose_out ? 64 : 256;
    else if (g.transpose_out || g.N <= 64) bn = 64;
    else if (g.N <= 128) bn = 128;
    else if (g.N <= 144 || g.N == 288) bn = 144;
    else bn = 256;
  }
  const int bn_out = g.epi == EPI_SWIGLU ? bn / 2 : bn;
  const int b_box = g.epi == EPI_SWIGLU ? bn / 2 : bn;

  CUtensorMap ma, mb, mb2;
  const uint64_t a_rows = (uint64_t)g.M;
  JB_TRY(make_map_2d(&ma, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.K, a_rows,
                     (uint64_t)g.lda * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
  if (!g.grouped) {
    JB_TRY(make_map_2d(&mb, g.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.K, (uint64_t)g.N,
                       (uint64_t)g.ldb * 2, 64, (uint32_t)b_box, CU_TENSOR_MAP_SWIZZLE_128B));
    mb2 = mb;
  } else {
    const uint64_t rs = (uint64_t)g.ldb * 2, os = rs * (uint64_t)g.b_rows;
    JB_TRY(make_map_3d(&mb, g.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.K, (uint64_t)g.b_rows,
                       (uint64_t)(g.group_mod > 0 ? g.group_mod : g.num_groups), rs, os, 64, (uint32_t)b_box, CU_TENSOR_MAP_SWIZZLE_128B));
    if (g.b2) {
      JB_TRY(make_map_3d(&mb2, g.b2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.K, (uint64_t)g.b_rows,
                         (uint64_t)(g.group_mod > 0 ? g.group_mod : g.num_groups), rs, os, 64, (uint32_t)b_box, CU_TENSOR_MAP_SWIZZLE_128B));
    } else {
      mb2 = mb;
    }
  }

  CUtensorMap mc = mb;
  if (g.epi == EPI_SOFTPLUS && !g.transpose_out)
    JB_TRY(make_map_2d(&mc, g.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)g.N, (uint64_t)g.M,
                       (uint64_t)g.ldo * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B));

  GemmParams p = {};
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.k_tiles = (g.K + 63) / 64;
  p.splits = g.splits < 1 ? 1 : g.splits;
  p.k_tiles_per_split = (p.k_tiles + p.splits - 1) / p.splits;
  p.splits = (p.k_tiles + p.k_tiles_per_split - 1) / p.k_tiles_per_split;
  p.m_tiles = (g.M + 127) / 128;
  p.n_tiles = (g.N + bn_out - 1) / bn_out;
  {
    // raster bands: as many m-tiles as keep their A rows within 32 MB, from
    // 16 to 32 of them.  A wave of CTAs then spans the band's whole height
    // and several n-tiles, and the next wave finds the same A rows in L2 as
    // long as they and a wave's B and C tiles fit it with room to spare: B
    // bands of 64 MB (with ~20 MB of A and C per wave) were measured to miss
    // on every wave, A bands of 16, 24 and 32 MB to hit.  Taller bands (512
    // m-tiles for dt_proj's K = 256) leave a wave inside one n-tile, and its
    // large output pushes the band out of L2 before the next n-tile reuses
    // it (dt_proj 0.95 -> 1.10 ms).  B is read once per band.
    const long long band_bytes = 128ll * g.K * 2;
    long long fit = (32ll << 20) / band_bytes;
    fit = fit < 16 ? 16 : fit > 32 ? 32 : fit;
    p.band_m = (int)(fit > p.m_tiles ? p.m_tiles : fit);
  }
  p.grouped = g.grouped;
  p.offsets = g.offsets;
  p.num_groups = g.num_groups;
  p.group_mod = g.group_mod;
  p.out = g.out;
  p.ldo = g.ldo;
  p.split_stride = g.split_stride;
  p.residual = g.residual;
  p.ldr = g.ldr;
  p.bias = g.bias;
  p.conv_w = reinterpret_cast<const bf16*>(g.conv_w);
  p.conv_b = reinterpret_cast<const bf16*>(g.conv_b);
  p.conv_state = g.conv_state;
  p.xc_out = reinterpret_cast<bf16*>(g.xc_out);
  p.conv_c = g.conv_c;
  p.conv_in = g.conv_in;
  p.conv_out = g.conv_out;
  p.conv_perm = g.conv_perm;
  p.conv_L = g.conv_L;
  p.err = device_error_word();
  if (!p.err) return fail(JAMBA_ERR_CUDA, "could not allocate the device status word");

  long long tiles = g.grouped ? (long long)(p.m_tiles + g.num_groups) * p.n_tiles
                              : (long long)p.m_tiles * p.n_tiles * p.splits;
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  if (g.transpose_out) {
    switch (g.epi) {
      case EPI_BF16: return launch_bn<EPI_BF16, true>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_F32: return launch_bn<EPI_F32, true>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_SOFTPLUS: return launch_bn<EPI_SOFTPLUS, true>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_CONV: return launch_bn<EPI_CONV, true>(bn, ma, mb, mb2, mc, p, grid, s);
      default: break;
    }
  } else {
    switch (g.epi) {
      case EPI_BF16: return launch_bn<EPI_BF16, false>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_F32: return launch_bn<EPI_F32, false>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_SOFTPLUS: return launch_bn<EPI_SOFTPLUS, false>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_SWIGLU: return launch_bn<EPI_SWIGLU, false>(bn, ma, mb, mb2, mc, p, grid, s);
      case EPI_CONVP: return launch_bn<EPI_CONVP, false>(bn, ma, mb, mb2, mc, p, grid, s);
      default: break;
    }
  }
  return fail(JAMBA_ERR_UNSUPPORTED, "gemm: unknown epilogue");
}

// ---------------------------------------------------------------- fp32 path
// 64 x 64 output tile per 256-thread block, 4 x 4 per thread, k-steps of 16.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, long long lda,
                                                       const float* __restrict__ B, long long ldb, int M, int N,
                                                       int K, int epi, int trans, GemmParams p) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  griddep_wait();
  griddep_launch();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i >> 4, k = i & 15;
      As[k][r] = (m0 + r < M && k0 + k < K) ? A[(long long)(m0 + r) * lda + k0 + k] : 0.f;
      Bs[k][r] = (n0 + r < N && k0 + k < K) ? B[(long long)(n0 + r) * ldb + k0 + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[k][ty * 4 + i];
        b[i] = Bs[k][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = reinterpret_cast<float*>(p.out);
  const float* res = reinterpret_cast<const float*>(p.residual);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (epi == EPI_SOFTPLUS) v = softplus(v + p.bias[trans ? m : n]);
      if (trans) {
        out[(long long)n * p.ldo + m] = v;
      } else {
        if (res) v += res[(long long)m * p.ldr + n];
        out[(long long)m * p.ldo + n] = v;
      }
    }
  }
}

jamba_status gemm_f32(const GemmDesc& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return fail(JAMBA_ERR_INVALID_ARG, "gemm: sizes must be positive");
  if (!g.a || !g.b || !g.out) return fail(JAMBA_ERR_INVALID_ARG, "gemm: null operand");
  if (g.grouped || g.splits > 1 || (g.epi != EPI_F32 && g.epi != EPI_SOFTPLUS))
    return fail(JAMBA_ERR_UNSUPPORTED, "fp32 gemm: dense, unsplit, fp32 or softplus epilogue only");
  GemmParams p = {};
  p.out = g.out;
  p.ldo = g.ldo;
  p.residual = g.residual;
  p.ldr = g.ldr;
  p.bias = g.bias;
  dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
  JB_CUDA(launch_pdl(gemm_f32_kernel, grid, dim3(256), 0, s, reinterpret_cast<const float*>(g.a), g.lda,
                     reinterpret_cast<const float*>(g.b), g.ldb, g.M, g.N, g.K, g.epi, g.transpose_out, p));
  return JAMBA_OK;
}

}  // namespace jb
