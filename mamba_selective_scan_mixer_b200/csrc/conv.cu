// Causal depthwise conv1d (d_conv = 4) + SiLU, prefill and decode step.
//
// Mamba layer used by Jamba ("Jamba: A Hybrid Transformer-Mamba Language
// Model", section 2, ref [17]): xc[t, c] = SiLU(b[c] + sum_k w[c, k] x[t-3+k, c]),
// x at negative times taken from the cache (the last three pre-conv inputs,
// oldest first) or zero.
//
// The bf16 prefill runs the conv in the in_proj GEMM's epilogue (gemm_tc.cuh,
// EPI_CONVP); conv_fixup_kernel here finishes the few rows that epilogue
// defers.  The standalone prefill kernel serves the fp32 path, sequences of
// fewer than three steps and jamba_causal_conv1d: each thread owns 16 bytes
// of channels (8 bf16 or 4 fp32) over a run of 64 time steps, keeping the
// three previous inputs in registers, so every input row is read once (plus
// a 3-row halo per run) with 16-byte loads that are contiguous across the
// warp; eight rows are requested at a time so that enough bytes are in
// flight to stream at HBM speed.
#include "common.cuh"
#include "host.hpp"

namespace jb {

constexpr int CONV_TQ = 64;
constexpr int CONV_THREADS = 128;
constexpr int CONV_BATCH = 8;   // input rows a thread has in flight

template <typename T> struct Vec16;
template <> struct Vec16<bf16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const bf16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(bf16* p, const float* v) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const float* p, float* v) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <typename T>
__global__ void __launch_bounds__(CONV_THREADS)
conv_prefill_kernel(const T* __restrict__ x, long long ld_x, const T* __restrict__ w, const T* __restrict__ bias,
                    T* __restrict__ out, const float* __restrict__ st_in, float* __restrict__ st_out, int L,
                    int C, const int* __restrict__ perm, int* err) {
  constexpr int V = Vec16<T>::N;
  griddep_wait();
  griddep_launch();
  const int c0 = (blockIdx.x * CONV_THREADS + threadIdx.x) * V;
  if (c0 >= C) return;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * CONV_TQ;
  const int t1 = min(L, t0 + CONV_TQ);
  float wk[4][V], bv[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
#pragma unroll
    for (int k = 0; k < 4; ++k) wk[k][i] = to_f(w[(long long)(c0 + i) * 4 + k]);
    bv[i] = to_f(bias[c0 + i]);
  }
  const T* xb = x + (long long)b * L * ld_x;
  float win[3][V];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int t = t0 - 3 + k;
    if (t >= 0) {
      Vec16<T>::load(xb + (long long)t * ld_x + c0, win[k]);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int cn = perm ? __ldg(perm + c0 + i) : c0 + i;   // cache row of this channel
        win[k][i] = st_in && checked(cn >= 0 && cn < C, err) ? st_in[((long long)b * C + cn) * 3 + (3 + t)] : 0.f;
      }
    }
  }
  T* ob = out + (long long)b * L * C;
  // eight input rows requested together (kept as raw 16-byte words), then consumed in order
  for (int tb = t0; tb < t1; tb += CONV_BATCH) {
    const int nb = min(CONV_BATCH, t1 - tb);
    uint4 raw[CONV_BATCH];
#pragma unroll
    for (int j = 0; j < CONV_BATCH; ++j)
      if (j < nb) raw[j] = *reinterpret_cast<const uint4*>(xb + (long long)(tb + j) * ld_x + c0);
#pragma unroll
    for (int j = 0; j < CONV_BATCH; ++j) {
      if (j >= nb) break;
      float cur[V], o[V];
      Vec16<T>::load(reinterpret_cast<const T*>(&raw[j]), cur);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        float acc = bv[i];
        acc = fmaf(wk[0][i], win[0][i], acc);
        acc = fmaf(wk[1][i], win[1][i], acc);
        acc = fmaf(wk[2][i], win[2][i], acc);
        acc = fmaf(wk[3][i], cur[i], acc);
        o[i] = silu(acc);
        win[0][i] = win[1][i];
        win[1][i] = win[2][i];
        win[2][i] = cur[i];
      }
      Vec16<T>::store(ob + (long long)(tb + j) * C + c0, o);
    }
  }
  if (st_out && t1 == L) {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int cn = perm ? __ldg(perm + c0 + i) : c0 + i;
      if (!checked(cn >= 0 && cn < C, err)) continue;
#pragma unroll
      for (int k = 0; k < 3; ++k) st_out[((long long)b * C + cn) * 3 + k] = win[k][i];
    }
  }
}

// decode: one thread per (batch row, channel); the cache shifts in place
template <typename T>
__global__ void __launch_bounds__(256)
conv_step_kernel(const T* __restrict__ x, long long ld_x, const T* __restrict__ w, const T* __restrict__ bias,
                 T* __restrict__ out, float* __restrict__ state, int batch, int C) {
  griddep_wait();
  griddep_launch();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)batch * C) return;
  const int b = (int)(i / C), c = (int)(i - (long long)b * C);
  float* s = state + i * 3;
  const float s0 = s[0], s1 = s[1], s2 = s[2];
  const float xv = to_f(x[(long long)b * ld_x + c]);
  float acc = to_f(bias[c]);
  acc = fmaf(to_f(w[(long long)c * 4 + 0]), s0, acc);
  acc = fmaf(to_f(w[(long long)c * 4 + 1]), s1, acc);
  acc = fmaf(to_f(w[(long long)c * 4 + 2]), s2, acc);
  acc = fmaf(to_f(w[(long long)c * 4 + 3]), xv, acc);
  out[i] = from_f<T>(silu(acc));
  s[0] = s1;
  s[1] = s2;
  s[2] = xv;
}

// conv cache [batch, C, 3] (fp32, oldest first) from the in_proj rows of the
// three tokens before a sequence slice: xz [batch * 3, *], x in the first C columns
template <typename T>
__global__ void __launch_bounds__(256)
conv_halo_kernel(const T* __restrict__ xz, long long ld, float* __restrict__ state, int batch, int C) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // flat (row, channel, tap)
  if (i >= (long long)batch * C * 3) return;
  const int k = (int)(i % 3);
  const long long bc = i / 3;
  const int b = (int)(bc / C), c = (int)(bc - (long long)b * C);
  state[i] = to_f(xz[((long long)b * 3 + k) * ld + c]);
}

// The rows an EPI_CONVP in_proj epilogue deferred: in each 32-row slab, rows
// j = 0..2 whose position t in their sequence exceeds j (their window reaches
// the slab above).  The epilogue left the raw x of slab rows 0-2 and 29-31 in
// the x columns of xz; taps before the sequence start come from the cache.
// A thread owns 8 channels and walks the slabs s = blockIdx.y, += gridDim.y
// (one wave of blocks), the six raw rows of the next slab in
// flight while the current one is computed.
constexpr int FIX_THREADS = 128;

__device__ __forceinline__ void fix_load(const bf16* __restrict__ xz, long long ld, int c0, int T, int s,
                                         uint4 (&raw)[6]) {
#pragma unroll
  for (int r = 0; r < 6; ++r) {
    const int row = s * 32 - 3 + r;
    raw[r] = row >= 0 && row < T ? *reinterpret_cast<const uint4*>(xz + (long long)row * ld + c0) : make_uint4(0, 0, 0, 0);
  }
}

__global__ void __launch_bounds__(FIX_THREADS)
conv_fixup_kernel(const bf16* __restrict__ xz, long long ld, const bf16* __restrict__ w, const bf16* __restrict__ bias,
                  bf16* __restrict__ xc, const float* __restrict__ st_in, int T, int L, int C,
                  const int* __restrict__ perm, int* err) {
  griddep_wait();
  griddep_launch();
  const int c0 = (blockIdx.x * FIX_THREADS + threadIdx.x) * 8;
  if (c0 >= C) return;
  const int slabs = (T + 31) / 32;
  int s = blockIdx.y;
  if (s >= slabs) return;
  uint4 cur[6], nxt[6];
  fix_load(xz, ld, c0, T, s, cur);
  float wk[4][8], bv[8];
  {
    const uint4* wq = reinterpret_cast<const uint4*>(w + (long long)c0 * 4);   // 8 channels x 4 taps
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float f[8];
      Vec16<bf16>::load(reinterpret_cast<const bf16*>(wq + q), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) wk[e & 3][2 * q + (e >> 2)] = f[e];
    }
    Vec16<bf16>::load(bias + c0, bv);
  }
  for (; s < slabs; s += gridDim.y) {
    const int sn = s + gridDim.y;
    if (sn < slabs) fix_load(xz, ld, c0, T, sn, nxt);
    float xw[6][8];
#pragma unroll
    for (int r = 0; r < 6; ++r) Vec16<bf16>::load(reinterpret_cast<const bf16*>(&cur[r]), xw[r]);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int m = s * 32 + j;
      if (m >= T) break;
      const int b = m / L, t = m - b * L;
      if (t <= j) continue;   // computed by the epilogue
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float x[4];   // x[t-3], x[t-2], x[t-1], x[t]
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int tk = t - 3 + k;
          if (tk >= 0) {
            x[k] = xw[j + k][i];
          } else {
            const int cn = perm ? __ldg(perm + c0 + i) : c0 + i;
            x[k] = st_in && checked(cn >= 0 && cn < C, err) ? st_in[((long long)b * C + cn) * 3 + (3 + tk)] : 0.f;
          }
        }
        float acc = bv[i];
        acc = fmaf(wk[0][i], x[0], acc);
        acc = fmaf(wk[1][i], x[1], acc);
        acc = fmaf(wk[2][i], x[2], acc);
        acc = fmaf(wk[3][i], x[3], acc);
        o[i] = silu(acc);
      }
      Vec16<bf16>::store(xc + (long long)m * C + c0, o);
    }
#pragma unroll
    for (int r = 0; r < 6; ++r) cur[r] = nxt[r];
  }
}

jamba_status conv_fixup(const void* xz, long long ld, const void* w, const void* b, void* xc, const float* st_in,
                        int T, int L, int C, const int* perm, cudaStream_t s) {
  if (C % 8 || ld % 8 || !aligned16(xz) || !aligned16(xc) || !aligned16(w) || !aligned16(b) || L < 1)
    return fail(JAMBA_ERR_INVALID_ARG, "conv fix-up: channels and row stride must fill 16-byte vectors");
  const int slabs = (T + 31) / 32;
  const int cblocks = (C / 8 + FIX_THREADS - 1) / FIX_THREADS;
  int sy = 3 * num_sms() / cblocks;   // one wave: three blocks per SM (156 registers a thread)
  sy = sy < 1 ? 1 : sy > slabs ? slabs : sy;
  JB_CUDA(launch_pdl(conv_fixup_kernel, dim3(cblocks, sy), dim3(FIX_THREADS), 0, s, reinterpret_cast<const bf16*>(xz),
                     ld, reinterpret_cast<const bf16*>(w), reinterpret_cast<const bf16*>(b), reinterpret_cast<bf16*>(xc),
                     st_in, T, L, C, perm, device_error_word()));
  return JAMBA_OK;
}

jamba_status conv_halo_state(const void* xz, long long ld, float* state, int batch, int C, int dtype,
                             cudaStream_t s) {
  const long long n = (long long)batch * C * 3;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == JAMBA_BF16)
    conv_halo_kernel<bf16><<<grid, 256, 0, s>>>(reinterpret_cast<const bf16*>(xz), ld, state, batch, C);
  else
    conv_halo_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(xz), ld, state, batch, C);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status conv_prefill(const void* x, long long ld_x, const void* w, const void* b, void* out,
                          const float* st_in, float* st_out, int batch, int L, int C, int dtype, const int* perm,
                          cudaStream_t s) {
  const int V = dtype == JAMBA_BF16 ? 8 : 4;
  if (C % V || ld_x % V || !aligned16(x) || !aligned16(out))
    return fail(JAMBA_ERR_INVALID_ARG, "conv: channels and row stride must fill 16-byte vectors");
  dim3 grid((C / V + CONV_THREADS - 1) / CONV_THREADS, (L + CONV_TQ - 1) / CONV_TQ, batch);
  if (dtype == JAMBA_BF16)
    JB_CUDA(launch_pdl(conv_prefill_kernel<bf16>, grid, dim3(CONV_THREADS), 0, s, reinterpret_cast<const bf16*>(x),
                       ld_x, reinterpret_cast<const bf16*>(w), reinterpret_cast<const bf16*>(b),
                       reinterpret_cast<bf16*>(out), st_in, st_out, L, C, perm, device_error_word()));
  else
    JB_CUDA(launch_pdl(conv_prefill_kernel<float>, grid, dim3(CONV_THREADS), 0, s, reinterpret_cast<const float*>(x),
                       ld_x, reinterpret_cast<const float*>(w), reinterpret_cast<const float*>(b),
                       reinterpret_cast<float*>(out), st_in, st_out, L, C, perm, device_error_word()));
  return JAMBA_OK;
}

jamba_status conv_step(const void* x, long long ld_x, const void* w, const void* b, void* out, float* state,
                       int batch, int C, int dtype, cudaStream_t s) {
  const long long n = (long long)batch * C;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == JAMBA_BF16)
    JB_CUDA(launch_pdl(conv_step_kernel<bf16>, dim3(grid), dim3(256), 0, s, reinterpret_cast<const bf16*>(x), ld_x,
                       reinterpret_cast<const bf16*>(w), reinterpret_cast<const bf16*>(b),
                       reinterpret_cast<bf16*>(out), state, batch, C));
  else
    JB_CUDA(launch_pdl(conv_step_kernel<float>, dim3(grid), dim3(256), 0, s, reinterpret_cast<const float*>(x), ld_x,
                       reinterpret_cast<const float*>(w), reinterpret_cast<const float*>(b),
                       reinterpret_cast<float*>(out), state, batch, C));
  return JAMBA_OK;
}

// ------------------------------------------------------------ weight reordering
// dst row r = src row perm[r]; 16-byte words when rows and pointers allow it,
// else 2-byte elements (row_bytes is even for every weight reordered here).
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, const int* __restrict__ perm,
                   int rows, int row_bytes, int word, int* err) {
  const int per_row = row_bytes / word;
  const long long n = (long long)rows * per_row;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / per_row), e = (int)(i - (long long)r * per_row);
    const int pr = __ldg(perm + r);
    if (!checked(pr >= 0 && pr < rows, err)) continue;
    const long long so = (long long)pr * row_bytes + (long long)e * word;
    const long long d = (long long)r * row_bytes + (long long)e * word;
    if (word == 16) *reinterpret_cast<uint4*>(dst + d) = *reinterpret_cast<const uint4*>(src + so);
    else if (word == 4) *reinterpret_cast<uint32_t*>(dst + d) = *reinterpret_cast<const uint32_t*>(src + so);
    else *reinterpret_cast<uint16_t*>(dst + d) = *reinterpret_cast<const uint16_t*>(src + so);
  }
}

// dst[i, j] = src[i, perm[j]] for a [rows, cols] matrix of 2- or 4-byte elements
__global__ void __launch_bounds__(256)
gather_cols_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, const int* __restrict__ perm, int rows,
                   int cols, int esize, int* err) {
  const long long n = (long long)rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / cols), j = (int)(i - (long long)r * cols);
    const int pj = __ldg(perm + j);
    if (!checked(pj >= 0 && pj < cols, err)) continue;
    const long long so = ((long long)r * cols + pj) * esize;
    if (esize == 4) *reinterpret_cast<uint32_t*>(dst + i * 4) = *reinterpret_cast<const uint32_t*>(src + so);
    else *reinterpret_cast<uint16_t*>(dst + i * 2) = *reinterpret_cast<const uint16_t*>(src + so);
  }
}

static unsigned gather_grid(long long n) {
  const long long b = (n + 255) / 256;
  const long long cap = 32LL * num_sms();
  return (unsigned)(b < 1 ? 1 : b < cap ? b : cap);
}

jamba_status gather_rows(const void* src, void* dst, const int* perm, int rows, int row_bytes, cudaStream_t s) {
  if (!src || !dst || !perm || rows <= 0 || row_bytes <= 0 || row_bytes % 2)
    return fail(JAMBA_ERR_INVALID_ARG, "gather_rows: bad argument");
  const bool a16 = aligned16(src) && aligned16(dst) && row_bytes % 16 == 0;
  const bool a4 = (reinterpret_cast<uintptr_t>(src) % 4 == 0) && (reinterpret_cast<uintptr_t>(dst) % 4 == 0) &&
                  row_bytes % 4 == 0;
  const int word = a16 ? 16 : a4 ? 4 : 2;
  gather_rows_kernel<<<gather_grid((long long)rows * (row_bytes / word)), 256, 0, s>>>(
      reinterpret_cast<const uint8_t*>(src), reinterpret_cast<uint8_t*>(dst), perm, rows, row_bytes, word,
      device_error_word());
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status gather_cols(const void* src, void* dst, const int* perm, int rows, int cols, int esize, cudaStream_t s) {
  if (!src || !dst || !perm || rows <= 0 || cols <= 0 || (esize != 2 && esize != 4))
    return fail(JAMBA_ERR_INVALID_ARG, "gather_cols: bad argument");
  gather_cols_kernel<<<gather_grid((long long)rows * cols), 256, 0, s>>>(
      reinterpret_cast<const uint8_t*>(src), reinterpret_cast<uint8_t*>(dst), perm, rows, cols, esize,
      device_error_word());
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

}  // namespace jb
