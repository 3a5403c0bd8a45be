// RMSNorms and split-K reductions.
//
// Jamba ("Jamba: A Hybrid Transformer-Mamba Language Model", section 2 and
// section 6.4 / figure 9) adds RMSNorm inside the Mamba layer; here it acts on
// the three parts of the x_proj output separately (dt_low over dt_rank
// columns, B and C over d_state columns each), fused with the sum of the
// split-K partials of x_proj.  The block RMSNorm in front of the mixer and the
// MoE is a plain row norm.
#include "common.cuh"
#include "host.hpp"

namespace jb {


// one 256-thread block per row
template <typename T>
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const T* __restrict__ x, const float* __restrict__ w, T* __restrict__ out, int cols, float eps) {
  griddep_wait();
  griddep_launch();
  const long long row = blockIdx.x;
  const T* xr = x + row * cols;
  T* orow = out + row * cols;
  float ss = 0.f;
  for (int c = threadIdx.x; c < cols; c += 256) {
    const float v = to_f(xr[c]);
    ss = fmaf(v, v, ss);
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < 8 ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv = rsqrtf(red[0] / (float)cols + eps);
  for (int c = threadIdx.x; c < cols; c += 256) orow[c] = from_f<T>(to_f(xr[c]) * inv * w[c]);
}

// x_proj output: sum the split-K partials [splits][T][R + 2N], then the three
// inner RMSNorms; dt_low goes out in the GEMM dtype, B | C in fp32.  One block
// per token, one thread per column.
template <typename TD>
__global__ void __launch_bounds__(512)
xproj_norm_kernel(const float* __restrict__ part, int splits, long long split_stride, int T, int R, int N,
                  const float* __restrict__ w_dt, const float* __restrict__ w_B, const float* __restrict__ w_C,
                  int inner_norm, float eps, TD* __restrict__ dtlow, float* __restrict__ bc) {
  griddep_wait();
  griddep_launch();
  const long long t = blockIdx.x;
  const int col = threadIdx.x, W = R + 2 * N;
  const int lane = col & 31, warp = col >> 5;
  __shared__ float red[16][3];
  __shared__ float inv[3];
  float v = 0.f;
  if (col < W) {
    // up to 32 partials in flight per round: the sum is one memory round trip
    // for the split counts used (at most 32 at decode sizes)
    const float* p = part + t * W + col;
    if (splits == 1) {
      v = *p;
    } else {
      for (int s0 = 0; s0 < splits; s0 += 32) {
        float a[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = s0 + i < splits ? p[(long long)(s0 + i) * split_stride] : 0.f;
#pragma unroll
        for (int w = 16; w; w >>= 1)
#pragma unroll
          for (int i = 0; i < w; ++i) a[i] += a[i + w];
        v += a[0];
      }
    }
  }
  const int seg = col < R ? 0 : (col < R + N ? 1 : 2);
  float sq[3] = {0.f, 0.f, 0.f};
  if (col < W) sq[seg] = v * v;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    sq[k] = warp_sum(sq[k]);
    if (lane == 0) red[warp][k] = sq[k];
  }
  __syncthreads();
  if (col < 3) {
    float acc = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) acc += red[w][col];
    const float n = col == 0 ? (float)R : (float)N;
    inv[col] = inner_norm ? rsqrtf(acc / n + eps) : 1.f;
  }
  __syncthreads();
  if (col >= W) return;
  if (seg == 0) {
    dtlow[t * R + col] = from_f<TD>(inner_norm ? v * inv[0] * w_dt[col] : v);
  } else if (seg == 1) {
    bc[t * 2 * N + (col - R)] = inner_norm ? v * inv[1] * w_B[col - R] : v;
  } else {
    bc[t * 2 * N + (col - R)] = inner_norm ? v * inv[2] * w_C[col - R - N] : v;
  }
}

// The same for one partial (the prefill's x_proj has no k-split at large T):
// a warp per token, lane l holding columns l, l + 32, ... (at most 16 of them),
// so there is no block barrier and a block covers eight tokens.
template <typename TD>
__global__ void __launch_bounds__(256)
xproj_norm_rows_kernel(const float* __restrict__ x, int T, int R, int N, const float* __restrict__ w_dt,
                       const float* __restrict__ w_B, const float* __restrict__ w_C, int inner_norm, float eps,
                       TD* __restrict__ dtlow, float* __restrict__ bc) {
  griddep_wait();
  griddep_launch();
  const long long t = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31, W = R + 2 * N;
  const float* xr = x + t * W;
  float v[16];
  float sq[3] = {0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int col = lane + 32 * i;
    v[i] = col < W ? xr[col] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int col = lane + 32 * i;
    const int seg = col < R ? 0 : (col < R + N ? 1 : 2);
    if (col < W) sq[seg] = fmaf(v[i], v[i], sq[seg]);
  }
  float inv[3] = {1.f, 1.f, 1.f};
  if (inner_norm) {
#pragma unroll
    for (int k = 0; k < 3; ++k) inv[k] = rsqrtf(warp_sum(sq[k]) / (float)(k == 0 ? R : N) + eps);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int col = lane + 32 * i;
    if (col >= W) break;
    if (col < R) {
      dtlow[t * R + col] = from_f<TD>(inner_norm ? v[i] * inv[0] * w_dt[col] : v[i]);
    } else if (col < R + N) {
      bc[t * 2 * N + (col - R)] = inner_norm ? v[i] * inv[1] * w_B[col - R] : v[i];
    } else {
      bc[t * 2 * N + (col - R)] = inner_norm ? v[i] * inv[2] * w_C[col - R - N] : v[i];
    }
  }
}

// out[r, c] = sum_s part[s][r][c] (+ residual[r, c])
template <typename T>
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ part, int splits, long long split_stride, long long n,
                     const T* __restrict__ residual, T* __restrict__ out) {
  griddep_wait();
  griddep_launch();
  const long long i = ((long long)blockIdx.x * 256 + threadIdx.x) * 4;
  if (i >= n) return;
  float4 acc = *reinterpret_cast<const float4*>(part + i);
  for (int s = 1; s < splits; ++s) {
    const float4 p = *reinterpret_cast<const float4*>(part + s * split_stride + i);
    acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
  }
  float r[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (residual) r[k] += to_f(residual[i + k]);
    out[i + k] = from_f<T>(r[k]);
  }
}

jamba_status rmsnorm(const void* x, const float* w, void* out, int rows, int cols, float eps, int dtype,
                     cudaStream_t s) {
  if (dtype == JAMBA_BF16)
    JB_CUDA(launch_pdl(rmsnorm_kernel<bf16>, dim3(rows), dim3(256), 0, s, reinterpret_cast<const bf16*>(x), w,
                       reinterpret_cast<bf16*>(out), cols, eps));
  else
    JB_CUDA(launch_pdl(rmsnorm_kernel<float>, dim3(rows), dim3(256), 0, s, reinterpret_cast<const float*>(x), w,
                       reinterpret_cast<float*>(out), cols, eps));
  return JAMBA_OK;
}

jamba_status xproj_norm(const float* part, int splits, long long split_stride, int T, int R, int N,
                        const float* w_dt, const float* w_B, const float* w_C, int inner_norm, float eps,
                        void* dtlow, float* bc, int dtype, cudaStream_t s) {
  if (R + 2 * N > 512) return fail(JAMBA_ERR_UNSUPPORTED, "x_proj width above 512");
  if (splits == 1 && T >= 1024) {
    const unsigned grid = (unsigned)((T + 7) / 8);
    if (dtype == JAMBA_BF16)
      JB_CUDA(launch_pdl(xproj_norm_rows_kernel<bf16>, dim3(grid), dim3(256), 0, s, part, T, R, N, w_dt, w_B, w_C,
                         inner_norm, eps, reinterpret_cast<bf16*>(dtlow), bc));
    else
      JB_CUDA(launch_pdl(xproj_norm_rows_kernel<float>, dim3(grid), dim3(256), 0, s, part, T, R, N, w_dt, w_B, w_C,
                         inner_norm, eps, reinterpret_cast<float*>(dtlow), bc));
    return JAMBA_OK;
  }
  const int threads = ((R + 2 * N + 31) / 32) * 32;
  if (dtype == JAMBA_BF16)
    JB_CUDA(launch_pdl(xproj_norm_kernel<bf16>, dim3(T), dim3(threads), 0, s, part, splits, split_stride, T, R, N, w_dt,
                       w_B, w_C, inner_norm, eps, reinterpret_cast<bf16*>(dtlow), bc));
  else
    JB_CUDA(launch_pdl(xproj_norm_kernel<float>, dim3(T), dim3(threads), 0, s, part, splits, split_stride, T, R, N,
                       w_dt, w_B, w_C, inner_norm, eps, reinterpret_cast<float*>(dtlow), bc));
  return JAMBA_OK;
}

jamba_status splitk_reduce(const float* part, int splits, long long split_stride, long long n,
                           const void* residual, void* out, int dtype, cudaStream_t s) {
  if (n % 4) return fail(JAMBA_ERR_INVALID_ARG, "split-K reduce: size must be a multiple of 4");
  const unsigned grid = (unsigned)((n / 4 + 255) / 256);
  if (dtype == JAMBA_BF16)
    JB_CUDA(launch_pdl(splitk_reduce_kernel<bf16>, dim3(grid), dim3(256), 0, s, part, splits, split_stride, n,
                       reinterpret_cast<const bf16*>(residual), reinterpret_cast<bf16*>(out)));
  else
    JB_CUDA(launch_pdl(splitk_reduce_kernel<float>, dim3(grid), dim3(256), 0, s, part, splits, split_stride, n,
                       reinterpret_cast<const float*>(residual), reinterpret_cast<float*>(out)));
  return JAMBA_OK;
}

}  // namespace jb
