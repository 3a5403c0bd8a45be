// MoE routing: router logits, softmax and top-K, the expert-sorted
// permutation, the row gather in front of the expert GEMMs and the weighted
// combine behind them.
//
// "Jamba: A Hybrid Transformer-Mamba Language Model" (summary page),
// section 2: MoE layers with n experts, the router picks the top K per token;
// section 3.1: n = 16, K = 2.  Expert choice is an integer decided by
// floating point, so the logits are accumulated in fp64 from products of the
// bf16 inputs (each product is exact in fp32): the choice then matches the
// exact-arithmetic one except for logit ties closer than about 1e-13.
#include "common.cuh"
#include "host.hpp"

namespace jb {

constexpr int ROUTER_EG = 16;  // experts per register group

// softmax over the E logits of token t and its top K (descending logit, ties
// to the lower index), probabilities not renormalised
__device__ __forceinline__ void route_token(const double* logit, int E, int K, int t, int* __restrict__ idx_out,
                                            float* __restrict__ w_out, int* __restrict__ counts) {
  double mx = logit[0];
  for (int e = 1; e < E; ++e) mx = logit[e] > mx ? logit[e] : mx;
  double den = 0.0;
  for (int e = 0; e < E; ++e) den += exp(logit[e] - mx);
  unsigned long long taken = 0ull;
  for (int k = 0; k < K; ++k) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken >> e & 1ull) continue;
      if (best < 0 || logit[e] > logit[best]) best = e;  // strict: ties keep the lower index
    }
    taken |= 1ull << best;
    idx_out[(long long)t * K + k] = best;
    w_out[(long long)t * K + k] = (float)(exp(logit[best] - mx) / den);
    atomicAdd(counts + best, 1);
  }
}

// one warp per token
__global__ void __launch_bounds__(256)
router_kernel(const bf16* __restrict__ x, const bf16* __restrict__ W, int T, int dm, int E, int K,
              int* __restrict__ idx_out, float* __restrict__ w_out, int* __restrict__ counts) {
  const int warps = gridDim.x * 8;
  const int lane = threadIdx.x & 31;
  double logit[64];
  for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += warps) {
    const bf16* xr = x + (long long)t * dm;
    for (int e0 = 0; e0 < E; e0 += ROUTER_EG) {
      double acc[ROUTER_EG];
#pragma unroll
      for (int e = 0; e < ROUTER_EG; ++e) acc[e] = 0.0;
      for (int k0 = lane * 8; k0 < dm; k0 += 256) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xr + k0);
        const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
        float xf[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(xh[i]);
          xf[2 * i] = f.x;
          xf[2 * i + 1] = f.y;
        }
#pragma unroll
        for (int e = 0; e < ROUTER_EG; ++e) {
          if (e0 + e >= E) break;
          const uint4 wv = __ldg(reinterpret_cast<const uint4*>(W + (long long)(e0 + e) * dm + k0));
          const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(wh[i]);
            acc[e] += (double)(xf[2 * i] * f.x);      // exact product of two bf16 values
            acc[e] += (double)(xf[2 * i + 1] * f.y);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < ROUTER_EG; ++e) {
        double v = acc[e];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (e0 + e < E) logit[e0 + e] = v;
      }
    }
    if (lane == 0) route_token(logit, E, K, t, idx_out, w_out, counts);
  }
}

// Few tokens: one block per token and one warp per expert (experts beyond the
// warps loop), each lane summing its 1/32 of d_model in four fp64 partials;
// then one warp takes the softmax and the top K with one expert per lane
// (two when E > 32), so the decision costs a few shuffles instead of a
// serial pass over the logits.
__global__ void __launch_bounds__(512)
router_token_kernel(const bf16* __restrict__ x, const bf16* __restrict__ W, int dm, int E, int K,
                    int* __restrict__ idx_out, float* __restrict__ w_out, int* __restrict__ counts) {
  __shared__ double logit[64];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const bf16* xr = x + (long long)t * dm;
  for (int e = warp; e < E; e += nw) {
    const bf16* wr = W + (long long)e * dm;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
    for (int k0 = lane * 8; k0 < dm; k0 += 256) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xr + k0);
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wr + k0));
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
      const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(xh[i]), b = __bfloat1622float2(wh[i]);
        acc[i] += (double)(a.x * b.x);      // exact product of two bf16 values
        acc[i] += (double)(a.y * b.y);
      }
    }
    double v = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) logit[e] = v;
  }
  __syncthreads();
  if (warp != 0) return;
  const double NEG = -1.0 / 0.0;
  const bool v0 = lane < E, v1 = lane + 32 < E;
  const double l0 = v0 ? logit[lane] : NEG, l1 = v1 ? logit[lane + 32] : NEG;
  double mx = l0 > l1 ? l0 : l1;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const double m2 = __shfl_xor_sync(0xffffffffu, mx, o);
    mx = m2 > mx ? m2 : mx;
  }
  double den = (v0 ? exp(l0 - mx) : 0.0) + (v1 ? exp(l1 - mx) : 0.0);
#pragma unroll
  for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  bool took0 = false, took1 = false;
  for (int k = 0; k < K; ++k) {
    // this lane's best untaken expert, then the warp's (ties: the lower index)
    double bv = NEG;
    int bi = 1 << 30;
    if (v0 && !took0) { bv = l0; bi = lane; }
    if (v1 && !took1 && (bi == (1 << 30) || l1 > bv)) { bv = l1; bi = lane + 32; }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    took0 = took0 || bi == lane;
    took1 = took1 || bi == lane + 32;
    if (lane == 0) {
      idx_out[(long long)t * K + k] = bi;
      w_out[(long long)t * K + k] = (float)(exp(bv - mx) / den);
      atomicAdd(counts + bi, 1);
    }
  }
}

// One block per expert: stable positions of that expert's (token, slot)
// pairs in flat order, i.e. routed rows sorted by (expert, token, slot).
__global__ void __launch_bounds__(1024)
permute_kernel(const int* __restrict__ idx, int TK, int E, const int* __restrict__ counts, int* __restrict__ offsets,
               int* __restrict__ perm, int* __restrict__ inv) {
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int s_warp[32];
  __shared__ int s_base;
  if (tid == 0) {
    int o = 0;
    for (int i = 0; i < e; ++i) o += counts[i];
    s_base = o;
    if (e == 0) {
      int acc = 0;
      offsets[0] = 0;
      for (int i = 0; i < E; ++i) {
        acc += counts[i];
        offsets[i + 1] = acc;
      }
    }
  }
  __syncthreads();
  int run = s_base;
  for (int f0 = 0; f0 < TK; f0 += 1024) {
    const int f = f0 + tid;
    const bool hit = f < TK && idx[f] == e;
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
      const int v = s_warp[lane];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      s_warp[lane] = incl - v;  // exclusive prefix per warp
      if (lane == 31) s_base = incl;  // block total (read after the next barrier)
    }
    __syncthreads();
    if (hit) {
      const int pos = run + s_warp[warp] + __popc(bal & ((1u << lane) - 1u));
      perm[pos] = f;
      inv[f] = pos;
    }
    run += s_base;
    __syncthreads();
  }
}

// routed row p <- token perm[p] / K
__global__ void __launch_bounds__(256)
gather_rows_kernel(const bf16* __restrict__ x, const int* __restrict__ perm, int K, int dm, bf16* __restrict__ out,
                   int* err) {
  const long long p = blockIdx.x;
  const int pp = perm[p];
  if (!checked(pp >= 0 && pp < (int)gridDim.x, err)) return;
  const int t = pp / K;
  const uint4* src = reinterpret_cast<const uint4*>(x + (long long)t * dm);
  uint4* dst = reinterpret_cast<uint4*>(out + p * dm);
  for (int i = threadIdx.x; i < dm / 8; i += 256) dst[i] = src[i];
}

// out[t] = residual[t] + sum_k w[t, k] * Y[inv[t K + k]], slot 0 first, fp32
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ Y, int splits, long long split_stride, const int* __restrict__ inv,
               const float* __restrict__ w, int K, int dm, const bf16* __restrict__ residual, bf16* __restrict__ out,
               int* err) {
  const long long t = blockIdx.x;
  const int rows = (int)gridDim.x * K;
  for (int c = threadIdx.x * 4; c < dm; c += 1024) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) {
      const float wk = w[t * K + k];
      const int j = inv[t * K + k];
      if (!checked(j >= 0 && j < rows, err)) continue;
      const float* yr = Y + (long long)j * dm + c;
      float4 y = *reinterpret_cast<const float4*>(yr);
      for (int sp = 1; sp < splits; ++sp) {   // k-split partial sums of the down GEMM, in split order
        const float4 y2 = *reinterpret_cast<const float4*>(yr + sp * split_stride);
        y.x += y2.x; y.y += y2.y; y.z += y2.z; y.w += y2.w;
      }
      acc[0] = fmaf(wk, y.x, acc[0]);
      acc[1] = fmaf(wk, y.y, acc[1]);
      acc[2] = fmaf(wk, y.z, acc[2]);
      acc[3] = fmaf(wk, y.w, acc[3]);
    }
    __nv_bfloat162 o[2];
    float r[4] = {0.f, 0.f, 0.f, 0.f};
    if (residual) {
      const uint2 rv = *reinterpret_cast<const uint2*>(residual + t * dm + c);
      const __nv_bfloat162* rh = reinterpret_cast<const __nv_bfloat162*>(&rv);
      const float2 a = __bfloat1622float2(rh[0]), b = __bfloat1622float2(rh[1]);
      r[0] = a.x; r[1] = a.y; r[2] = b.x; r[3] = b.y;
    }
    o[0] = __floats2bfloat162_rn(acc[0] + r[0], acc[1] + r[1]);
    o[1] = __floats2bfloat162_rn(acc[2] + r[2], acc[3] + r[3]);
    *reinterpret_cast<uint2*>(out + t * dm + c) = *reinterpret_cast<uint2*>(o);
  }
}

// ExpertsInt8 weight format: one warp per row, absolute maximum, then the
// codes.  Both passes read the row; the second finds it in L1/L2.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float* f);
template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float* f) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(256)
quantize_rows_kernel(const T* __restrict__ w, long long rows, int cols, int8_t* __restrict__ q,
                     float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * 8;
  for (long long r = blockIdx.x * 8ll + (threadIdx.x >> 5); r < rows; r += warps) {
    const T* wr = w + r * cols;
    float amax = 0.f;
    for (int c = lane * 8; c < cols; c += 256) {
      float f[8];
      load8(wr + c, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 127.0f);
    if (lane == 0) scale[r] = s;
    int8_t* qr = q + r * cols;
    for (int c = lane * 8; c < cols; c += 256) {
      float f[8];
      load8(wr + c, f);
      uint32_t pk[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // round half to even of the correctly rounded quotient; |w| <= amax keeps it within 127
        const int v = s > 0.f ? max(-127, min(127, __float2int_rn(__fdiv_rn(f[i], s)))) : 0;
        pk[i >> 2] |= (uint32_t)(v & 0xff) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(qr + c) = make_uint2(pk[0], pk[1]);
    }
  }
}

jamba_status quantize_int8_rows(const void* w, int dtype, long long rows, int cols, int8_t* q, float* scale,
                                cudaStream_t s) {
  long long blocks = (rows + 7) / 8;
  const long long cap = 16ll * num_sms();
  if (blocks > cap) blocks = cap;
  if (dtype == JAMBA_BF16)
    quantize_rows_kernel<bf16><<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const bf16*>(w), rows, cols, q, scale);
  else
    quantize_rows_kernel<float><<<(int)blocks, 256, 0, s>>>(reinterpret_cast<const float*>(w), rows, cols, q, scale);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status moe_route(const void* x, const void* W, int T, int dm, int E, int K, int* idx, float* w, int* counts,
                       int* offsets, int* perm, int* inv, cudaStream_t s) {
  JB_CUDA(cudaMemsetAsync(counts, 0, sizeof(int) * E, s));
  if (T <= 4096) {
    router_token_kernel<<<T, 32 * (E < 16 ? E : 16), 0, s>>>(reinterpret_cast<const bf16*>(x),
                                                             reinterpret_cast<const bf16*>(W), dm, E, K, idx, w, counts);
  } else {
    int blocks = (T + 7) / 8;
    const int cap = 8 * num_sms();
    if (blocks > cap) blocks = cap;
    router_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const bf16*>(x), reinterpret_cast<const bf16*>(W), T, dm,
                                         E, K, idx, w, counts);
  }
  JB_CUDA(cudaGetLastError());
  permute_kernel<<<E, 1024, 0, s>>>(idx, T * K, E, counts, offsets, perm, inv);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

// offsets[0] = 0, offsets[g + 1] = offsets[g] + counts[g] (one thread; n is small)
__global__ void group_offsets_kernel(const int* __restrict__ counts, int n, int* __restrict__ offsets) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    offsets[0] = 0;
    for (int g = 0; g < n; ++g) {
      acc += counts[g];
      offsets[g + 1] = acc;
    }
  }
}

jamba_status group_offsets(const int* counts, int n, int* offsets, cudaStream_t s) {
  group_offsets_kernel<<<1, 32, 0, s>>>(counts, n, offsets);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status moe_gather(const void* x, const int* perm, int rows, int K, int dm, void* out, cudaStream_t s) {
  gather_rows_kernel<<<rows, 256, 0, s>>>(reinterpret_cast<const bf16*>(x), perm, K, dm, reinterpret_cast<bf16*>(out),
                                          device_error_word());
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status moe_combine(const float* Y, int splits, long long split_stride, const int* inv, const float* w, int T,
                         int K, int dm, const void* residual, void* out, cudaStream_t s) {
  combine_kernel<<<T, 256, 0, s>>>(Y, splits, split_stride, inv, w, K, dm, reinterpret_cast<const bf16*>(residual),
                                   reinterpret_cast<bf16*>(out), device_error_word());
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

}  // namespace jb
