// tcgen05 / TMEM GEMM for sm_100a: D[m, n] = sum_k A[m, k] * B[n, k], bf16
// inputs, fp32 accumulation in tensor memory.
//
// One persistent CTA per SM, 10 warps:
//   warp 0     TMA producer: 128 x 64 A tile and BN x 64 B tile per k-step
//              (128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 1     allocates TMEM and issues tcgen05.mma (one thread), M = 128,
//              N = BN, K = 16 per instruction, into one of two TMEM
//              accumulators so the epilogue of tile i overlaps tile i + 1;
//   warps 2-9  epilogue: two warps per 32-lane TMEM quarter, splitting the
//              32-column chunks between them; tcgen05.ld, fused elementwise
//              op, stores to global memory.
// The epilogue kind is a template parameter, so each instantiation carries
// only its own epilogue code.  Used for in_proj (+ causal conv + SiLU of the
// x columns), x_proj, dt_proj (+bias+softplus), out_proj (+residual), the
// decode projections (swap-AB: weights as A so the 64-row token batch is the
// N side, stored transposed; in_proj + conv step) and the grouped MoE expert
// GEMMs (SwiGLU epilogue).  Every wait is bounded (see common.cuh).
#pragma once
#include "common.cuh"

namespace jb {

enum EpiKind : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_SOFTPLUS = 2, EPI_SWIGLU = 3, EPI_CONV = 4, EPI_CONVP = 5 };

constexpr int GEMM_THREADS = 320;
constexpr int GEMM_EPI_WARPS = 8;

struct GemmParams {
  int M, N, K;           // N counts output columns (SwiGLU: d_ff)
  int k_tiles;           // ceil(K / 64)
  int splits, k_tiles_per_split;
  int m_tiles, n_tiles;  // dense mode
  int band_m;            // dense mode: m-tiles per raster band (their A rows stay in L2 while B streams)
  int grouped;           // A rows split by offsets[], B is [groups, rows, K]
  const int* offsets;
  int num_groups;
  int group_mod;         // > 0: group g uses weight set g % group_mod (groups of rows from several ranks)
  void* out;
  long long ldo, split_stride;
  const void* residual;  // bf16, same layout as out (non-transposed only)
  long long ldr;
  const float* bias;     // indexed by n (or by m when transposed)
  const float* scale_b;  // INT8 weights: per-row scales [groups, N] (SwiGLU: of the gate rows)
  const float* scale_b2; // INT8 weights, SwiGLU: scales of the up rows
  // EPI_CONV (decode in_proj, swap-AB): output rows m < conv_c are the conv's
  // input x: the causal conv over [cache, x] + SiLU goes to xc_out [N, conv_c]
  // and the cache [N, conv_c, 3] shifts in place; rows >= conv_c are stored
  // as in EPI_BF16
  const bf16* conv_w;    // [conv_c, 4]
  const bf16* conv_b;    // [conv_c]
  float* conv_state;
  bf16* xc_out;
  int conv_c;
  // EPI_CONVP (prefill in_proj, rows = tokens b * conv_L + t, N = 2 conv_c):
  // columns n < conv_c are x, the causal conv + SiLU of which goes to xc_out
  // [M, conv_c]; columns >= conv_c (z) are stored into out as in EPI_BF16.
  // conv_in [M / conv_L, conv_c, 3] (or null: zeros) holds the three inputs
  // before each sequence, conv_out receives its last three; both indexed by
  // the cache row conv_perm[c] of channel c (identity when null)
  const float* conv_in;
  float* conv_out;
  const int* conv_perm;
  int conv_L;
  int* err;
};

struct TileInfo {
  int m0, m_end, n0, kt0, kt1, group, split;
};

// Rows [o0, o1) of group g.  The offsets are device data (a caller's counts in
// the expert-parallel path): they are clamped into [0, M] with o1 >= o0, so a
// bad table gives empty or clipped groups, never rows past A or the output,
// and every role of a kernel decodes the same tiles from it.
__device__ __forceinline__ void group_rows(const GemmParams& p, int g, int& o0, int& o1) {
  const int a = __ldg(p.offsets + g), b = __ldg(p.offsets + g + 1);
  o0 = min(max(a, 0), p.M);
  o1 = min(max(b, o0), p.M);
  checked(o0 == a && o1 == b, p.err);
}

__device__ __forceinline__ int total_tiles(const GemmParams& p) {
  if (!p.grouped) return p.m_tiles * p.n_tiles * p.splits;
  int tot = 0;
  for (int g = 0; g < p.num_groups; ++g) {
    int o0, o1;
    group_rows(p, g, o0, o1);
    tot += ((o1 - o0 + 127) >> 7) * p.n_tiles;
  }
  return tot;
}

template <int BN_OUT>
__device__ __forceinline__ void decode_tile(const GemmParams& p, int t, TileInfo& ti) {
  if (!p.grouped) {
    const int per_split = p.m_tiles * p.n_tiles;
    const int s = t / per_split;
    const int r = t - s * per_split;
    // rasterise in bands of band_m m-tiles, m fastest within a band: the
    // band's A rows (sized on the host to stay in L2) are read from DRAM
    // once, the CTAs of a wave share each B tile, and B is read once per band
    const int span = p.band_m * p.n_tiles;
    const int gi = r / span;
    const int first_m = gi * p.band_m;
    const int gsize = min(p.m_tiles - first_m, p.band_m);
    const int rr = r - gi * span;
    const int mb = first_m + rr % gsize;
    const int nb = rr / gsize;
    ti.m0 = mb * 128;
    ti.m_end = p.M;
    ti.n0 = nb * BN_OUT;
    ti.kt0 = s * p.k_tiles_per_split;
    ti.kt1 = min(p.k_tiles, ti.kt0 + p.k_tiles_per_split);
    ti.group = 0;
    ti.split = s;
  } else {
    for (int g = 0; g < p.num_groups; ++g) {
      int o0, o1;
      group_rows(p, g, o0, o1);
      const int mt = (o1 - o0 + 127) >> 7;
      const int tg = mt * p.n_tiles;
      if (t < tg) {
        const int mb = t % mt, nb = t / mt;  // m fastest: neighbours share the weight tile
        ti.m0 = o0 + mb * 128;
        ti.m_end = o1;
        ti.n0 = nb * BN_OUT;
        ti.kt0 = 0;
        ti.kt1 = p.k_tiles;
        ti.group = p.group_mod > 0 ? g % p.group_mod : g;
        ti.split = 0;
        return;
      }
      t -= tg;
    }
    ti.m0 = ti.m_end = ti.n0 = ti.kt0 = ti.kt1 = ti.group = ti.split = 0;
  }
}

__device__ __forceinline__ void store_bf16x8(bf16* dst, const float* v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(dst) = u;
}

__device__ __forceinline__ float log1p_small(float e) {
  // log(1 + e) for 0 <= e < 1/8: Taylor series through e^7 (relative error < 1e-7)
  return e * (1.0f - e * (0.5f - e * (0.33333334f - e * (0.25f - e * (0.2f - e * (0.16666667f - e * 0.14285715f))))));
}

// log(1 + e) for two values at once (0 <= e <= 1/8): the same series in Horner
// form with packed fp32x2 arithmetic.
__device__ __forceinline__ float2 log1p_small2(float2 e) {
  float2 p = ffma2(e, make_float2(0.14285715f, 0.14285715f), make_float2(-0.16666667f, -0.16666667f));
  p = ffma2(p, e, make_float2(0.2f, 0.2f));
  p = ffma2(p, e, make_float2(-0.25f, -0.25f));
  p = ffma2(p, e, make_float2(0.33333334f, 0.33333334f));
  p = ffma2(p, e, make_float2(-0.5f, -0.5f));
  p = ffma2(p, e, make_float2(1.0f, 1.0f));
  return fmul2(p, e);
}

// softplus of 32 values in place, each given as x = v * log2(e) (v the
// pre-activation): one ex2 each, then the series when every e^v of the warp
// is at most 1/8 (x <= -3: the common case for dt), otherwise one lg2 as well.
__device__ __forceinline__ void softplus32_log2(float* w) {
  float e[32];
  float mx = w[0];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    e[i] = ex2(w[i]);
    mx = fmaxf(mx, w[i]);
  }
  if (__all_sync(0xffffffffu, mx <= -3.0f)) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float2 r = log1p_small2(make_float2(e[i], e[i + 1]));
      w[i] = r.x; w[i + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float l;
      asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.0f + e[i]));
      const float v = 0.6931471805599453f * w[i];
      const float r = e[i] <= 0.125f ? log1p_small(e[i]) : 0.6931471805599453f * l;
      w[i] = v > 15.0f ? v : r;
    }
  }
}

// v[c] *= scale[n + c] for the 32 columns n..n+31 (columns >= N untouched)
__device__ __forceinline__ void scale32(float* v, const float* __restrict__ scale, int n, int N) {
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    if (n + c + 4 <= N) {
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(scale + n + c));
      v[c] *= s4.x; v[c + 1] *= s4.y; v[c + 2] *= s4.z; v[c + 3] *= s4.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (n + c + i < N) v[c + i] *= __ldg(scale + n + c + i);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

template <int EPI, bool TRANS, int NC>
__device__ __forceinline__ void epi_chunk(const GemmParams& p, const TileInfo& ti, int m, int n, const float* v);

// EPI_CONVP, one 32-column chunk of row m (token t of sequence b).  The x
// value is the bf16 activation, as an unfused conv would read it back.  A
// warp holds 32 consecutive rows (a slab), so the three inputs before row m
// are the lanes below it; where the window reaches above the slab inside the
// same sequence (lanes 0-2 with t > lane) the row is deferred: its raw x, and
// the raw x of lanes 29-31 of every slab, is stored into the x columns of out
// for conv_fixup_kernel.  Taps before the sequence start come from conv_in.
// The multiply-add order is the one of the standalone conv kernels.
__device__ __forceinline__ void epi_conv_prefill(const GemmParams& p, const TileInfo& ti, int m, int n,
                                                 const float* v) {
  if (n >= p.conv_c) {   // z columns (the chunk is all x or all z: conv_c % 32 == 0)
    epi_chunk<EPI_BF16, false, 32>(p, ti, m, n, v);
    return;
  }
  const int lane = threadIdx.x & 31;
  uint32_t r0[16], r1[16], r2[16], r3[16];   // bf16 pairs of rows m, m-1, m-2, m-3
#pragma unroll
  for (int i = 0; i < 16; ++i) r0[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    r1[i] = __shfl_up_sync(0xffffffffu, r0[i], 1);
    r2[i] = __shfl_up_sync(0xffffffffu, r0[i], 2);
    r3[i] = __shfl_up_sync(0xffffffffu, r0[i], 3);
  }
  if (m >= ti.m_end) return;
  const int L = p.conv_L, C = p.conv_c;
  const int b = m / L, t = m - b * L;
  const bool deferred = lane < 3 && t > lane;
  if (deferred || lane >= 29) {
    uint4* xo = reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(p.out) + (long long)m * p.ldo + n);
#pragma unroll
    for (int k = 0; k < 4; ++k) xo[k] = make_uint4(r0[4 * k], r0[4 * k + 1], r0[4 * k + 2], r0[4 * k + 3]);
  }
  if (p.conv_out && t >= L - 3) {   // the cache after this sequence: its last three inputs
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 x = unpack_bf16x2(r0[i]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = n + 2 * i + e;
        const int cn = p.conv_perm ? __ldg(p.conv_perm + c) : c;
        if (checked(cn >= 0 && cn < C, p.err)) p.conv_out[((long long)b * C + cn) * 3 + (t - (L - 3))] = e ? x.y : x.x;
      }
    }
  }
  if (deferred) return;
  uint4* xc = reinterpret_cast<uint4*>(p.xc_out + (long long)m * C + n);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * k + q;
      const uint4 wq = __ldg(reinterpret_cast<const uint4*>(p.conv_w + (long long)(n + 2 * i) * 4));
      const float2 w01 = unpack_bf16x2(wq.x), w23 = unpack_bf16x2(wq.y);   // channel n + 2i
      const float2 u01 = unpack_bf16x2(wq.z), u23 = unpack_bf16x2(wq.w);   // channel n + 2i + 1
      float2 acc = unpack_bf16x2(__ldg(reinterpret_cast<const uint32_t*>(p.conv_b + n + 2 * i)));
      float2 x3 = unpack_bf16x2(r3[i]), x2 = unpack_bf16x2(r2[i]), x1 = unpack_bf16x2(r1[i]);
      if (t < 3) {   // taps before the sequence start: the cache (exact fp32 values)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = n + 2 * i + e;
          const int cn = p.conv_perm ? __ldg(p.conv_perm + c) : c;
          const float* ci = p.conv_in && checked(cn >= 0 && cn < C, p.err) ? p.conv_in + ((long long)b * C + cn) * 3
                                                                           : nullptr;
          const float s3 = ci ? ci[t] : 0.f, s2 = ci && t < 2 ? ci[t + 1] : 0.f, s1 = ci && t < 1 ? ci[t + 2] : 0.f;
          if (e) { x3.y = s3; if (t < 2) x2.y = s2; if (t < 1) x1.y = s1; }
          else   { x3.x = s3; if (t < 2) x2.x = s2; if (t < 1) x1.x = s1; }
        }
      }
      acc = ffma2(make_float2(w01.x, u01.x), x3, acc);
      acc = ffma2(make_float2(w01.y, u01.y), x2, acc);
      acc = ffma2(make_float2(w23.x, u23.x), x1, acc);
      acc = ffma2(make_float2(w23.y, u23.y), unpack_bf16x2(r0[i]), acc);
      o[q] = pack_bf16x2(silu(acc.x), silu(acc.y));
    }
    xc[k] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Epilogue of one 32-column chunk held by this thread (row m, columns n..n+NC-1).
template <int EPI, bool TRANS, int NC>
__device__ __forceinline__ void epi_chunk(const GemmParams& p, const TileInfo& ti, int m, int n, const float* v) {
  if constexpr (EPI == EPI_CONVP) {
    static_assert(!TRANS && NC == 32, "the prefill conv epilogue works on whole 32-column chunks");
    epi_conv_prefill(p, ti, m, n, v);
    return;
  }
  if (m >= ti.m_end) return;
  if constexpr (!TRANS) {
    if constexpr (EPI == EPI_BF16) {
      bf16* o = reinterpret_cast<bf16*>(p.out) + (long long)m * p.ldo;
      const bf16* r = p.residual ? reinterpret_cast<const bf16*>(p.residual) + (long long)m * p.ldr : nullptr;
#pragma unroll
      for (int c = 0; c < NC; c += 8) {
        const int nn = n + c;
        float w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = v[c + i];
        if (nn + 8 <= p.N) {
          if (r) {
            const uint4 rv = *reinterpret_cast<const uint4*>(r + nn);
            const bf16* rb = reinterpret_cast<const bf16*>(&rv);
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] += __bfloat162float(rb[i]);
          }
          store_bf16x8(o + nn, w);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (nn + i < p.N) o[nn + i] = __float2bfloat16_rn(w[i] + (r ? __bfloat162float(r[nn + i]) : 0.f));
        }
      }
    } else {  // EPI_F32 / EPI_SOFTPLUS
      float* o = reinterpret_cast<float*>(p.out) + (long long)ti.split * p.split_stride + (long long)m * p.ldo;
#pragma unroll
      for (int c = 0; c < NC; c += 4) {
        const int nn = n + c;
        float w[4];
        if (EPI == EPI_SOFTPLUS && nn + 4 <= p.N) {
          const float4 b4 = __ldg(reinterpret_cast<const float4*>(p.bias + nn));
          w[0] = softplus_fast(v[c] + b4.x);
          w[1] = softplus_fast(v[c + 1] + b4.y);
          w[2] = softplus_fast(v[c + 2] + b4.z);
          w[3] = softplus_fast(v[c + 3] + b4.w);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            w[i] = v[c + i];
            if (EPI == EPI_SOFTPLUS && nn + i < p.N) w[i] = softplus_fast(w[i] + __ldg(p.bias + nn + i));
          }
        }
        if (nn + 4 <= p.N) {
          *reinterpret_cast<float4*>(o + nn) = make_float4(w[0], w[1], w[2], w[3]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (nn + i < p.N) o[nn + i] = w[i];
        }
      }
    }
  } else {
    // swap-AB: row m is an output feature, column n a token; lanes hold consecutive m
    if constexpr (EPI == EPI_CONV) {
      if (m < p.conv_c) {
        // decode conv step of channel m for tokens n..n+NC-1: window [cache (oldest first), x]
        const uint2 wr = *reinterpret_cast<const uint2*>(p.conv_w + (long long)m * 4);
        const bf16* wb = reinterpret_cast<const bf16*>(&wr);
        const float w0 = __bfloat162float(wb[0]), w1 = __bfloat162float(wb[1]);
        const float w2 = __bfloat162float(wb[2]), w3 = __bfloat162float(wb[3]);
        const float bias = __bfloat162float(p.conv_b[m]);
        // eight tokens at a time: their cache loads are all issued before any
        // of the stores (which the compiler may not move the next loads past)
#pragma unroll
        for (int c0 = 0; c0 < NC; c0 += 8) {
          float sv[8][3];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (n + c0 + c < p.N) {
              const float* st = p.conv_state + ((long long)(n + c0 + c) * p.conv_c + m) * 3;
              sv[c][0] = st[0];
              sv[c][1] = st[1];
              sv[c][2] = st[2];
            }
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (n + c0 + c < p.N) {
              const long long bc = (long long)(n + c0 + c) * p.conv_c + m;
              float* st = p.conv_state + bc * 3;
              const float xv = __bfloat162float(__float2bfloat16_rn(v[c0 + c]));   // x as the bf16 activation
              float acc = bias;
              acc = fmaf(w0, sv[c][0], acc);
              acc = fmaf(w1, sv[c][1], acc);
              acc = fmaf(w2, sv[c][2], acc);
              acc = fmaf(w3, xv, acc);
              p.xc_out[bc] = __float2bfloat16_rn(silu(acc));
              st[0] = sv[c][1];
              st[1] = sv[c][2];
              st[2] = xv;
            }
          }
        }
      } else {
        bf16* o = reinterpret_cast<bf16*>(p.out);
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (n + c < p.N) o[(long long)(n + c) * p.ldo + m] = __float2bfloat16_rn(v[c]);
      }
    } else if constexpr (EPI == EPI_BF16) {
      bf16* o = reinterpret_cast<bf16*>(p.out);
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (n + c < p.N) o[(long long)(n + c) * p.ldo + m] = __float2bfloat16_rn(v[c]);
    } else {
      float* o = reinterpret_cast<float*>(p.out) + (long long)ti.split * p.split_stride;
      const float b = (EPI == EPI_SOFTPLUS) ? __ldg(p.bias + m) : 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (n + c < p.N) {
          float w = v[c];
          if constexpr (EPI == EPI_SOFTPLUS) w = softplus_fast(w + b);
          o[(long long)(n + c) * p.ldo + m] = w;
        }
      }
    }
  }
}

// EW epilogue warps, EW / 4 per TMEM lane quarter; NSTG staging boxes per
// epilogue warp in the staged (TMA-store) epilogue.
template <int BN, int STAGES, bool STAGED = false, int EW = GEMM_EPI_WARPS, int NSTG = 2>
struct GemmSmem {
  static constexpr uint32_t A_BYTES = 128 * 128;
  static constexpr uint32_t B_BYTES = BN * 128;
  // STAGED: per epilogue warp NSTG 32 x 32 fp32 boxes for TMA stores (1024-aligned)
  static constexpr uint32_t STG_OFF = STAGES * (A_BYTES + B_BYTES);
  static constexpr uint32_t STG_BYTES = STAGED ? EW * NSTG * 4096 : 0;
  // STAGED: per epilogue warp the bias of its 32-column chunks of the tile
  static constexpr int SB_CHUNKS = (BN / 32 + EW / 4 - 1) / (EW / 4);
  static constexpr uint32_t SB_OFF = STG_OFF + STG_BYTES;
  static constexpr uint32_t SB_BYTES = STAGED ? EW * SB_CHUNKS * 128 : 0;
  static constexpr uint32_t BAR_OFF = SB_OFF + SB_BYTES;
  // barrier slots: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], drain, tmem holder
  static_assert(8 * (2 * STAGES + 6) <= 256, "barrier slots");
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;  // + barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                        : (2 * BN <= 256) ? 256 : 512;
};

// Staging boxes per epilogue warp: two with the default eight epilogue warps,
// one with more (shared memory is the limit).
template <int EW> constexpr int gemm_nstg() { return EW > GEMM_EPI_WARPS ? 1 : 2; }

template <int BN, int STAGES, int EPI, bool TRANS, int EW = GEMM_EPI_WARPS>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmC,
                    const GemmParams p) {
  // fp32 softplus outputs (dt) leave through shared memory and TMA stores
  constexpr bool STAGED = EPI == EPI_SOFTPLUS && !TRANS;
  constexpr int NSTG = gemm_nstg<EW>();
  constexpr int WPQ = EW / 4;                 // epilogue warps per TMEM lane quarter
  static_assert(EW % 4 == 0 && EW >= 4, "whole lane quarters");
  using S = GemmSmem<BN, STAGES, STAGED, EW, NSTG>;
  static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "UMMA N for M = 128");
  constexpr int BN_OUT = EPI == EPI_SWIGLU ? BN / 2 : BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  constexpr uint32_t STAGE_TX = S::A_BYTES + S::B_BYTES;   // bytes the TMA loads land per stage

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, EW);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    if (EPI == EPI_SWIGLU) tma_prefetch(&tmB2);
    if (STAGED) tma_prefetch(&tmC);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  griddep_launch();   // the next kernel may begin its own prologue

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // Swap-AB (decode): A is a weight matrix, independent of the previous
      // kernel, so the first ring stages of it stream in before the wait.
      int pre = 0;
      if constexpr (TRANS) {
        if ((int)blockIdx.x < p.m_tiles * p.n_tiles * p.splits) {
          TileInfo t0;
          decode_tile<BN_OUT>(p, blockIdx.x, t0);
          for (int kt = t0.kt0; kt < t0.kt1 && pre < STAGES; ++kt, ++pre) {
            const uint32_t fb = full0 + 8 * pre;
            mbar_arrive_tx(fb, STAGE_TX);
            tma_load_2d(smem_u32(sA + pre * S::A_BYTES), &tmA, fb, kt * 64, t0.m0);
          }
        }
      }
      griddep_wait();
      const int ntiles = total_tiles(p);
      int issued = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        TileInfo ti;
        decode_tile<BN_OUT>(p, t, ti);
        for (int kt = ti.kt0; kt < ti.kt1; ++kt, ++issued) {
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t a_dst = smem_u32(sA + stage * S::A_BYTES);
          const uint32_t b_dst = smem_u32(sB + stage * S::B_BYTES);
          if (issued >= pre) {
            if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, p.err)) { ok = false; break; }
            mbar_arrive_tx(fb, STAGE_TX);
            tma_load_2d(a_dst, &tmA, fb, kt * 64, ti.m0);
          }
          if (!p.grouped) {
            tma_load_2d(b_dst, &tmB, fb, kt * 64, ti.n0);
          } else if (EPI != EPI_SWIGLU) {
            tma_load_3d(b_dst, &tmB, fb, kt * 64, ti.n0, ti.group);
          } else {
            tma_load_3d(b_dst, &tmB, fb, kt * 64, ti.n0, ti.group);
            tma_load_3d(b_dst + (BN / 2) * 128, &tmB2, fb, kt * 64, ti.n0, ti.group);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    griddep_wait();
    const int ntiles = total_tiles(p);
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, BN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        TileInfo ti;
        decode_tile<BN_OUT>(p, t, ti);
        const int acc = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(tempty0 + 8 * acc, (use & 1) ^ 1, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tbase + acc * BN;
        for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
          if (!mbar_wait(full0 + 8 * stage, phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(sA + stage * S::A_BYTES));
          const uint64_t bd = sw128_desc(smem_u32(sB + stage * S::B_BYTES));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, IDESC, (kt > ti.kt0 || kk > 0) ? 1u : 0u);
          umma_commit(empty0 + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * acc);
      }
      // drain: no MMA may still be writing TMEM when the CTA frees it
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    griddep_wait();
    const int ntiles = total_tiles(p);
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;       // which of the WPQ warps of this quarter
    int it = 0;
    int stg_count = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      TileInfo ti;
      decode_tile<BN_OUT>(p, t, ti);
      const int acc = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      // staged epilogue: the bias of this warp's chunks (lane = column within
      // a chunk) is fetched while the accumulator is still being computed
      float bl[S::SB_CHUNKS];
      if constexpr (STAGED) {
#pragma unroll
        for (int jj = 0; jj < S::SB_CHUNKS; ++jj) {
          const int col = ti.n0 + (half + WPQ * jj) * 32 + lane;
          // scaled by log2(e): the epilogue forms (acc + bias) * log2(e) in one FMA
          bl[jj] = (half + WPQ * jj < BN / 32 && col < p.N) ? __ldg(p.bias + col) * 1.4426950408889634f : 0.f;
        }
      }
      if (!mbar_wait_warp(tfull0 + 8 * acc, use & 1, p.err)) break;
      tc_fence_after();
      const int m = ti.m0 + q * 32 + lane;
      const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + acc * BN;
      if constexpr (STAGED) {
        static_assert(BN % 32 == 0, "staged epilogue works on whole 32-column chunks");
        uint8_t* stg = smem + S::STG_OFF + (warp - 2) * (NSTG * 4096);
        float* sb = reinterpret_cast<float*>(smem + S::SB_OFF) + (warp - 2) * S::SB_CHUNKS * 32;
        __syncwarp();                    // every lane is done with the last tile's bias
#pragma unroll
        for (int jj = 0; jj < S::SB_CHUNKS; ++jj) sb[jj * 32 + lane] = bl[jj];
        __syncwarp();
        // this warp's chunks j = half, half + WPQ, ...; the TMEM load of the
        // next one is in flight while the current one is processed
        // (with more than two warps per quarter the others hide the load latency,
        // and a single buffer keeps the registers within the budget)
        constexpr int NCH = BN / 32;
        constexpr int NVB = WPQ > 2 ? 1 : 2;
        const int cnt = (NCH - half + WPQ - 1) / WPQ;
        float vb[NVB][32];
        if (cnt > 0) tmem_ld32(tl + half * 32, vb[0]);
#pragma unroll
        for (int jj = 0; jj < (NCH + WPQ - 1) / WPQ; ++jj) {
          if (jj >= cnt) break;
          const int j = half + WPQ * jj;
          float* v = vb[jj % NVB];
          tmem_wait_ld32(v);
          if (NVB == 2 && jj + 1 < cnt) tmem_ld32(tl + (j + WPQ) * 32, vb[(jj + 1) % NVB]);
          const int n = ti.n0 + j * 32;
          // the same 32 bias values for every lane: broadcast reads (zero past N,
          // where the TMA store clips the columns anyway)
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 b4 = *reinterpret_cast<const float4*>(sb + jj * 32 + c);
            const float2 l2e = make_float2(1.4426950408889634f, 1.4426950408889634f);
            const float2 lo = ffma2(make_float2(v[c], v[c + 1]), l2e, make_float2(b4.x, b4.y));
            const float2 hi = ffma2(make_float2(v[c + 2], v[c + 3]), l2e, make_float2(b4.z, b4.w));
            v[c] = lo.x; v[c + 1] = lo.y; v[c + 2] = hi.x; v[c + 3] = hi.y;
          }
          softplus32_log2(v);
          uint8_t* buf = stg + (stg_count % NSTG) * 4096;
          if (lane == 0) bulk_wait_read<NSTG - 1>();   // this buffer's previous store has read it
          __syncwarp();
          // row `lane` of the 32 x 32 box, 16-byte chunks placed by the 128-byte swizzle
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, smem_u32(buf), n, ti.m0 + q * 32);
            bulk_commit();
          }
          ++stg_count;
          if (NVB == 1 && jj + 1 < cnt) tmem_ld32(tl + (j + WPQ) * 32, vb[0]);
        }
      } else if constexpr (EPI != EPI_SWIGLU) {
#pragma unroll 1
        for (int j = half; j < BN / 32; j += WPQ) {
          float v[32];
          tmem_ld32(tl + j * 32, v);
          tmem_wait_ld();
          epi_chunk<EPI, TRANS, 32>(p, ti, m, ti.n0 + j * 32, v);
        }
        if constexpr (BN % 32 != 0) {
          if (half == (BN / 32) % WPQ) {
            float v[16];
            tmem_ld16(tl + (BN / 32) * 32, v);
            tmem_wait_ld();
            epi_chunk<EPI, TRANS, 16>(p, ti, m, ti.n0 + (BN / 32) * 32, v);
          }
        }
      } else {
        bf16* o = reinterpret_cast<bf16*>(p.out) + (long long)m * p.ldo;
#pragma unroll 1
        for (int j = half; j < BN / 64; j += WPQ) {
          float g[32], u[32];
          tmem_ld32(tl + j * 32, g);
          tmem_ld32(tl + BN / 2 + j * 32, u);
          tmem_wait_ld();
          if (m < ti.m_end) {
            const int n = ti.n0 + j * 32;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              float w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) w[i] = silu(g[c + i]) * u[c + i];
              if (n + c + 8 <= p.N) {
                store_bf16x8(o + n + c, w);
              } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  if (n + c + i < p.N) o[n + c + i] = __float2bfloat16_rn(w[i]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
    }
    if constexpr (STAGED) {
      if (lane == 0) bulk_wait_all();   // shared memory must outlive the stores reading it
      __syncwarp();
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, S::TMEM_COLS);
  }
}

}  // namespace jb
