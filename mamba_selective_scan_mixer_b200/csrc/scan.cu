// Selective scan with D skip and SiLU(z) gate (prefill), and the one-token
// decode state update.
//
// Recurrence of the Mamba layer used by Jamba ("Jamba: A Hybrid
// Transformer-Mamba Language Model", section 2, ref [17]), per channel c and
// state n:  h_t = exp(dt_t A) h_{t-1} + dt_t B_t x_t,
//           y_t = (C_t . h_t + D x_t) * SiLU(z_t).
//
// Prefill kernel layout: a CTA owns 256 channels (2 per thread, all 16 states
// of each in fp32 registers) of one batch row and one time chunk.  x, z, dt, B
// and C arrive through a 4-stage TMA ring of 4-step tiles.  Chunks run
// concurrently; CTAs take tickets in (chunk, group) order and pass the state
// between chunks with a decoupled look-back over per-chunk records
// (aggregate: decay product P and local end state; inclusive: true end state).
// Until the carried-in state is known, a chunk's outputs depend on it through
// C_t . (P_t * h_in); those steps are written as fp32 pre-gate values and
// finished once h_in arrives.  P_t only shrinks towards zero: once it is
// exactly zero for every channel of a warp, later steps no longer depend on
// h_in and are gated and stored directly.
//
// When every channel of the CTA has A[c, n] == (n + 1) * A[c, 0] (the
// initialisation used by Mamba layers), exp(dt A_n) = r^(n+1) with
// r = exp(dt A_0): one exponential and 15 products per step instead of 16
// exponentials.  Other A take the general path.
#include <string>

#include "common.cuh"
#include "host.hpp"

namespace jb {

constexpr int SCAN_THREADS = 128;
constexpr int SCAN_CH = 256;   // channels per CTA (2 per thread)
constexpr int SCAN_Q = 4;      // time steps per pipeline stage
constexpr int SCAN_STAGES = 4;
constexpr int NS = 16;         // d_state
constexpr float LOG2E = 1.4426950408889634f;

__host__ __device__ constexpr int al128(int v) { return (v + 127) & ~127; }

template <typename TX, typename TBC>
struct ScanLayout {
  static constexpr int X = SCAN_Q * SCAN_CH * (int)sizeof(TX);
  static constexpr int DT = SCAN_Q * SCAN_CH * 4;
  static constexpr int BCB = SCAN_Q * NS * (int)sizeof(TBC);
  static constexpr int STAGE_TX = 2 * X + DT + 2 * BCB;  // bytes landed per stage
  static constexpr int OFF_Z = X, OFF_DT = 2 * X, OFF_B = 2 * X + DT, OFF_C = OFF_B + al128(BCB);
  static constexpr int STAGE = OFF_C + al128(BCB);
  static constexpr int OFF_BCF = SCAN_STAGES * STAGE;                 // fp32 B|C [STAGES][Q][32]
  static constexpr int OFF_A2 = OFF_BCF + SCAN_STAGES * SCAN_Q * 32 * 4;  // A*log2(e) [256][16]
  static constexpr int OFF_BAR = OFF_A2 + SCAN_CH * NS * 4;
  static constexpr int BYTES = OFF_BAR + 128 + 128;                  // + alignment slack
  static_assert(SCAN_Q * 32 == SCAN_THREADS, "one B|C element per thread per stage");
  static_assert(2 * SCAN_CH * NS * 4 <= SCAN_STAGES * STAGE, "look-back scratch fits the stage ring");
};

struct ScanArgs {
  long long ld_x, ld_z, ld_dt, ld_b, ld_c, ld_y;
  const float* dt;       // for the fix-up pass
  const void* z;
  const void* C;
  const float* A;
  const float* D;
  const float* h0;
  void* y;
  float* h_out;
  int batch, L, di;
  int chunk_len, n_chunks, cgroups;
  int* ticket;
  int* flags;            // [batch * cgroups * n_chunks]
  float* rec;            // per record: P[256][16], h[256][16], incl[256][16]
  float* ylocal;         // [batch * L, di] fp32
  int* err;
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <typename T> struct Pair;
template <> struct Pair<bf16> {
  static __device__ __forceinline__ float2 load(const bf16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  }
  static __device__ __forceinline__ void store(bf16* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
  }
};
template <> struct Pair<float> {
  static __device__ __forceinline__ float2 load(const float* p) { return *reinterpret_cast<const float2*>(p); }
  static __device__ __forceinline__ void store(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  }
};

// r^1 .. r^16
__device__ __forceinline__ void powers16(float r, float* pw) {
  pw[0] = r;
  pw[1] = r * r;
  float2 p34 = fmul2(make_float2(pw[1], pw[1]), make_float2(pw[0], pw[1]));
  pw[2] = p34.x; pw[3] = p34.y;
  float2 p56 = fmul2(make_float2(pw[3], pw[3]), make_float2(pw[0], pw[1]));
  float2 p78 = fmul2(make_float2(pw[3], pw[3]), make_float2(pw[2], pw[3]));
  pw[4] = p56.x; pw[5] = p56.y; pw[6] = p78.x; pw[7] = p78.y;
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    float2 q = fmul2(make_float2(pw[7], pw[7]), make_float2(pw[i], pw[i + 1]));
    pw[8 + i] = q.x; pw[9 + i] = q.y;
  }
}

template <typename TX, typename TBC, bool FAST>
__device__ __forceinline__ void scan_chunk(const CUtensorMap* mx, const CUtensorMap* mz, const CUtensorMap* mdt,
                                           const CUtensorMap* mB, const CUtensorMap* mC, const ScanArgs& a,
                                           uint8_t* smem, int b, int cg, int chunk, int grp) {
  using Lyt = ScanLayout<TX, TBC>;
  const int tid = threadIdx.x, lane = tid & 31;
  const int c_base = cg * SCAN_CH;
  const int cl = tid * 2;            // local channel of this thread's first channel
  const int c = c_base + cl;
  const bool valid = c < a.di;       // d_inner is a multiple of 8: both channels valid or neither
  const int t0 = chunk * a.chunk_len;
  const int t1 = min(a.L, t0 + a.chunk_len);
  const long long row0 = (long long)b * a.L;
  float* sBCf = reinterpret_cast<float*>(smem + Lyt::OFF_BCF);
  const float* sA2 = reinterpret_cast<const float*>(smem + Lyt::OFF_A2);
  const uint32_t full0 = smem_u32(smem + Lyt::OFF_BAR);
  __shared__ int s_flag;

  float A2_0[2], Dv[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    A2_0[j] = sA2[(cl + j) * NS];
    Dv[j] = valid ? __ldg(a.D + c + j) : 0.f;
  }

  const bool known = (chunk == 0);   // the state entering chunk 0 is h0 (or zero)
  float2 h[2][8];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (known && a.h0 && valid) {
        const float* src = a.h0 + ((long long)b * a.di + c + j) * NS + 2 * i;
        h[j][i] = make_float2(src[0], src[1]);
      } else {
        h[j][i] = make_float2(0.f, 0.f);
      }
    }
  // decay product since t0 (only tracked while the warp still buffers)
  float R[2] = {1.f, 1.f};
  float2 P[2][8];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 8; ++i) P[j][i] = make_float2(1.f, 1.f);
  bool buffering = !known;
  int tA_end = t0;

  const int nsub = (t1 - t0 + SCAN_Q - 1) / SCAN_Q;
  auto issue = [&](int i) {
    const int slot = i % SCAN_STAGES;
    uint8_t* st = smem + slot * Lyt::STAGE;
    const uint32_t bar = full0 + 8 * slot;
    const int row = (int)(row0 + t0 + i * SCAN_Q);
    mbar_arrive_tx(bar, Lyt::STAGE_TX);
    tma_load_2d(smem_u32(st), mx, bar, c_base, row);
    tma_load_2d(smem_u32(st + Lyt::OFF_Z), mz, bar, c_base, row);
    tma_load_2d(smem_u32(st + Lyt::OFF_DT), mdt, bar, c_base, row);
    tma_load_2d(smem_u32(st + Lyt::OFF_B), mB, bar, 0, row);
    tma_load_2d(smem_u32(st + Lyt::OFF_C), mC, bar, 0, row);
  };
  if (tid == 0)
    for (int i = 0; i < SCAN_STAGES - 1 && i < nsub; ++i) issue(i);

  bool aborted = false;
  for (int i = 0; i < nsub; ++i) {
    const int slot = i % SCAN_STAGES;
    const uint8_t* st = smem + slot * Lyt::STAGE;
    const bool ok = mbar_wait(full0 + 8 * slot, (uint32_t)((i / SCAN_STAGES) & 1), a.err);
    if (ok) {
      // widen B|C of this stage to fp32, one element per thread
      const int q = tid >> 5, k = tid & 31;
      const TBC* src = reinterpret_cast<const TBC*>(st + (k < 16 ? Lyt::OFF_B : Lyt::OFF_C));
      sBCf[(slot * SCAN_Q + q) * 32 + k] = to_f(src[q * NS + (k & 15)]);
    }
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    if (tid == 0 && i + SCAN_STAGES - 1 < nsub) issue(i + SCAN_STAGES - 1);

    const TX* sx = reinterpret_cast<const TX*>(st);
    const TX* sz = reinterpret_cast<const TX*>(st + Lyt::OFF_Z);
    const float* sdt = reinterpret_cast<const float*>(st + Lyt::OFF_DT);
#pragma unroll
    for (int q = 0; q < SCAN_Q; ++q) {
      const int t = t0 + i * SCAN_Q + q;
      if (t >= t1) break;
      const float2 xv = Pair<TX>::load(sx + q * SCAN_CH + cl);
      const float2 dv = *reinterpret_cast<const float2*>(sdt + q * SCAN_CH + cl);
      const float* bc = sBCf + (slot * SCAN_Q + q) * 32;
      float y[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float xj = j ? xv.y : xv.x, dj = j ? dv.y : dv.x;
        const float u = dj * xj;
        float pw[16];
        if constexpr (FAST) {
          const float r = ex2(dj * A2_0[j]);
          powers16(r, pw);
          if (buffering) R[j] *= r;
        } else {
#pragma unroll
          for (int n = 0; n < NS; ++n) pw[n] = ex2(dj * sA2[(cl + j) * NS + n]);
        }
        float2 ya = make_float2(0.f, 0.f);
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          const float2 Bn = *reinterpret_cast<const float2*>(bc + 2 * n2);
          const float2 Cn = *reinterpret_cast<const float2*>(bc + 16 + 2 * n2);
          const float2 uB = fmul2(make_float2(u, u), Bn);
          h[j][n2] = ffma2(make_float2(pw[2 * n2], pw[2 * n2 + 1]), h[j][n2], uB);
          ya = ffma2(Cn, h[j][n2], ya);
          if constexpr (!FAST) {
            if (buffering) P[j][n2] = fmul2(P[j][n2], make_float2(pw[2 * n2], pw[2 * n2 + 1]));
          }
        }
        y[j] = ya.x + ya.y + Dv[j] * xj;
      }
      if (valid) {
        const long long row = row0 + t;
        if (buffering) {
          *reinterpret_cast<float2*>(a.ylocal + row * a.di + c) = make_float2(y[0], y[1]);
        } else {
          const float2 zv = Pair<TX>::load(sz + q * SCAN_CH + cl);
          Pair<TX>::store(reinterpret_cast<TX*>(a.y) + row * a.ld_y + c, y[0] * silu(zv.x), y[1] * silu(zv.y));
        }
      }
    }
    if (buffering) {
      bool zero;
      if constexpr (FAST) {
        zero = (R[0] == 0.f && R[1] == 0.f) || !valid;
      } else {
        zero = true;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int n2 = 0; n2 < 8; ++n2) zero = zero && P[j][n2].x == 0.f && P[j][n2].y == 0.f;
        zero = zero || !valid;
      }
      if (__all_sync(0xffffffffu, zero)) {
        buffering = false;
        tA_end = min(t1, t0 + (i + 1) * SCAN_Q);
      }
    }
  }
  if (buffering) tA_end = t1;
  if (__syncthreads_or(aborted)) return;

  // ---------------------------------------------------------- carry
  const long long rbase = (long long)grp * a.n_chunks;
  constexpr int REC = 3 * SCAN_CH * NS;
  float* myrec = a.rec + (rbase + chunk) * REC;
  int* myflag = a.flags + rbase + chunk;
  const bool independent = __syncthreads_and(!buffering) != 0;  // end state does not depend on h_in
  float Pend[2][16];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    if constexpr (FAST) {
      powers16(R[j], Pend[j]);
    } else {
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2) { Pend[j][2 * n2] = P[j][n2].x; Pend[j][2 * n2 + 1] = P[j][n2].y; }
    }
  }
  if (independent) {
    // publish the true end state right away so later chunks need not wait
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2)
        *reinterpret_cast<float2*>(myrec + 2 * SCAN_CH * NS + (cl + j) * NS + 2 * n2) = h[j][n2];
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(myflag, 2);
  } else {
    // aggregate: decay product of the chunk (exactly zero for warps whose carry died out) and local end state
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n = 0; n < NS; n += 2) {
        *reinterpret_cast<float2*>(myrec + (cl + j) * NS + n) = make_float2(Pend[j][n], Pend[j][n + 1]);
        *reinterpret_cast<float2*>(myrec + SCAN_CH * NS + (cl + j) * NS + n) = h[j][n / 2];
      }
    __threadfence();
    __syncthreads();
    if (tid == 0) st_release(myflag, 1);
  }

  float hin[2][16];
  if (!known) {
    // look back: h_in = h_{k-1} + P_{k-1} (h_{k-2} + P_{k-2} (... + incl_j))
    float* sP = reinterpret_cast<float*>(smem);              // [256][16], the stage ring is free now
    float* sH = sP + SCAN_CH * NS;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n = 0; n < NS; ++n) {
        sP[(cl + j) * NS + n] = 1.f;
        sH[(cl + j) * NS + n] = 0.f;
      }
    int jc = chunk - 1;
    bool done = false;
    while (!done) {
      if (tid == 0) {
        int f = ld_acquire(a.flags + rbase + jc);
        if (f == 0) {
          const uint64_t start = globaltimer();
          for (uint32_t it = 1; f == 0; ++it) {
            f = ld_acquire(a.flags + rbase + jc);
            if (f == 0 && (it & 255) == 0) {
              if (error_raised(a.err)) { f = -1; break; }
              if (globaltimer() - start > kWaitLimitNs) { set_error(a.err, JAMBA_ERR_TIMEOUT); f = -1; break; }
            }
          }
        }
        s_flag = f;
      }
      __syncthreads();
      const int f = s_flag;
      if (f < 0) return;   // uniform: every thread read the same s_flag
      __threadfence();
      const float* rP = a.rec + (rbase + jc) * REC;
      bool allzero = true;
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int n = 0; n < NS; ++n) {
          const int o = (cl + j) * NS + n;
          if (f == 2) {
            sH[o] = fmaf(sP[o], __ldcg(rP + 2 * SCAN_CH * NS + o), sH[o]);
          } else {
            sH[o] = fmaf(sP[o], __ldcg(rP + SCAN_CH * NS + o), sH[o]);
            sP[o] *= __ldcg(rP + o);
            allzero = allzero && sP[o] == 0.f;
          }
        }
      if (f == 2) {
        done = true;
      } else {
        --jc;
        if (__syncthreads_and(allzero)) done = true;
      }
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n = 0; n < NS; ++n) hin[j][n] = sH[(cl + j) * NS + n];

    if (!independent) {
      // true end state h + P_end * h_in, published as this chunk's inclusive record
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          h[j][n2].x = fmaf(Pend[j][2 * n2], hin[j][2 * n2], h[j][n2].x);
          h[j][n2].y = fmaf(Pend[j][2 * n2 + 1], hin[j][2 * n2 + 1], h[j][n2].y);
          *reinterpret_cast<float2*>(myrec + 2 * SCAN_CH * NS + (cl + j) * NS + 2 * n2) = h[j][n2];
        }
      __threadfence();
      __syncthreads();
      if (tid == 0) st_release(myflag, 2);
    }

    // finish the buffered steps of this warp: y = (y_local + C . (P_t * h_in)) * SiLU(z)
    if (valid) {
      const TX* zg = reinterpret_cast<const TX*>(a.z);
      const TBC* Cg = reinterpret_cast<const TBC*>(a.C);
      float Rf[2] = {1.f, 1.f};
      float2 Pf[2][8];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) Pf[j][n2] = make_float2(1.f, 1.f);
#pragma unroll 2
      for (int t = t0; t < tA_end; ++t) {
        const long long row = row0 + t;
        const float2 yl = __ldcg(reinterpret_cast<const float2*>(a.ylocal + row * a.di + c));
        const float2 dv = __ldg(reinterpret_cast<const float2*>(a.dt + row * a.ld_dt + c));
        const float2 zv = Pair<TX>::load(zg + row * a.ld_z + c);
        float Cv[16];
#pragma unroll
        for (int n = 0; n < NS; ++n) Cv[n] = to_f(Cg[row * a.ld_c + n]);
        float yo[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float dj = j ? dv.y : dv.x;
          float corr;
          if constexpr (FAST) {
            Rf[j] *= ex2(dj * A2_0[j]);
            float acc = Cv[15] * hin[j][15];
#pragma unroll
            for (int n = 14; n >= 0; --n) acc = fmaf(acc, Rf[j], Cv[n] * hin[j][n]);
            corr = acc * Rf[j];
          } else {
            corr = 0.f;
#pragma unroll
            for (int n2 = 0; n2 < 8; ++n2) {
              const float2 e = make_float2(ex2(dj * sA2[(cl + j) * NS + 2 * n2]),
                                           ex2(dj * sA2[(cl + j) * NS + 2 * n2 + 1]));
              Pf[j][n2] = fmul2(Pf[j][n2], e);
              corr = fmaf(Cv[2 * n2] * hin[j][2 * n2], Pf[j][n2].x, corr);
              corr = fmaf(Cv[2 * n2 + 1] * hin[j][2 * n2 + 1], Pf[j][n2].y, corr);
            }
          }
          yo[j] = ((j ? yl.y : yl.x) + corr) * silu(j ? zv.y : zv.x);
        }
        Pair<TX>::store(reinterpret_cast<TX*>(a.y) + row * a.ld_y + c, yo[0], yo[1]);
      }
    }
  }

  // final state of the batch row
  if (t1 == a.L && a.h_out && valid) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2)
        *reinterpret_cast<float2*>(a.h_out + ((long long)b * a.di + c + j) * NS + 2 * n2) = h[j][n2];
  }
}

template <typename TX, typename TBC>
__global__ void __launch_bounds__(SCAN_THREADS)
selective_scan_kernel(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mz,
                      const __grid_constant__ CUtensorMap mdt, const __grid_constant__ CUtensorMap mB,
                      const __grid_constant__ CUtensorMap mC, const ScanArgs a) {
  using Lyt = ScanLayout<TX, TBC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ int s_ticket;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_ticket = atomicAdd(a.ticket, 1);
    const uint32_t full0 = smem_u32(smem + Lyt::OFF_BAR);
    for (int s = 0; s < SCAN_STAGES; ++s) mbar_init(full0 + 8 * s, 1);
    mbar_fence_init();
    tma_prefetch(&mx);
    tma_prefetch(&mz);
    tma_prefetch(&mdt);
    tma_prefetch(&mB);
    tma_prefetch(&mC);
  }
  __syncthreads();
  const int groups_total = a.batch * a.cgroups;
  const int ticket = s_ticket;
  const int chunk = ticket / groups_total;
  const int grp = ticket - chunk * groups_total;
  const int b = grp / a.cgroups, cg = grp - b * a.cgroups;

  // A * log2(e) of this CTA's channels, and whether A[c, n] == (n + 1) A[c, 0]
  float* sA2 = reinterpret_cast<float*>(smem + Lyt::OFF_A2);
  bool ok = true;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int c = cg * SCAN_CH + tid * 2 + j;
    const bool v = c < a.di;
    const float a0 = v ? __ldg(a.A + (long long)c * NS) : 0.f;
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      const float an = v ? __ldg(a.A + (long long)c * NS + n) : 0.f;
      ok = ok && (an == (float)(n + 1) * a0);
      sA2[(tid * 2 + j) * NS + n] = an * LOG2E;
    }
  }
  const bool fast = __syncthreads_and(ok) != 0;
  if (fast)
    scan_chunk<TX, TBC, true>(&mx, &mz, &mdt, &mB, &mC, a, smem, b, cg, chunk, grp);
  else
    scan_chunk<TX, TBC, false>(&mx, &mz, &mdt, &mB, &mC, a, smem, b, cg, chunk, grp);
}

// ------------------------------------------------------------ decode step
// One thread per (batch row, channel): advances the cached state by one token.
template <typename TX>
__global__ void __launch_bounds__(256)
ssm_step_kernel(const TX* __restrict__ xc, const TX* __restrict__ z, long long ld_z, const float* __restrict__ dt,
                const float* __restrict__ bc, long long ld_bc, const float* __restrict__ A,
                const float* __restrict__ D, float* __restrict__ state, TX* __restrict__ y, int batch, int di) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)batch * di) return;
  const int b = (int)(i / di), c = (int)(i - (long long)b * di);
  const float x = to_f(xc[i]);
  const float d = dt[i];
  const float* Bv = bc + (long long)b * ld_bc;
  const float* Cv = Bv + NS;
  float4* hs = reinterpret_cast<float4*>(state + i * NS);
  const float4* Ar = reinterpret_cast<const float4*>(A + (long long)c * NS);
  float acc = 0.f;
  const float u = d * x;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float4 h = hs[k];
    const float4 av = __ldg(Ar + k);
    h.x = fmaf(ex2(d * av.x * LOG2E), h.x, u * Bv[4 * k + 0]);
    h.y = fmaf(ex2(d * av.y * LOG2E), h.y, u * Bv[4 * k + 1]);
    h.z = fmaf(ex2(d * av.z * LOG2E), h.z, u * Bv[4 * k + 2]);
    h.w = fmaf(ex2(d * av.w * LOG2E), h.w, u * Bv[4 * k + 3]);
    acc = fmaf(Cv[4 * k + 0], h.x, acc);
    acc = fmaf(Cv[4 * k + 1], h.y, acc);
    acc = fmaf(Cv[4 * k + 2], h.z, acc);
    acc = fmaf(Cv[4 * k + 3], h.w, acc);
    hs[k] = h;
  }
  const float zv = to_f(z[(long long)b * ld_z + c]);
  y[i] = from_f<TX>((acc + __ldg(D + c) * x) * silu(zv));
}

// ------------------------------------------------------------ host side
size_t scan_workspace_bytes(int batch, int L, int di, int chunk_len) {
  const int cgroups = (di + SCAN_CH - 1) / SCAN_CH;
  const int n_chunks = (L + chunk_len - 1) / chunk_len;
  const size_t recs = (size_t)batch * cgroups * n_chunks;
  size_t bytes = 256;                                       // ticket
  bytes += (recs * sizeof(int) + 255) & ~size_t(255);       // flags
  bytes += recs * 3 * SCAN_CH * NS * sizeof(float);         // records
  bytes += (size_t)batch * L * di * sizeof(float);          // buffered pre-gate outputs
  return bytes;
}

int scan_auto_chunk(int batch, int L, int di) {
  const int cgroups = (di + SCAN_CH - 1) / SCAN_CH;
  const int groups = batch * cgroups;
  // aim for about two resident CTAs per SM
  const int want = 2 * num_sms();
  int n_chunks = (want + groups - 1) / groups;
  if (n_chunks < 1) n_chunks = 1;
  int chunk = (L + n_chunks - 1) / n_chunks;
  chunk = (chunk + 15) & ~15;
  if (chunk < 16) chunk = 16;
  return chunk;
}


template <typename TX, typename TBC>
static jamba_status launch_scan(const ScanCall& s, cudaStream_t st) {
  using Lyt = ScanLayout<TX, TBC>;
  const CUtensorMapDataType tx = sizeof(TX) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapDataType tb = sizeof(TBC) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const uint64_t rows = (uint64_t)s.batch * s.L;
  CUtensorMap mx, mz, mdt, mB, mC;
  JB_TRY(make_map_2d(&mx, s.x, tx, sizeof(TX), s.di, rows, s.ld_x * sizeof(TX), SCAN_CH, SCAN_Q, CU_TENSOR_MAP_SWIZZLE_NONE));
  JB_TRY(make_map_2d(&mz, s.z, tx, sizeof(TX), s.di, rows, s.ld_z * sizeof(TX), SCAN_CH, SCAN_Q, CU_TENSOR_MAP_SWIZZLE_NONE));
  JB_TRY(make_map_2d(&mdt, s.dt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, s.di, rows, s.ld_dt * 4, SCAN_CH, SCAN_Q, CU_TENSOR_MAP_SWIZZLE_NONE));
  JB_TRY(make_map_2d(&mB, s.B, tb, sizeof(TBC), NS, rows, s.ld_b * sizeof(TBC), NS, SCAN_Q, CU_TENSOR_MAP_SWIZZLE_NONE));
  JB_TRY(make_map_2d(&mC, s.C, tb, sizeof(TBC), NS, rows, s.ld_c * sizeof(TBC), NS, SCAN_Q, CU_TENSOR_MAP_SWIZZLE_NONE));

  ScanArgs a;
  a.ld_x = s.ld_x; a.ld_z = s.ld_z; a.ld_dt = s.ld_dt; a.ld_b = s.ld_b; a.ld_c = s.ld_c; a.ld_y = s.ld_y;
  a.dt = s.dt; a.z = s.z; a.C = s.C; a.A = s.A; a.D = s.D; a.h0 = s.h0; a.y = s.y; a.h_out = s.h_out;
  a.batch = s.batch; a.L = s.L; a.di = s.di;
  a.chunk_len = s.chunk;
  a.n_chunks = (s.L + s.chunk - 1) / s.chunk;
  a.cgroups = (s.di + SCAN_CH - 1) / SCAN_CH;
  const size_t recs = (size_t)s.batch * a.cgroups * a.n_chunks;
  uint8_t* w = reinterpret_cast<uint8_t*>(s.ws);
  a.ticket = reinterpret_cast<int*>(w);
  a.flags = reinterpret_cast<int*>(w + 256);
  const size_t flags_bytes = (recs * sizeof(int) + 255) & ~size_t(255);
  a.rec = reinterpret_cast<float*>(w + 256 + flags_bytes);
  a.ylocal = a.rec + recs * 3 * SCAN_CH * NS;
  a.err = device_error_word();
  if (!a.err) return fail(JAMBA_ERR_CUDA, "could not allocate the device status word");
  JB_CUDA(cudaMemsetAsync(w, 0, 256 + flags_bytes, st));

  static bool configured[64] = {false};
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(selective_scan_kernel<TX, TBC>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lyt::BYTES));
    configured[dev] = true;
  }
  const long long grid = (long long)recs;
  selective_scan_kernel<TX, TBC><<<(unsigned)grid, SCAN_THREADS, Lyt::BYTES, st>>>(mx, mz, mdt, mB, mC, a);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

jamba_status scan_run(const ScanCall& s, cudaStream_t st) {
  if (s.batch <= 0 || s.L <= 0 || s.di <= 0) return fail(JAMBA_ERR_INVALID_ARG, "scan: sizes must be positive");
  if (s.di % 8) return fail(JAMBA_ERR_UNSUPPORTED, "scan: d_inner must be a multiple of 8");
  if (!s.x || !s.z || !s.dt || !s.B || !s.C || !s.A || !s.D || !s.y)
    return fail(JAMBA_ERR_INVALID_ARG, "scan: null tensor");
  if (s.chunk <= 0 || s.chunk % 16) return fail(JAMBA_ERR_INVALID_ARG, "scan: chunk must be a positive multiple of 16");
  if (s.ld_x < s.di || s.ld_z < s.di || s.ld_dt < s.di || s.ld_y < s.di || s.ld_b < NS || s.ld_c < NS)
    return fail(JAMBA_ERR_INVALID_ARG, "scan: leading dimension below the row width");
  if (s.ld_y % 2 || s.ld_z % 2 || s.ld_dt % 2)
    return fail(JAMBA_ERR_INVALID_ARG, "scan: leading dimensions of y, z, dt must be even");
  if (!aligned16(s.y) || !aligned16(s.z) || !aligned16(s.dt))
    return fail(JAMBA_ERR_INVALID_ARG, "scan: y, z and dt must be 16-byte aligned");
  if (s.ws_bytes < scan_workspace_bytes(s.batch, s.L, s.di, s.chunk) || !s.ws || !aligned16(s.ws))
    return fail(JAMBA_ERR_WORKSPACE, "scan: workspace too small");
  if (s.dtype == JAMBA_BF16 && s.bc_dtype == JAMBA_BF16) return launch_scan<bf16, bf16>(s, st);
  if (s.dtype == JAMBA_BF16 && s.bc_dtype == JAMBA_F32) return launch_scan<bf16, float>(s, st);
  if (s.dtype == JAMBA_F32 && s.bc_dtype == JAMBA_F32) return launch_scan<float, float>(s, st);
  return fail(JAMBA_ERR_UNSUPPORTED, "scan: unsupported dtype combination");
}

jamba_status ssm_step(const void* xc, const void* z, long long ld_z, const float* dt, const float* bc,
                      long long ld_bc, const float* A, const float* D, float* state, void* y, int batch, int di,
                      int dtype, cudaStream_t st) {
  const long long n = (long long)batch * di;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == JAMBA_BF16)
    ssm_step_kernel<bf16><<<grid, 256, 0, st>>>(reinterpret_cast<const bf16*>(xc), reinterpret_cast<const bf16*>(z),
                                               ld_z, dt, bc, ld_bc, A, D, state, reinterpret_cast<bf16*>(y), batch, di);
  else
    ssm_step_kernel<float><<<grid, 256, 0, st>>>(reinterpret_cast<const float*>(xc), reinterpret_cast<const float*>(z),
                                                ld_z, dt, bc, ld_bc, A, D, state, reinterpret_cast<float*>(y), batch, di);
  JB_CUDA(cudaGetLastError());
  return JAMBA_OK;
}

}  // namespace jb
