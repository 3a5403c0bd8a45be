// Grouped expert GEMM with INT8 weights (ExpertsInt8: the expert matrices are
// stored as 8-bit codes with one fp32 scale per output row and are widened
// inside this kernel; activations stay bf16).
//
//   D[m, n] = scale[g, n] * sum_k A[m, k] * q[g, n, k]     (rows m of group g)
//
// A: the gathered activations [rows, K] bf16; q: [groups, N_rows, K] int8.
// The widened weights are exact (|q| <= 127 fits bf16), so the only rounding
// is the fp32 accumulation and the scale product, as in the bf16 path.
//
// One persistent CTA per SM, 14 warps:
//   warp 0      TMA producer: per k-step MT activation tiles (128 x 64 bf16,
//               128-byte swizzle) and the 256 x 64 code tile (unswizzled
//               bytes) into a TSTAGES-deep ring;
//   warp 1      TMEM owner and MMA issuer: M = 128, N = 256, K = 16 per
//               instruction, MT accumulators per tile (MT = 2: both halves of
//               a 256-row tile share one widened weight tile);
//   warps 2-9   epilogue: scales, SwiGLU or fp32 stores;
//   warps 10-13 dequantisers: code tile -> bf16 weight tile in the 128-byte
//               swizzled K-major layout, into a separate BSTAGES-deep ring,
//               so widening k-step i + 1 overlaps the MMAs of k-step i.
// Widening one code: the low 7 bits l go under the bf16 exponent of 128
// (value 128 + l) and the sign bit under the same exponent (value 128 or
// 256); their bf16 difference is the code exactly.  Two codes per
// instruction: 2 LOP3 + 4 PRMT + 2 HSUB2 per 4 codes.
// Every wait is bounded (see common.cuh).
#pragma once
#include "gemm_tc.cuh"

namespace jb {

constexpr int I8W_THREADS = 448;
constexpr int I8W_BN = 256;          // MMA N: SwiGLU 128 gate + 128 up rows, or 256 down rows
constexpr int I8W_TSTAGES = 3;
constexpr int I8W_BSTAGES = 2;
constexpr int I8W_DQ_WARPS = 4;

template <int MT>
struct I8wSmem {
  static constexpr uint32_t A_BYTES = 128 * 128;              // one 128 x 64 bf16 activation tile
  static constexpr uint32_t Q_BYTES = I8W_BN * 64;            // 256 x 64 codes
  static constexpr uint32_t B_BYTES = I8W_BN * 128;           // 256 x 64 bf16 widened weights
  static constexpr uint32_t T_STAGE = MT * A_BYTES + Q_BYTES;
  static constexpr uint32_t B_OFF = I8W_TSTAGES * T_STAGE;
  static constexpr uint32_t BAR_OFF = B_OFF + I8W_BSTAGES * B_BYTES;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};

// bf16x2 a - b (exact here: both operands and the result are small integers)
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 16 int8 codes (little-endian) -> 16 bf16 values, exactly
__device__ __forceinline__ void widen16(uint4 v, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t l = w[i] & 0x7F7F7F7Fu, s = w[i] & 0x80808080u;
    // bytes {l0, 0x43, l1, 0x43}: bf16 128 + l; {s0, 0x43, s1, 0x43}: bf16 128 or 256
    o[2 * i] = bf16x2_sub(__byte_perm(l, 0x43434343u, 0x5140u), __byte_perm(s, 0x43434343u, 0x5140u));
    o[2 * i + 1] = bf16x2_sub(__byte_perm(l, 0x43434343u, 0x5342u), __byte_perm(s, 0x43434343u, 0x5342u));
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// ROWS x 64 codes (row-major, 64-byte rows) -> ROWS x 64 bf16 in the 128-byte
// swizzled K-major layout, by the I8W_DQ_WARPS dequantiser warps.  16 codes
// per load become two 16-byte chunks of the same row; a quarter-warp covers
// two rows and stores to eight distinct chunks (no bank conflicts).  The
// offsets are the same for every stage and are worked out once.
template <int ROWS>
struct WidenPlanLinear {
  static constexpr int PER = 32 * I8W_DQ_WARPS;
  static constexpr int IT = ROWS * 4 / PER;
  static_assert(IT * PER == ROWS * 4, "whole iterations");
  uint32_t dlo[IT], dhi[IT];
  uint32_t src0;
  __device__ __forceinline__ explicit WidenPlanLinear(int ct) {
    src0 = ct * 16;
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      const int idx = ct + PER * i;
      const int row = idx >> 2, g = idx & 3;
      dlo[i] = row * 128 + (((2 * g) ^ (row & 7)) << 4);
      dhi[i] = row * 128 + (((2 * g + 1) ^ (row & 7)) << 4);
    }
  }
  // q, b: shared-memory addresses of the code tile and the widened tile.  All
  // loads go out before the first store: the accesses are ordered asm
  // statements, so a load placed after a store would wait for the widening of
  // the codes before it, one load latency per iteration.
  __device__ __forceinline__ void run(uint32_t q, uint32_t b) const {
    uint4 v[IT];
#pragma unroll
    for (int i = 0; i < IT; ++i)
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w) : "r"(q + src0 + PER * 16 * i));
#pragma unroll
    for (int i = 0; i < IT; ++i) {
      uint4 lo, hi;
      widen16(v[i], lo, hi);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(b + dlo[i]), "r"(lo.x), "r"(lo.y), "r"(lo.z),
                   "r"(lo.w) : "memory");
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(b + dhi[i]), "r"(hi.x), "r"(hi.y), "r"(hi.z),
                   "r"(hi.w) : "memory");
    }
  }
};

template <int MH>
__device__ __forceinline__ int total_tiles_grouped(const GemmParams& p) {
  int tot = 0;
  for (int g = 0; g < p.num_groups; ++g) {
    int o0, o1;
    group_rows(p, g, o0, o1);
    tot += ((o1 - o0 + MH - 1) / MH) * p.n_tiles;
  }
  return tot;
}

// grouped tile t -> (group, rows m0..m0+MH-1 clipped at m_end, output columns n0..)
template <int MH, int BN_OUT>
__device__ __forceinline__ void decode_tile_grouped(const GemmParams& p, int t, TileInfo& ti) {
  for (int g = 0; g < p.num_groups; ++g) {
    int o0, o1;
    group_rows(p, g, o0, o1);
    const int mt = (o1 - o0 + MH - 1) / MH;
    const int tg = mt * p.n_tiles;
    if (t < tg) {
      const int mb = t % mt, nb = t / mt;   // m fastest: neighbouring CTAs share the code tile in L2
      ti.m0 = o0 + mb * MH;
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

template <int EPI, int MT>
__global__ void __launch_bounds__(I8W_THREADS, 1)
gemm_i8w_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                const __grid_constant__ CUtensorMap tmQ2, const GemmParams p) {
  static_assert(EPI == EPI_SWIGLU || EPI == EPI_F32, "expert GEMMs only");
  static_assert(MT == 1 || MT == 2, "one or two 128-row halves per tile");
  using S = I8wSmem<MT>;
  constexpr int BN = I8W_BN;
  constexpr int BN_OUT = EPI == EPI_SWIGLU ? BN / 2 : BN;
  constexpr int MH = 128 * MT;
  constexpr int NBUF = 2 / MT;             // accumulator sets in TMEM (512 columns in all)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem + S::B_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + I8W_TSTAGES);
  const uint32_t bfull0 = smem_u32(bars + 2 * I8W_TSTAGES);
  const uint32_t bempty0 = smem_u32(bars + 2 * I8W_TSTAGES + I8W_BSTAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * I8W_TSTAGES + 2 * I8W_BSTAGES);
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tfull0 + 32;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * I8W_TSTAGES + 2 * I8W_BSTAGES + 5);
  static_assert(8 * (2 * I8W_TSTAGES + 2 * I8W_BSTAGES + 6) <= 256, "barrier slots");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < I8W_TSTAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < I8W_BSTAGES; ++s) {
      mbar_init(bfull0 + 8 * s, I8W_DQ_WARPS);
      mbar_init(bempty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, GEMM_EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
    tma_prefetch(&tmA);
    tma_prefetch(&tmQ);
    if (EPI == EPI_SWIGLU) tma_prefetch(&tmQ2);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  griddep_launch();
  griddep_wait();   // offsets and activations come from the previous kernels
  const int ntiles = total_tiles_grouped<MH>(p);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        TileInfo ti;
        decode_tile_grouped<MH, BN_OUT>(p, t, ti);
        const bool two = MT == 2 && ti.m0 + 128 < ti.m_end;
        for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          uint8_t* st = smem + stage * S::T_STAGE;
          mbar_arrive_tx(fb, (two ? 2 : 1) * S::A_BYTES + S::Q_BYTES);
          tma_load_2d(smem_u32(st), &tmA, fb, kt * 64, ti.m0);
          if (two) tma_load_2d(smem_u32(st + S::A_BYTES), &tmA, fb, kt * 64, ti.m0 + 128);
          const uint32_t q_dst = smem_u32(st + MT * S::A_BYTES);
          if constexpr (EPI == EPI_SWIGLU) {
            tma_load_3d(q_dst, &tmQ, fb, kt * 64, ti.n0, ti.group);
            tma_load_3d(q_dst + (BN / 2) * 64, &tmQ2, fb, kt * 64, ti.n0, ti.group);
          } else {
            tma_load_3d(q_dst, &tmQ, fb, kt * 64, ti.n0, ti.group);
          }
          if (++stage == I8W_TSTAGES) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, BN);
      int ts = 0, bs = 0;
      uint32_t tph = 0, bph = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        TileInfo ti;
        decode_tile_grouped<MH, BN_OUT>(p, t, ti);
        const bool two = MT == 2 && ti.m0 + 128 < ti.m_end;
        const int buf = it % NBUF;
        const uint32_t use = (uint32_t)(it / NBUF);
        if (!mbar_wait(tempty0 + 8 * buf, (use & 1) ^ 1, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tbase + buf * BN;   // MT = 2: buf is 0, the halves use columns 0 and 256
        for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
          if (!mbar_wait(full0 + 8 * ts, tph, p.err)) { ok = false; break; }
          if (!mbar_wait(bfull0 + 8 * bs, bph, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint8_t* st = smem + ts * S::T_STAGE;
          const uint64_t bd = sw128_desc(smem_u32(sB + bs * S::B_BYTES));
          const uint64_t ad0 = sw128_desc(smem_u32(st));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d0, ad0 + 2 * kk, bd + 2 * kk, IDESC, (kt > ti.kt0 || kk > 0) ? 1u : 0u);
          if (two) {
            const uint64_t ad1 = sw128_desc(smem_u32(st + S::A_BYTES));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(d0 + BN, ad1 + 2 * kk, bd + 2 * kk, IDESC, (kt > ti.kt0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(empty0 + 8 * ts);
          umma_commit(bempty0 + 8 * bs);
          if (++ts == I8W_TSTAGES) { ts = 0; tph ^= 1; }
          if (++bs == I8W_BSTAGES) { bs = 0; bph ^= 1; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * buf);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else if (warp >= 2 + GEMM_EPI_WARPS) {
    const WidenPlanLinear<BN> plan(threadIdx.x - 32 * (2 + GEMM_EPI_WARPS));
    const uint32_t qbase = smem_u32(smem + MT * S::A_BYTES), bbase = smem_u32(sB);
    int ts = 0, bs = 0;
    uint32_t tph = 0, bph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      TileInfo ti;
      decode_tile_grouped<MH, BN_OUT>(p, t, ti);
      for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
        if (!mbar_wait_warp(full0 + 8 * ts, tph, p.err)) { ok = false; break; }
        if (!mbar_wait_warp(bempty0 + 8 * bs, bph ^ 1, p.err)) { ok = false; break; }
        plan.run(qbase + ts * S::T_STAGE, bbase + bs * S::B_BYTES);
        fence_async_shared();   // the tensor core reads these stores through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(bfull0 + 8 * bs);
        if (++ts == I8W_TSTAGES) { ts = 0; tph ^= 1; }
        if (++bs == I8W_BSTAGES) { bs = 0; bph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;       // which of the two warps of this quarter
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      TileInfo ti;
      decode_tile_grouped<MH, BN_OUT>(p, t, ti);
      const bool two = MT == 2 && ti.m0 + 128 < ti.m_end;
      const int buf = it % NBUF;
      const uint32_t use = (uint32_t)(it / NBUF);
      if (!mbar_wait_warp(tfull0 + 8 * buf, use & 1, p.err)) break;
      tc_fence_after();
      const float* sc = p.scale_b + (long long)ti.group * p.N;
      for (int h = 0; h < (two ? 2 : 1); ++h) {
        const int m = ti.m0 + h * 128 + q * 32 + lane;
        const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + buf * BN + h * BN;
        if constexpr (EPI == EPI_F32) {
#pragma unroll 1
          for (int j = half; j < BN / 32; j += 2) {
            float v[32];
            tmem_ld32(tl + j * 32, v);
            tmem_wait_ld();
            scale32(v, sc, ti.n0 + j * 32, p.N);
            epi_chunk<EPI_F32, false, 32>(p, ti, m, ti.n0 + j * 32, v);
          }
        } else {
          const float* sc2 = p.scale_b2 + (long long)ti.group * p.N;
          bf16* o = reinterpret_cast<bf16*>(p.out) + (long long)m * p.ldo;
#pragma unroll 1
          for (int j = half; j < BN / 64; j += 2) {
            float g[32], u[32];
            tmem_ld32(tl + j * 32, g);
            tmem_ld32(tl + BN / 2 + j * 32, u);
            tmem_wait_ld();
            if (m < ti.m_end) {
              const int n = ti.n0 + j * 32;
              scale32(g, sc, n, p.N);
              scale32(u, sc2, n, p.N);
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// Few routed rows per expert (decode batches): weights on the M side.
//
//   D[f, m] = sum_k w[g, f, k] * A[m, k]  for 128 weight rows f and BNT rows m
//
// The widened weight tile is the MMA's A operand and a BNT-row activation tile
// its B operand (M = 128, N = BNT), so the tensor core does no work for empty
// rows and the shared memory goes to a deep ring of code tiles: this mode is
// bound by streaming the codes from HBM.  Code tiles are 128 codes deep
// (128-byte rows, 128-byte swizzle): TMA moves whole 128-byte lines, and each
// ring stage feeds two 64-deep MMA steps.  The epilogue writes the transpose
// (consecutive lanes are consecutive weight rows, so stores stay coalesced).
// SwiGLU holds the gate and up rows f in two accumulators.
constexpr int I8T_BNT = 32;
constexpr int I8T_EPI_WARPS = 4;   // one per TMEM lane quarter: a 32-token tile is one chunk
// Dequantiser warps: two groups that widen alternate 64-deep halves of the
// code stages, each group one warp per TMEM lane quarter per 128-row tile
// (gate and up: two tiles).
template <int EPI> constexpr int i8t_dq_warps() { return EPI == EPI_SWIGLU ? 16 : 8; }
template <int EPI> constexpr int i8t_threads() { return 32 * (2 + I8T_EPI_WARPS + i8t_dq_warps<EPI>()); }

// The widened weights never touch shared memory: the dequantiser warps write
// them into tensor memory (tcgen05.st, one weight row per TMEM lane) and the
// MMA takes its A operand from there, so shared memory carries only the codes
// (1 byte per weight) and the activations.
template <int EPI>
struct I8tSmem {
  static constexpr int QROWS = EPI == EPI_SWIGLU ? 256 : 128;     // gate + up, or down rows
  static constexpr uint32_t X_SUB = I8T_BNT * 128;                  // BNT x 64 bf16 activations
  static constexpr uint32_t X_BYTES = 2 * X_SUB;                    // two 64-deep steps per stage
  static constexpr uint32_t Q_BYTES = QROWS * 128;                  // QROWS x 128 codes
  static constexpr uint32_t T_STAGE = X_BYTES + Q_BYTES;            // a multiple of 1024
  static constexpr int TSTAGES = EPI == EPI_SWIGLU ? 5 : 8;
  static constexpr int BSTAGES = 4;                                 // widened 64-deep steps in TMEM
  static constexpr uint32_t BAR_OFF = TSTAGES * T_STAGE;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
  static constexpr int ACC = EPI == EPI_SWIGLU ? 2 * I8T_BNT : I8T_BNT;   // TMEM columns per accumulator
  static constexpr int A_COLS = (QROWS / 128) * 32;                 // widened 128 x 64 tiles, 32 columns each
  static constexpr int A_OFF = 2 * ACC;                             // after the two accumulators
  static constexpr int USED = A_OFF + BSTAGES * A_COLS;
  static constexpr uint32_t TMEM_COLS = USED <= 32 ? 32 : USED <= 64 ? 64 : USED <= 128 ? 128 : USED <= 256 ? 256 : 512;
  static_assert(USED <= 512, "tensor memory");
};

// tile t -> (group, token rows m0.. clipped at m_end, weight rows n0..n0+127,
// k-split); with p.splits > 1 (fp32 output only) split s covers 64-deep steps
// [s k_tiles_per_split, (s + 1) k_tiles_per_split) and writes its partial sums
// at out + s split_stride
__device__ __forceinline__ int total_tiles_tok(const GemmParams& p) {
  int tot = 0;
  for (int g = 0; g < p.num_groups; ++g) {
    int o0, o1;
    group_rows(p, g, o0, o1);
    tot += ((o1 - o0 + I8T_BNT - 1) / I8T_BNT) * p.n_tiles * p.splits;
  }
  return tot;
}
__device__ __forceinline__ void decode_tile_tok(const GemmParams& p, int t, TileInfo& ti) {
  for (int g = 0; g < p.num_groups; ++g) {
    int o0, o1;
    group_rows(p, g, o0, o1);
    const int nt = (o1 - o0 + I8T_BNT - 1) / I8T_BNT;
    const int tg = nt * p.n_tiles * p.splits;
    if (t < tg) {
      // token tiles of one weight tile are neighbours, then its k-splits
      const int tb = t % nt, r = t / nt, sp = r % p.splits, wb = r / p.splits;
      ti.m0 = o0 + tb * I8T_BNT;
      ti.m_end = o1;
      ti.n0 = wb * 128;
      ti.kt0 = sp * p.k_tiles_per_split;    // 64-deep steps, even counts here
      ti.kt1 = min(p.k_tiles, ti.kt0 + p.k_tiles_per_split);
      ti.group = p.group_mod > 0 ? g % p.group_mod : g;
      ti.split = sp;
      return;
    }
    t -= tg;
  }
  ti.m0 = ti.m_end = ti.n0 = ti.kt0 = ti.kt1 = ti.group = ti.split = 0;
}

template <int EPI>
__global__ void __launch_bounds__(i8t_threads<EPI>(), 1)
gemm_i8w_tok_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmQ2, const GemmParams p) {
  static_assert(EPI == EPI_SWIGLU || EPI == EPI_F32, "expert GEMMs only");
  using S = I8tSmem<EPI>;
  constexpr int BNT = I8T_BNT;
  constexpr int TST = S::TSTAGES;
  constexpr int BST = S::BSTAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + TST);
  const uint32_t bfull0 = smem_u32(bars + 2 * TST);
  const uint32_t bempty0 = smem_u32(bars + 2 * TST + BST);
  const uint32_t tfull0 = smem_u32(bars + 2 * TST + 2 * BST);
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tfull0 + 32;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * TST + 2 * BST + 5);
  static_assert(8 * (2 * TST + 2 * BST + 6) <= 256, "barrier slots");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < TST; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int s = 0; s < BST; ++s) {
      mbar_init(bfull0 + 8 * s, i8t_dq_warps<EPI>() / 2);   // one group widens each half-stage
      mbar_init(bempty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, I8T_EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
    tma_prefetch(&tmA);
    tma_prefetch(&tmQ);
    if (EPI == EPI_SWIGLU) tma_prefetch(&tmQ2);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), S::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  griddep_launch();
  griddep_wait();
  const int ntiles = total_tiles_tok(p);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        TileInfo ti;
        decode_tile_tok(p, t, ti);
        for (int kt = ti.kt0; kt < ti.kt1; kt += 2) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t st = smem_u32(smem + stage * S::T_STAGE);
          mbar_arrive_tx(fb, S::T_STAGE);
          tma_load_2d(st, &tmA, fb, kt * 64, ti.m0);
          tma_load_2d(st + S::X_SUB, &tmA, fb, kt * 64 + 64, ti.m0);
          tma_load_3d(st + S::X_BYTES, &tmQ, fb, kt * 64, ti.n0, ti.group);
          if constexpr (EPI == EPI_SWIGLU)
            tma_load_3d(st + S::X_BYTES + 128 * 128, &tmQ2, fb, kt * 64, ti.n0, ti.group);
          if (++stage == TST) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, BNT);
      int ts = 0, bs = 0;
      uint32_t tph = 0, bph = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        TileInfo ti;
        decode_tile_tok(p, t, ti);
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!mbar_wait(tempty0 + 8 * buf, (use & 1) ^ 1, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tbase + buf * S::ACC;
        for (int kt = ti.kt0; kt < ti.kt1 && ok; kt += 2) {
          if (!mbar_wait(full0 + 8 * ts, tph, p.err)) { ok = false; break; }
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(bfull0 + 8 * bs, bph, p.err)) { ok = false; break; }
            tc_fence_after();
            const uint64_t xd = sw128_desc(smem_u32(smem + ts * S::T_STAGE + h * S::X_SUB));
            const uint32_t wa = tbase + S::A_OFF + bs * S::A_COLS;   // widened weights in TMEM
            const uint32_t acc0 = (kt > ti.kt0 || h > 0) ? 1u : 0u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) umma_bf16_ta(d0, wa + 8 * kk, xd + 2 * kk, IDESC, (acc0 || kk > 0) ? 1u : 0u);
            if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16_ta(d0 + BNT, wa + 32 + 8 * kk, xd + 2 * kk, IDESC, (acc0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(bempty0 + 8 * bs);
            if (++bs == BST) { bs = 0; bph ^= 1; }
          }
          if (!ok) break;
          umma_commit(empty0 + 8 * ts);
          if (++ts == TST) { ts = 0; tph ^= 1; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * buf);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else if (warp >= 2 + I8T_EPI_WARPS) {
    // Dequantiser warps in two groups: group h widens the h-th 64-deep half of
    // every code stage, so consecutive halves are widened concurrently.
    // Within a group, warp w takes TMEM lane quarter q = w & 3 (thread `lane`
    // widens row 32 q + lane of a 128-row weight tile; gate and up: the
    // group's two warps of a quarter take one tile each) and stores the row's
    // 64 widened codes with one tcgen05.st into its lane.  Codes sit in
    // 128-byte rows under the 128-byte swizzle (16-byte chunk c of row r at
    // r * 128 + ((c ^ (r & 7)) << 4)): eight consecutive rows read eight
    // distinct chunk positions, so a quarter-warp's loads are conflict-free.
    constexpr int DQ = i8t_dq_warps<EPI>();
    constexpr bool SW = EPI == EPI_SWIGLU;
    const int d = warp - 2 - I8T_EPI_WARPS;           // 0 .. DQ-1
    const int h = d / (DQ / 2);                         // which half this warp's group widens
    const int tile = SW ? (d % (DQ / 2)) >> 2 : 0;      // gate (0) or up (1) tile
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t row_off = (uint32_t)(tile * 128 + r) * 128;
    const uint32_t qbase = smem_u32(smem + S::X_BYTES) + row_off;
    const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + S::A_OFF + tile * 32;
    int ts = 0, k = h;                                  // k: this group's half-stages, 2 j + h
    uint32_t tph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      TileInfo ti;
      decode_tile_tok(p, t, ti);
      for (int kt = ti.kt0; kt < ti.kt1 && ok; kt += 2) {
        if (!mbar_wait_warp(full0 + 8 * ts, tph, p.err)) { ok = false; break; }
        const int bs = k % BST;
        const uint32_t bph = (uint32_t)(k / BST) & 1u;
        if (!mbar_wait_warp(bempty0 + 8 * bs, bph ^ 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qs = qbase + ts * S::T_STAGE;
        uint32_t wv[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = 4 * h + i;
          uint4 v, lo, hi;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(qs + ((c ^ (r & 7)) << 4)));
          widen16(v, lo, hi);
          wv[8 * i] = lo.x; wv[8 * i + 1] = lo.y; wv[8 * i + 2] = lo.z; wv[8 * i + 3] = lo.w;
          wv[8 * i + 4] = hi.x; wv[8 * i + 5] = hi.y; wv[8 * i + 6] = hi.z; wv[8 * i + 7] = hi.w;
        }
        tmem_st32u(tl + bs * S::A_COLS, wv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bfull0 + 8 * bs);
        k += 2;
        if (++ts == TST) { ts = 0; tph ^= 1; }
      }
    }
  } else {
    const int q = warp & 3;                // warps 2-5: TMEM lane quarters 2, 3, 0, 1
    int it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      TileInfo ti;
      decode_tile_tok(p, t, ti);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      if (!mbar_wait_warp(tfull0 + 8 * buf, use & 1, p.err)) break;
      tc_fence_after();
      const int f = ti.n0 + q * 32 + lane;   // weight row (output column); N is a multiple of 128
      const uint32_t tl = tbase + ((uint32_t)(q * 32) << 16) + buf * S::ACC;
      const float s1 = __ldg(p.scale_b + (long long)ti.group * p.N + f);
#pragma unroll 1
      for (int j = 0; j < BNT / 32; ++j) {
        float v[32];
        tmem_ld32(tl + j * 32, v);
        if constexpr (EPI == EPI_SWIGLU) {
          float u[32];
          tmem_ld32(tl + BNT + j * 32, u);
          tmem_wait_ld();
          const float s2 = __ldg(p.scale_b2 + (long long)ti.group * p.N + f);
          bf16* o = reinterpret_cast<bf16*>(p.out) + f;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int m = ti.m0 + j * 32 + c;
            if (m < ti.m_end) o[(long long)m * p.ldo] = __float2bfloat16_rn(silu(v[c] * s1) * (u[c] * s2));
          }
        } else {
          tmem_wait_ld();
          float* o = reinterpret_cast<float*>(p.out) + ti.split * p.split_stride + f;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int m = ti.m0 + j * 32 + c;
            if (m < ti.m_end) o[(long long)m * p.ldo] = v[c] * s1;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, S::TMEM_COLS);
  }
}

}  // namespace jb
