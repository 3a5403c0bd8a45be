// Grouped-query attention layer of the Jamba block.
//
// "Jamba: A Hybrid Transformer-Mamba Language Model" (summary page),
// section 2: one layer in eight is attention, of the standard kind with
// grouped-query attention; no explicit positional information is used (no
// positional embedding, no RoPE).  Query head h reads KV head h / (H / G);
// causal softmax of q . k / sqrt(head_dim).
//
// Prefill: the fused q|k|v projection is one tcgen05 GEMM ([T, (H + 2G) D]
// rows); the attention kernel reads its Q and K tiles in place from that
// buffer with TMA.  V is written transposed ([B*G*D, L]) by kv_prep_kernel so
// that P.V is a K-major product like every other operand here; the same
// kernel fills the KV cache.  flash_attn_kernel: one CTA per (sequence,
// query head, 128-query block), heavy (late) blocks first; per 128-key block
// S = Q K^T (tcgen05, fp32 in TMEM, double-buffered), an online softmax by
// eight warps (two threads per query row, 64 keys each, meeting in shared
// memory for the row maximum; the running maximum is raised lazily, only
// when a row's maximum grows by more than 2^8, and O is then rescaled in
// TMEM), P in bf16 through swizzled shared memory, O += P V (tcgen05, fp32
// in TMEM).  Every wait is bounded (see common.cuh).
//
// Decode: the new token's k and v are appended to the cache at the
// sequence's current length, then attn_decode_kernel splits the cached
// positions of each (sequence, KV head) over CTAs (all query heads of the
// group read each key and value once) and attn_combine_kernel merges the
// partial softmaxes and advances the lengths.  Bound by reading the cache.
#include "common.cuh"
#include "host.hpp"

namespace jb {

constexpr int ATT_D = 128;       // head width (the only one supported)
constexpr int ATT_BQ = 128;      // query rows per CTA
constexpr int ATT_BK = 128;      // keys per block
constexpr int ATT_KVST = 2;      // K / V^T ring stages
constexpr int ATT_SM_WARPS = 8;  // softmax: two warps per TMEM lane quarter, 64 keys each
constexpr int ATT_THREADS = 32 * (2 + ATT_SM_WARPS);

struct AttnSmem {
  static constexpr uint32_t SUB = 128 * 128;                 // 128 rows x 64 bf16, swizzled
  static constexpr uint32_t Q_OFF = 0;                       // Q: dims 0-63 | 64-127
  static constexpr uint32_t KV_OFF = 2 * SUB;                // per stage: K (dims) x2, V^T (keys) x2
  static constexpr uint32_t KV_STAGE = 4 * SUB;
  static constexpr uint32_t P_OFF = KV_OFF + ATT_KVST * KV_STAGE;   // P: keys 0-63 | 64-127
  static constexpr uint32_t RED_OFF = P_OFF + 2 * SUB;        // row maxima / sums exchanged by the two halves
  static constexpr uint32_t BAR_OFF = RED_OFF + 2 * 2 * 128 * 4;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};

// named barrier over the softmax warps only
__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * ATT_SM_WARPS) : "memory");
}

struct AttnParams {
  int B, L, H, G, rep, nq;
  bf16* o;
  long long ldo;
  float sl2;   // log2(e) / sqrt(head_dim)
  int* err;
};

__global__ void __launch_bounds__(ATT_THREADS, 1)
flash_attn_kernel(const __grid_constant__ CUtensorMap tmQK, const __grid_constant__ CUtensorMap tmVt,
                  const AttnParams p) {
  using S = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t q_full = smem_u32(bars);
  const uint32_t kv_full0 = smem_u32(bars + 1), kv_empty0 = smem_u32(bars + 3);
  const uint32_t s_full0 = smem_u32(bars + 5), s_free0 = smem_u32(bars + 7);
  const uint32_t p_full = smem_u32(bars + 9), pv_done = smem_u32(bars + 10), drain = smem_u32(bars + 11);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 12);

  const int bh = blockIdx.x % (p.B * p.H);
  const int qi = p.nq - 1 - (int)(blockIdx.x / (p.B * p.H));   // late query blocks (more keys) first
  const int b = bh / p.H, h = bh % p.H, g = h / p.rep;
  const int nkv = qi + 1;
  const int row0 = b * p.L + qi * ATT_BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_full0 + 8 * i, 1);
      mbar_init(kv_empty0 + 8 * i, 1);
      mbar_init(s_full0 + 8 * i, 1);
      mbar_init(s_free0 + 8 * i, ATT_SM_WARPS);
    }
    mbar_init(p_full, ATT_SM_WARPS);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
    tma_prefetch(&tmQK);
    tma_prefetch(&tmVt);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const uint32_t tS = tbase, tO = tbase + 256;   // S buffers at columns 0 and 128, O at 256
  griddep_launch();
  griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_tx(q_full, 2 * S::SUB);
      tma_load_2d(smem_u32(smem + S::Q_OFF), &tmQK, q_full, h * ATT_D, row0);
      tma_load_2d(smem_u32(smem + S::Q_OFF + S::SUB), &tmQK, q_full, h * ATT_D + 64, row0);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(kv_empty0 + 8 * st, ((j >> 1) & 1) ^ 1, p.err)) break;
        const uint32_t fb = kv_full0 + 8 * st;
        const uint32_t base = smem_u32(smem + S::KV_OFF + st * S::KV_STAGE);
        mbar_arrive_tx(fb, 4 * S::SUB);
        const int krow = b * p.L + j * ATT_BK, kcol = (p.H + g) * ATT_D, vrow = (b * p.G + g) * ATT_D;
        tma_load_2d(base, &tmQK, fb, kcol, krow);
        tma_load_2d(base + S::SUB, &tmQK, fb, kcol + 64, krow);
        tma_load_2d(base + 2 * S::SUB, &tmVt, fb, j * ATT_BK, vrow);
        tma_load_2d(base + 3 * S::SUB, &tmVt, fb, j * ATT_BK + 64, vrow);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, 128);
      const uint64_t qd[2] = {sw128_desc(smem_u32(smem + S::Q_OFF)), sw128_desc(smem_u32(smem + S::Q_OFF + S::SUB))};
      const uint64_t pd[2] = {sw128_desc(smem_u32(smem + S::P_OFF)), sw128_desc(smem_u32(smem + S::P_OFF + S::SUB))};
      // S = Q K^T over the head width: k-steps 0-3 in the first 64 dims, 4-7 in the second
      auto issue_s = [&](uint32_t d, int st) {
        const uint32_t base = smem_u32(smem + S::KV_OFF + st * S::KV_STAGE);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(d, qd[kk >> 2] + 2 * (kk & 3), sw128_desc(base + (kk >> 2) * S::SUB) + 2 * (kk & 3), IDESC,
                    kk > 0 ? 1u : 0u);
      };
      bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(kv_full0, 0, p.err);
      if (ok) {
        tc_fence_after();
        issue_s(tS, 0);
        umma_commit(s_full0);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv) {
          const int nb = (j + 1) & 1;
          if (!mbar_wait(s_free0 + 8 * nb, (((j + 1) >> 1) & 1) ^ 1, p.err)) break;
          if (!mbar_wait(kv_full0 + 8 * nb, ((j + 1) >> 1) & 1, p.err)) break;
          tc_fence_after();
          issue_s(tS + nb * 128, nb);
          umma_commit(s_full0 + 8 * nb);
        }
        if (!mbar_wait(p_full, j & 1, p.err)) break;
        tc_fence_after();
        // O += P V: keys 0-63 in the first P / V^T sub-tiles, 64-127 in the second
        const uint32_t vbase = smem_u32(smem + S::KV_OFF + (j & 1) * S::KV_STAGE + 2 * S::SUB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(tO, pd[kk >> 2] + 2 * (kk & 3), sw128_desc(vbase + (kk >> 2) * S::SUB) + 2 * (kk & 3), IDESC,
                    (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(kv_empty0 + 8 * (j & 1));
        umma_commit(pv_done);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    // softmax: query row r of this warp's TMEM lane quarter, keys half*64 .. half*64+63 of
    // each block (and the same 64 columns of O); the two halves of a row meet in shared memory
    const int q4 = warp & 3, half = (warp - 2) >> 2;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + S::RED_OFF);   // [2 parities][2 halves][128 rows]
    float m = 0.f, l = 0.f;
    bool ok = true;
    // After a failed wait the loop still runs to its end (on whatever the buffers hold), so
    // that every softmax warp reaches every named barrier; the error is already latched.
    for (int j = 0; j < nkv; ++j) {
      const int buf = j & 1;
      ok = mbar_wait_warp(s_full0 + 8 * buf, (j >> 1) & 1, p.err) && ok;
      tc_fence_after();
      float s[64];
      tmem_ld32(tS + lane_off + buf * 128 + half * 64, s);
      tmem_ld32(tS + lane_off + buf * 128 + half * 64 + 32, s + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free0 + 8 * buf);
      if (j == qi) {   // diagonal block: key c is visible to row r when c <= r
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (half * 64 + c > r) s[c] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mx8[t] = s[t];
#pragma unroll
      for (int c = 8; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      red[(buf * 2 + half) * 128 + r] = mx;
      softmax_sync();
      mx = fmaxf(mx, red[(buf * 2 + (half ^ 1)) * 128 + r]);   // finite: key 0 of the block is visible
      const float mnew = mx * p.sl2;
      float corr = 1.f;
      if (j == 0) {
        m = mnew;
      } else if (mnew > m + 8.f) {   // raise the reference only when the terms would exceed 2^8
        corr = ex2(m - mnew);
        m = mnew;
      }
      float sm8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        s[c] = ex2(fmaf(s[c], p.sl2, -m));
        sm8[c & 7] += s[c];
      }
      l = l * corr + (((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7])));
      if (j > 0) {
        // P_{j-1} and the O it fed are done: P may be overwritten and O rescaled
        ok = mbar_wait_warp(pv_done, (j - 1) & 1, p.err) && ok;
        tc_fence_after();
        if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float o[32];
            tmem_ld32(tO + lane_off + half * 64 + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] *= corr;
            tmem_st32(tO + lane_off + half * 64 + 32 * c, o);
          }
          tmem_wait_st();
        }
      }
      // P row r, keys half*64.. (bf16): sub-tile `half`, 16-byte chunk k of row r at (k ^ (r & 7))
      uint8_t* prow = smem + S::P_OFF + half * S::SUB + r * 128;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint4 u;
        __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t) hh[t] = __floats2bfloat162_rn(s[8 * k + 2 * t], s[8 * k + 2 * t + 1]);
        *reinterpret_cast<uint4*>(prow + ((k ^ (r & 7)) << 4)) = u;
      }
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // the row sum is split over the two halves (same reference m, same corrections); the
    // parity slot the last block did not use is free (its reads came before the last sync)
    const float lpart = l;
    const int fb = nkv & 1;
    red[(fb * 2 + half) * 128 + r] = lpart;
    softmax_sync();
    l = lpart + red[(fb * 2 + (half ^ 1)) * 128 + r];
    if (ok && mbar_wait_warp(pv_done, (nkv - 1) & 1, p.err)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const int row = qi * ATT_BQ + r;
      bf16* dst = p.o + (long long)(b * p.L + row) * p.ldo + h * ATT_D + half * 64;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float o[32];
        tmem_ld32(tO + lane_off + half * 64 + 32 * c, o);
        tmem_wait_ld();
        if (row < p.L) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 u;
            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int t = 0; t < 4; ++t) hh[t] = __floats2bfloat162_rn(o[8 * k + 2 * t] * inv, o[8 * k + 2 * t + 1] * inv);
            *reinterpret_cast<uint4*>(dst + 32 * c + 8 * k) = u;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// Two query heads of one KV group per CTA (used when the group size is even):
// tiles A and B share every K and V^T tile, and the tensor core alternates
// between them so that one tile's softmax runs while the other's products
// do.  MMA order per key block j: O_A += P_A V_j, S_A(j+1) = Q_A K_{j+1}^T,
// O_B += P_B V_j, S_B(j+1).  K_j and V^T_j are separate 32 KB items of a
// three-slot ring (K_0, V_0, K_1, V_1, ...).  Softmax: four warps per tile,
// thread = query row, the running maximum raised lazily as above.
constexpr int ATT2_THREADS = 320;   // producer, MMA, 4 + 4 softmax warps

struct Attn2Smem {
  static constexpr uint32_t SUB = 128 * 128;
  static constexpr uint32_t Q_OFF = 0;            // Q_A (2 sub-tiles), Q_B (2)
  static constexpr uint32_t P_OFF = 4 * SUB;      // P_A (2), P_B (2)
  static constexpr uint32_t KV_OFF = 8 * SUB;     // 3 slots x 2 sub-tiles
  static constexpr int SLOTS = 3;
  static constexpr uint32_t BAR_OFF = KV_OFF + SLOTS * 2 * SUB;
  static constexpr uint32_t BYTES = BAR_OFF + 256 + 1024;
};

__global__ void __launch_bounds__(ATT2_THREADS, 1)
flash_attn2_kernel(const __grid_constant__ CUtensorMap tmQK, const __grid_constant__ CUtensorMap tmVt,
                   const AttnParams p) {
  using S = Attn2Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BAR_OFF);
  const uint32_t q_full = smem_u32(bars);
  const uint32_t kv_full0 = smem_u32(bars + 1), kv_empty0 = smem_u32(bars + 4);
  // per tile t: s_full, s_free, p_full, pv_done at slots 7 + 4t ..
  const uint32_t tb0 = smem_u32(bars + 7);
  const uint32_t drain = smem_u32(bars + 15);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 16);
#define S_FULL(t) (tb0 + 32 * (t))
#define S_FREE(t) (tb0 + 32 * (t) + 8)
#define P_FULL(t) (tb0 + 32 * (t) + 16)
#define PV_DONE(t) (tb0 + 32 * (t) + 24)

  const int HP = p.H / 2;
  const int bp = blockIdx.x % (p.B * HP);
  const int qi = p.nq - 1 - (int)(blockIdx.x / (p.B * HP));
  const int b = bp / HP, h0 = 2 * (bp % HP), g = h0 / p.rep;
  const int nkv = qi + 1;
  const int row0 = b * p.L + qi * ATT_BQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < S::SLOTS; ++i) {
      mbar_init(kv_full0 + 8 * i, 1);
      mbar_init(kv_empty0 + 8 * i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(S_FULL(t), 1);
      mbar_init(S_FREE(t), 4);
      mbar_init(P_FULL(t), 4);
      mbar_init(PV_DONE(t), 1);
    }
    mbar_init(drain, 1);
    mbar_fence_init();
    tma_prefetch(&tmQK);
    tma_prefetch(&tmVt);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_holder), 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;   // tile t: S at 256 t, O at 256 t + 128
  griddep_launch();
  griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_tx(q_full, 4 * S::SUB);
      for (int t = 0; t < 2; ++t)
        for (int k = 0; k < 2; ++k)
          tma_load_2d(smem_u32(smem + S::Q_OFF + (2 * t + k) * S::SUB), &tmQK, q_full, (h0 + t) * ATT_D + 64 * k,
                      row0);
      const int kcol = (p.H + g) * ATT_D, vrow = (b * p.G + g) * ATT_D;
      for (int item = 0; item < 2 * nkv; ++item) {
        const int slot = item % S::SLOTS, j = item >> 1;
        if (!mbar_wait(kv_empty0 + 8 * slot, ((item / S::SLOTS) & 1) ^ 1, p.err)) break;
        const uint32_t fb = kv_full0 + 8 * slot;
        const uint32_t dst = smem_u32(smem + S::KV_OFF + slot * 2 * S::SUB);
        mbar_arrive_tx(fb, 2 * S::SUB);
        if ((item & 1) == 0) {   // K_j: keys 128j.., dims 0-63 | 64-127
          tma_load_2d(dst, &tmQK, fb, kcol, b * p.L + j * ATT_BK);
          tma_load_2d(dst + S::SUB, &tmQK, fb, kcol + 64, b * p.L + j * ATT_BK);
        } else {                 // V^T_j: dims 0-127, keys 128j.. | +64
          tma_load_2d(dst, &tmVt, fb, j * ATT_BK, vrow);
          tma_load_2d(dst + S::SUB, &tmVt, fb, j * ATT_BK + 64, vrow);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, 128);
      auto slot_of = [](int item) { return item % S::SLOTS; };
      auto ph_of = [](int item) { return (uint32_t)((item / S::SLOTS) & 1); };
      auto issue_s = [&](int t, int j) {
        const uint32_t kb = smem_u32(smem + S::KV_OFF + slot_of(2 * j) * 2 * S::SUB);
        const uint32_t qb = smem_u32(smem + S::Q_OFF + 2 * t * S::SUB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(tbase + 256 * t, sw128_desc(qb + (kk >> 2) * S::SUB) + 2 * (kk & 3),
                    sw128_desc(kb + (kk >> 2) * S::SUB) + 2 * (kk & 3), IDESC, kk > 0 ? 1u : 0u);
        umma_commit(S_FULL(t));
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t vb = smem_u32(smem + S::KV_OFF + slot_of(2 * j + 1) * 2 * S::SUB);
        const uint32_t pb = smem_u32(smem + S::P_OFF + 2 * t * S::SUB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16(tbase + 256 * t + 128, sw128_desc(pb + (kk >> 2) * S::SUB) + 2 * (kk & 3),
                    sw128_desc(vb + (kk >> 2) * S::SUB) + 2 * (kk & 3), IDESC, (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(PV_DONE(t));
      };
      bool ok = mbar_wait(q_full, 0, p.err) && mbar_wait(kv_full0 + 8 * slot_of(0), ph_of(0), p.err);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        umma_commit(kv_empty0 + 8 * slot_of(0));
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const uint32_t par = j & 1;
        const bool more = j + 1 < nkv;
        if (!mbar_wait(P_FULL(0), par, p.err) || !mbar_wait(kv_full0 + 8 * slot_of(2 * j + 1), ph_of(2 * j + 1), p.err)) break;
        tc_fence_after();
        issue_pv(0, j);
        if (more) {
          if (!mbar_wait(kv_full0 + 8 * slot_of(2 * j + 2), ph_of(2 * j + 2), p.err) ||
              !mbar_wait(S_FREE(0), par, p.err)) break;
          tc_fence_after();
          issue_s(0, j + 1);
        }
        if (!mbar_wait(P_FULL(1), par, p.err)) break;
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(kv_empty0 + 8 * slot_of(2 * j + 1));
        if (more) {
          if (!mbar_wait(S_FREE(1), par, p.err)) break;
          tc_fence_after();
          issue_s(1, j + 1);
          umma_commit(kv_empty0 + 8 * slot_of(2 * j + 2));
        }
      }
      umma_commit(drain);
      mbar_wait(drain, 0, p.err);
    }
  } else {
    // softmax of tile t (warps 2-5: head h0, warps 6-9: head h0 + 1); thread = query row r
    const int t = (warp - 2) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + 256 * t, tO = tS + 128;
    // One read of S per block in the common case: the terms are formed against the running
    // reference m while the block maximum is tracked; only when that maximum exceeds m by more
    // than 8 (log2 units; always for the first block) is the block read again with the new m.
    // The tensor core runs O += P V of the previous block before this block's S, so by the
    // time S is complete the shared P tile is free and P goes straight to it.
    float m = 0.f, l = 0.f;
    bool ok = true;
    uint8_t* prow = smem + S::P_OFF + 2 * t * S::SUB + r * 128;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait_warp(S_FULL(t), j & 1, p.err) && ok;
      if (j > 0) ok = mbar_wait_warp(PV_DONE(t), (j - 1) & 1, p.err) && ok;
      tc_fence_after();
      const bool diag = j == qi;   // key c visible to row r when c <= r
      float sum = 0.f;
      // form the terms against reference `ref` into the P tile; returns the block maximum
      auto pass = [&](float ref) {
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        float sm4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          float sv[64];
          tmem_ld32(tS + lane_off + 64 * c2, sv);
          tmem_ld32(tS + lane_off + 64 * c2 + 32, sv + 32);
          tmem_wait_ld();
          if (diag) {
#pragma unroll
            for (int k2 = 0; k2 < 64; ++k2)
              if (64 * c2 + k2 > r) sv[k2] = -INFINITY;
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {   // 16-byte chunk kc = 8 c2 + q: keys 8kc .. 8kc+7
            uint32_t w[4];
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2) {
              const float a = sv[8 * q + 2 * i2] * p.sl2, bb = sv[8 * q + 2 * i2 + 1] * p.sl2;
              mx4[i2] = fmaxf(mx4[i2], fmaxf(a, bb));
              const float ea = ex2(a - ref), eb = ex2(bb - ref);
              sm4[i2] += ea + eb;
              __nv_bfloat162 hh = __floats2bfloat162_rn(ea, eb);
              w[i2] = *reinterpret_cast<uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(prow + c2 * S::SUB + ((q ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        sum = (sm4[0] + sm4[1]) + (sm4[2] + sm4[3]);
        return fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      };
      float corr = 1.f;
      if (j == 0) {
        // first block: find the maximum, then form the terms against it
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float sv[32];
          tmem_ld32(tS + lane_off + 32 * c, sv);
          tmem_wait_ld();
#pragma unroll
          for (int k2 = 0; k2 < 32; ++k2) {
            const float v = (diag && 32 * c + k2 > r) ? -INFINITY : sv[k2];
            mx4[k2 & 3] = fmaxf(mx4[k2 & 3], v);
          }
        }
        m = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * p.sl2;
        pass(m);
      } else {
        const float mx = pass(m);
        const bool raise = mx > m + 8.f;
        // rare: raise the reference and form the block again.  The TMEM loads in pass() are
        // warp-collective, so the whole warp repeats it; rows that keep their reference
        // recompute the same terms.
        if (__any_sync(0xffffffffu, raise)) {
          if (raise) {
            corr = ex2(m - mx);
            m = mx;
          }
          pass(m);
        }
      }
      l = l * corr + sum;
      if (j > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tO + lane_off + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k2 = 0; k2 < 32; ++k2) o[k2] *= corr;
          tmem_st32(tO + lane_off + 32 * c, o);
        }
        tmem_wait_st();
      }
      fence_async_shared();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(S_FREE(t));   // S may be overwritten
        mbar_arrive(P_FULL(t));
      }
    }
    if (ok && mbar_wait_warp(PV_DONE(t), (nkv - 1) & 1, p.err)) {
      tc_fence_after();
      const float inv = 1.f / l;
      const int row = qi * ATT_BQ + r;
      bf16* dst = p.o + (long long)(b * p.L + row) * p.ldo + (h0 + t) * ATT_D;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tO + lane_off + 32 * c, o);
        tmem_wait_ld();
        if (row < p.L) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 u;
            __nv_bfloat162* hh = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) hh[i] = __floats2bfloat162_rn(o[8 * k + 2 * i] * inv, o[8 * k + 2 * i + 1] * inv);
            *reinterpret_cast<uint4*>(dst + 32 * c + 8 * k) = u;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}
#undef S_FULL
#undef S_FREE
#undef P_FULL
#undef PV_DONE

// qkv [B*L, W] (W = (H + 2G) D): V transposed into vt [B*G*D, ldv] (row
// (b, g, d), column = position) and, when given, K and V into the caches
// [B, G, max_len, D].  Block: one (sequence, KV head, 64 positions).
__global__ void __launch_bounds__(256)
kv_prep_kernel(const bf16* __restrict__ qkv, int L, int H, int G, bf16* __restrict__ vt, long long ldv,
               bf16* __restrict__ kc, bf16* __restrict__ vc, int max_len) {
  __shared__ bf16 tile[64][ATT_D + 8];
  griddep_wait();
  griddep_launch();
  const int bg = blockIdx.y, b = bg / G, g = bg % G;
  const int pos0 = blockIdx.x * 64;
  const long long W = (long long)(H + 2 * G) * ATT_D;
  // rows: 64 positions x 16 chunks of 8 values
  for (int i = threadIdx.x; i < 64 * 16; i += 256) {
    const int pr = i >> 4, ch = i & 15, pos = pos0 + pr;
    uint4 vv = make_uint4(0, 0, 0, 0);
    if (pos < L) {
      const bf16* row = qkv + (long long)(b * L + pos) * W;
      vv = *reinterpret_cast<const uint4*>(row + (long long)(H + G + g) * ATT_D + ch * 8);
      if (kc) {
        const uint4 kv = *reinterpret_cast<const uint4*>(row + (long long)(H + g) * ATT_D + ch * 8);
        const long long o = (((long long)b * G + g) * max_len + pos) * ATT_D + ch * 8;
        *reinterpret_cast<uint4*>(kc + o) = kv;
        *reinterpret_cast<uint4*>(vc + o) = vv;
      }
    }
    *reinterpret_cast<uint4*>(&tile[pr][ch * 8]) = vv;
  }
  __syncthreads();
  // columns: 128 dims x 64 positions, two positions per thread-step
  for (int i = threadIdx.x; i < ATT_D * 32; i += 256) {
    const int d = i >> 5, pp = (i & 31) * 2, pos = pos0 + pp;
    if (pos < L) {
      bf16* dst = vt + ((long long)bg * ATT_D + d) * ldv + pos;
      dst[0] = tile[pp][d];
      if (pos + 1 < L) dst[1] = tile[pp + 1][d];
    }
  }
}

jamba_status attn_prefill_core(const void* qkv, void* vt, long long ldv, void* o, void* k_cache, void* v_cache,
                               int max_len, int B, int L, int H, int G, cudaStream_t s) {
  const int W = (H + 2 * G) * ATT_D;
  if ((long long)B * G > 65535) return fail(JAMBA_ERR_UNSUPPORTED, "attention prefill: batch * n_kv_heads above 65535");
  JB_CUDA(launch_pdl(kv_prep_kernel, dim3((L + 63) / 64, B * G), dim3(256), 0, s,
                     reinterpret_cast<const bf16*>(qkv), L, H, G, reinterpret_cast<bf16*>(vt), ldv,
                     reinterpret_cast<bf16*>(k_cache), reinterpret_cast<bf16*>(v_cache), max_len));
  CUtensorMap mqk, mvt;
  JB_TRY(make_map_2d(&mqk, qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)W, (uint64_t)B * L, (uint64_t)W * 2,
                     64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
  JB_TRY(make_map_2d(&mvt, vt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)L, (uint64_t)B * G * ATT_D,
                     (uint64_t)ldv * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
  AttnParams p;
  p.B = B;
  p.L = L;
  p.H = H;
  p.G = G;
  p.rep = H / G;
  p.nq = (L + ATT_BQ - 1) / ATT_BQ;
  p.o = reinterpret_cast<bf16*>(o);
  p.ldo = (long long)H * ATT_D;
  p.sl2 = 1.4426950408889634f / sqrtf((float)ATT_D);
  p.err = device_error_word();
  if (!p.err) return fail(JAMBA_ERR_CUDA, "could not allocate the device status word");
  static std::atomic<bool> configured[64];
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(flash_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)AttnSmem::BYTES));
    JB_CUDA(cudaFuncSetAttribute(flash_attn2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Attn2Smem::BYTES));
    configured[dev] = true;
  }
  if (p.rep % 2 == 0) {   // pairs of query heads stay inside one KV group
    JB_CUDA(launch_pdl(flash_attn2_kernel, dim3((unsigned)(B * (H / 2) * p.nq)), dim3(ATT2_THREADS),
                       Attn2Smem::BYTES, s, mqk, mvt, p));
  } else {
    JB_CUDA(launch_pdl(flash_attn_kernel, dim3((unsigned)(B * H * p.nq)), dim3(ATT_THREADS), AttnSmem::BYTES, s,
                       mqk, mvt, p));
  }
  return JAMBA_OK;
}

// ---------------------------------------------------------------- decode

// qkv [B, W]: k and v of the new token into the caches at position lengths[b]
__global__ void __launch_bounds__(256)
kv_append_kernel(const bf16* __restrict__ qkv, int H, int G, const int* __restrict__ lengths, bf16* __restrict__ kc,
                 bf16* __restrict__ vc, int max_len, int* err) {
  griddep_wait();
  griddep_launch();
  const int b = blockIdx.x;
  const int pos = lengths[b];
  // out-of-range lengths append nothing (and are reported by the checked build)
  if (!checked(pos >= 0 && pos < max_len, err) || pos < 0 || pos >= max_len) return;
  const long long W = (long long)(H + 2 * G) * ATT_D;
  for (int i = threadIdx.x; i < G * 16; i += 256) {
    const int g = i >> 4, ch = i & 15;
    const bf16* row = qkv + b * W;
    const long long o = (((long long)b * G + g) * max_len + pos) * ATT_D + ch * 8;
    *reinterpret_cast<uint4*>(kc + o) = *reinterpret_cast<const uint4*>(row + (long long)(H + g) * ATT_D + ch * 8);
    *reinterpret_cast<uint4*>(vc + o) =
        *reinterpret_cast<const uint4*>(row + (long long)(H + G + g) * ATT_D + ch * 8);
  }
}

constexpr int DEC_REP = 8;   // query heads per KV head the decode kernel takes at most (the padded N of its tiles)

// One CTA of four warps per (sequence, KV head, split of the positions
// 0..lengths[b]): for each of the group's query heads, the partial
// softmax (max, sum, weighted sum of values) over its positions.  A warp takes
// 16 positions at a time: their key and value rows are copied into shared
// memory (cp.async, 16 bytes per copy, two buffers so the next rows stream in
// while these are used; rows padded to 272 bytes so ldmatrix reads hit 32
// distinct banks), then two tensor-core products per 16 positions
// (mma.sync m16n8k16, bf16 in, fp32 out):
//   S^T = K Q^T   positions on M, the group's query heads (up to 8; padded to 8) on N,
//                 head width as K;
//   O^T += V^T P^T   head width on M (8 tiles of 16), heads on N, positions as K
//                    (V^T through ldmatrix .trans).
// In the S^T layout lane (g, t) holds positions g and g + 8 of heads 2t and
// 2t + 1, which is also where O^T keeps those heads, so the running maximum,
// sum and rescaling of a head stay in its lanes; the softmax reduces over
// positions with three shuffles.  P^T's fragment is gathered with eight.
constexpr int DEC_PITCH = 272;                     // bytes per staged row (256 + 16)
constexpr int DEC_TILE = 16 * DEC_PITCH;           // 16 rows
constexpr uint32_t DEC_SMEM = 4 * 2 * 2 * DEC_TILE;   // warps x buffers x (K, V)

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// 16 bytes global -> shared; src_bytes 0 writes zeros (the source is not read)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(128)
attn_decode_kernel(const bf16* __restrict__ qkv, int H, int G, const int* __restrict__ lengths,
                   const bf16* __restrict__ kc, const bf16* __restrict__ vc, int max_len, int splits, float sl2,
                   float* __restrict__ part) {
  extern __shared__ uint8_t dsm[];
  __shared__ float w_m[4][DEC_REP], w_l[4][DEC_REP];
  __shared__ float w_o[4][DEC_REP][ATT_D];
  const int rep = H / G;   // query heads of the group: 1 .. DEC_REP
  griddep_wait();
  griddep_launch();
  const int bg = blockIdx.x, b = bg / G, g = bg % G, split = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;   // mma fragment coordinates
  const int n = max(0, min(lengths[b] + 1, max_len));   // the appended token included; never past the cache
  const int per = (n + splits - 1) / splits;
  const int p0 = split * per, p1 = min(n, p0 + per);
  const long long W = (long long)(H + 2 * G) * ATT_D;
  // B fragments of Q^T (k = head dims, n = head gq; heads 4-7 are zero padding)
  uint32_t qb[8][2];
  {
    const bf16* qrow = qkv + b * W + (long long)(g * rep + (gq < rep ? gq : 0)) * ATT_D;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t lo = 0, hi = 0;
      if (gq < rep) {
        lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * tq);
        hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * tq + 8);
      }
      qb[kk][0] = lo;
      qb[kk][1] = hi;
    }
  }
  const bf16* kbase = kc + ((long long)b * G + g) * max_len * ATT_D;
  const bf16* vbase = vc + ((long long)b * G + g) * max_len * ATT_D;
  const uint32_t wbase = smem_u32(dsm) + warp * 2 * 2 * DEC_TILE;   // [buffer][K, V]
  // stage 16 rows of K and V at positions c0.. into buffer `buf` (zeros past p1)
  auto stage = [&](int c0, int buf) {
    const uint32_t kd = wbase + buf * 2 * DEC_TILE, vd = kd + DEC_TILE;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = lane + 32 * i;          // 16 rows x 16 pieces of 16 bytes
      const int row = idx >> 4, piece = idx & 15;
      const int pos = c0 + row;
      const bool in = pos < p1;
      const long long off = (long long)(in ? pos : 0) * ATT_D + piece * 8;
      cp_async16(kd + row * DEC_PITCH + piece * 16, kbase + off, in ? 16 : 0);
      cp_async16(vd + row * DEC_PITCH + piece * 16, vbase + off, in ? 16 : 0);
    }
    cp_async_commit();
  };
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // heads 2tq, 2tq + 1
  float acc[8][4];
#pragma unroll
  for (int mm = 0; mm < 8; ++mm) acc[mm][0] = acc[mm][1] = acc[mm][2] = acc[mm][3] = 0.f;
  const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: matrix and row this lane addresses
  int c0 = p0 + warp * 16, buf = 0;
  if (c0 < p1) stage(c0, 0);
  for (; c0 < p1; c0 += 64, buf ^= 1) {
    if (c0 + 64 < p1) {
      stage(c0 + 64, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const uint32_t kt = wbase + buf * 2 * DEC_TILE, vt = kt + DEC_TILE;
    // S^T = K Q^T: [16 positions x 8 heads]
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t a[4];
      ldsm_x4(a, kt + (rr + 8 * (mi & 1)) * DEC_PITCH + (16 * kk + 8 * (mi >> 1)) * 2);
      mma_bf16_16816(sc, a, qb[kk][0], qb[kk][1]);
    }
    // online softmax per head (lane-local heads 2tq, 2tq + 1; positions gq and gq + 8)
    const bool in0 = c0 + gq < p1, in8 = c0 + gq + 8 < p1;
    float pr[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float s0 = in0 ? sc[e] * sl2 : -INFINITY, s8 = in8 ? sc[2 + e] * sl2 : -INFINITY;
      float mx = fmaxf(s0, s8);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[e], mx);                  // finite: position c0 is valid
      const float corr = ex2(m[e] - mn);                 // 0 when m was -inf
      pr[e] = ex2(s0 - mn);
      pr[2 + e] = ex2(s8 - mn);
      float sum = pr[e] + pr[2 + e];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      l[e] = l[e] * corr + sum;
      m[e] = mn;
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        acc[mm][e] *= corr;
        acc[mm][2 + e] *= corr;
      }
    }
    // P^T fragment: (positions 2tq, 2tq+1 | 2tq+8, 2tq+9; head gq) from the lanes holding them
    uint32_t pb0, pb1;
    {
      const int srcA = (2 * tq) * 4 + (gq >> 1), srcB = (2 * tq + 1) * 4 + (gq >> 1);
      const bool odd = gq & 1;
      float v[4];
      const float a0 = __shfl_sync(0xffffffffu, pr[0], srcA), a1 = __shfl_sync(0xffffffffu, pr[1], srcA);
      const float b0 = __shfl_sync(0xffffffffu, pr[0], srcB), b1 = __shfl_sync(0xffffffffu, pr[1], srcB);
      const float a2 = __shfl_sync(0xffffffffu, pr[2], srcA), a3 = __shfl_sync(0xffffffffu, pr[3], srcA);
      const float b2 = __shfl_sync(0xffffffffu, pr[2], srcB), b3 = __shfl_sync(0xffffffffu, pr[3], srcB);
      v[0] = odd ? a1 : a0;   // position 2tq
      v[1] = odd ? b1 : b0;   // position 2tq + 1
      v[2] = odd ? a3 : a2;   // position 2tq + 8
      v[3] = odd ? b3 : b2;   // position 2tq + 9
      __nv_bfloat162 h01 = __floats2bfloat162_rn(v[0], v[1]), h23 = __floats2bfloat162_rn(v[2], v[3]);
      pb0 = *reinterpret_cast<uint32_t*>(&h01);
      pb1 = *reinterpret_cast<uint32_t*>(&h23);
    }
    // O^T += V^T P^T: 8 tiles of 16 head dims
#pragma unroll
    for (int mm = 0; mm < 8; ++mm) {
      uint32_t a[4];
      ldsm_x4_t(a, vt + (rr + 8 * (mi >> 1)) * DEC_PITCH + (16 * mm + 8 * (mi & 1)) * 2);
      mma_bf16_16816(acc[mm], a, pb0, pb1);
    }
    __syncwarp();   // this buffer is refilled two groups later
  }
  // merge the four warps, then write this split's partial per query head
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int hq = 2 * tq + e;
    if (hq < rep) {
      if (gq == 0) {
        w_m[warp][hq] = m[e];
        w_l[warp][hq] = l[e];
      }
#pragma unroll
      for (int mm = 0; mm < 8; ++mm) {
        w_o[warp][hq][16 * mm + gq] = acc[mm][e];
        w_o[warp][hq][16 * mm + gq + 8] = acc[mm][2 + e];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < rep * ATT_D; i += 128) {
    const int h = i / ATT_D, d = i % ATT_D;
    float mm = -INFINITY;
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, w_m[w][h]);
    float ls = 0.f, os = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = w_m[w][h] == -INFINITY ? 0.f : ex2(w_m[w][h] - mm);
      ls += w_l[w][h] * f;
      os += w_o[w][h][d] * f;
    }
    // part layout: [B*H][splits][D + 2]: o (unnormalised), then max (log2 units), sum
    float* dst = part + ((long long)(b * H + g * rep + h) * splits + split) * (ATT_D + 2);
    dst[d] = os;
    if (d == 0) {
      dst[ATT_D] = mm;
      dst[ATT_D + 1] = ls;
    }
  }
}

// o[b, h*D + d] = sum over splits, normalised; then lengths[b] += 1
__global__ void __launch_bounds__(128)
attn_combine_kernel(const float* __restrict__ part, int H, int splits, bf16* __restrict__ o, int* __restrict__ lengths) {
  griddep_wait();
  griddep_launch();
  const int bh = blockIdx.x, d = threadIdx.x;
  const float* src = part + (long long)bh * splits * (ATT_D + 2);
  float mm = -INFINITY;
  for (int s = 0; s < splits; ++s) mm = fmaxf(mm, src[s * (ATT_D + 2) + ATT_D]);
  float ls = 0.f, os = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ms = src[s * (ATT_D + 2) + ATT_D];
    const float f = ms == -INFINITY ? 0.f : ex2(ms - mm);
    ls += src[s * (ATT_D + 2) + ATT_D + 1] * f;
    os += src[s * (ATT_D + 2) + d] * f;
  }
  o[(long long)bh * ATT_D + d] = __float2bfloat16_rn(os / ls);
  __syncthreads();
  if (d == 0 && bh % H == 0) lengths[bh / H] += 1;
}

int attn_decode_splits(int B, int G, int max_len) {
  // enough CTAs for ~16 per SM over the run (three are resident at a time),
  // so the last wave is a small part of the whole
  const int ctas = B * G;
  int s = (16 * num_sms() + ctas - 1) / ctas;
  const int cap = (max_len + 255) / 256;   // at least 256 positions per split
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  return s;
}

jamba_status attn_decode_core(const void* qkv, void* k_cache, void* v_cache, int max_len, int* lengths, float* part,
                              int splits, void* o, int B, int H, int G, cudaStream_t s) {
  if (splits > 65535) return fail(JAMBA_ERR_UNSUPPORTED, "attention step: too many position splits");
  if (H / G > DEC_REP) return fail(JAMBA_ERR_UNSUPPORTED, "attention step: at most 8 query heads per KV head");
  JB_CUDA(launch_pdl(kv_append_kernel, dim3(B), dim3(256), 0, s, reinterpret_cast<const bf16*>(qkv), H, G,
                     (const int*)lengths, reinterpret_cast<bf16*>(k_cache), reinterpret_cast<bf16*>(v_cache),
                     max_len, device_error_word()));
  const float sl2 = 1.4426950408889634f / sqrtf((float)ATT_D);
  static std::atomic<bool> configured[64];
  int dev = 0;
  JB_CUDA(cudaGetDevice(&dev));
  if (dev < 64 && !configured[dev]) {
    JB_CUDA(cudaFuncSetAttribute(attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DEC_SMEM));
    configured[dev] = true;
  }
  JB_CUDA(launch_pdl(attn_decode_kernel, dim3(B * G, splits), dim3(128), DEC_SMEM, s, reinterpret_cast<const bf16*>(qkv),
                     H, G, (const int*)lengths, reinterpret_cast<const bf16*>(k_cache),
                     reinterpret_cast<const bf16*>(v_cache), max_len, splits, sl2, part));
  JB_CUDA(launch_pdl(attn_combine_kernel, dim3(B * H), dim3(ATT_D), 0, s, (const float*)part, H, splits,
                     reinterpret_cast<bf16*>(o), lengths));
  return JAMBA_OK;
}

}  // namespace jb
