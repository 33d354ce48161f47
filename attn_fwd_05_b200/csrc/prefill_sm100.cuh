// prefill_sm100.cuh — exact attention forward (prefill) for sm_100a.
//
// The method: O = softmax(scale * Q K^T + mask) V computed tile by tile with an online
// softmax (running row maximum and running sum of exponentials, earlier partial
// results rescaled when the maximum moves), so the N x N score matrix never leaves the
// chip.  Sources: polydesk.ai glossary "FlashAttention", sections "Le goulot
// d'étranglement de l'attention standard" (the formula) and "L'idée clé :
// IO-awareness" (tiling, online softmax and its rescaling correction); zimaspace.com,
// "Comment Flash Attention réduit-il le trafic mémoire lors de l'inférence locale ?",
// sections on tiles held on chip, the online softmax and kernel fusion (score, scale,
// mask, normalisation and value aggregation in one kernel).
//
// B200 design (not the pages' A100/H100 kernels):
//   * Q, K and V tiles are brought in by TMA into 128-byte-swizzled shared memory and
//     stream through a ring of stages guarded by mbarriers.
//   * One thread issues tcgen05 MMAs: S = Q K^T lands in tensor memory (TMEM); the
//     softmax warps read S from TMEM, write P (bf16) back over S, and the MMA
//     O += P V takes P straight from TMEM; O accumulates in TMEM.
//   * Kernel "pingpong" (d = 64 or 128): two 128-row Q tiles per CTA, each with its own
//     softmax warpgroup, so one tile's softmax overlaps the other tile's MMAs (the
//     FA4 page, section "Pipeline ping-pong avec double tuile Query", describes the same
//     idea for Blackwell).  TMEM: S0 | S1 | O0 | O1 = 128 + 128 + d + d columns.
//   * Kernel "single" (d = 256): one Q tile, S double-buffered in TMEM (64 + 64 columns)
//     next to O (256 columns), so the next S = Q K^T runs while the softmax works.
//   * The rescale of O is skipped unless a row maximum grows by more than 2^8; the
//     stale maximum stays exact because O and both row sums use the same reference.
//     O is normalised by the sum of the bf16-rounded P that actually multiplied V, and
//     the log-sum-exp uses the fp32 sum of the unrounded P.
#pragma once

#include "sm100_common.cuh"

namespace attn {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

struct FwdArgs {
  CUtensorMap tm_q;  // [B*Hq, Nq, d] bf16, box {64, 128, 1}
  CUtensorMap tm_k;  // [B*Hkv, Nk, d] bf16, box {64, BN, 1}
  CUtensorMap tm_v;
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk;
  int group;       // Hq / Hkv
  int causal;
  int o_f32;
  float scale_log2;  // scale * log2(e)
  int pair_heads;    // pingpong kernel: 1 = the two tiles are heads h, h+1 of one KV group
  int n_qtiles;      // ceil(Nq / 128)
  int n_units;
  uint64_t timeout_ns;
};

struct TileJob {
  int hq;    // query head
  int q0;    // first query row of the tile
  int rows;  // valid rows (0 if the tile lies past Nq)
  int nblk;  // KV blocks this tile visits
};

template <int BN>
__device__ __forceinline__ TileJob make_tile(const FwdArgs& a, int hq, int q0) {
  TileJob t;
  t.hq = hq;
  t.q0 = q0;
  if (q0 >= a.Nq) {
    t.rows = 0;
    t.nblk = 0;
    return t;
  }
  t.rows = min(128, a.Nq - q0);
  long long nkeys = a.Nk;
  if (a.causal) {
    // last visible key of the tile's last row: (q0 + rows - 1) + (Nk - Nq)
    long long last = (long long)q0 + t.rows - 1 + (long long)a.Nk - a.Nq;
    nkeys = last + 1;
    if (nkeys < 0) nkeys = 0;
    if (nkeys > a.Nk) nkeys = a.Nk;
  }
  t.nblk = (int)((nkeys + BN - 1) / BN);
  return t;
}

// Does block j of this tile contain a masked key for some row of the tile?
template <int BN>
__device__ __forceinline__ bool block_needs_mask(const FwdArgs& a, const TileJob& t, int j) {
  long long hi = (long long)(j + 1) * BN;  // one past the block's last key
  if (hi > a.Nk) return true;
  if (a.causal && hi - 1 > (long long)t.q0 + a.Nk - a.Nq) return true;
  return false;
}

// Largest visible key index for query row q (may be < 0: nothing visible).
__device__ __forceinline__ int row_key_limit(const FwdArgs& a, int q) {
  long long lim = a.Nk - 1;
  if (a.causal) {
    long long c = (long long)q + a.Nk - a.Nq;
    if (c < lim) lim = c;
  }
  if (lim < -1) lim = -1;
  return (int)lim;
}

template <int D, int BN>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t sQ, uint32_t sK) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, BN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t da = smem_desc_sw128(sQ + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
    const uint64_t db = smem_desc_sw128(sK + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16, 1024);
    mma_ss(s_tmem, da, db, idesc, kk > 0 ? 1u : 0u);
  }
}

template <int D, int BN>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t sV, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    const uint64_t db = smem_desc_sw128(sV + kk * (16 * 128), BN * 128, 1024);
    mma_ts(o_tmem, p_tmem + kk * 8, db, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// One softmax step for the calling thread's row over NCOL score columns held in TMEM.
// Writes the bf16 probabilities over the first NCOL/2 columns of the same TMEM block.
// Returns the factor the row's O accumulator must be multiplied by (1 when the
// reference maximum did not move).
template <int NCOL>
__device__ __forceinline__ float softmax_step(uint32_t s_taddr, bool masked, int col_limit, float sl2,
                                              float& m, float& l, float& lr) {
  static_assert(NCOL == 64 || NCOL == 128, "score block width");
  uint32_t r[NCOL];
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) tmem_ld32(s_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));

  float s[NCOL];
#pragma unroll
  for (int c = 0; c < NCOL; ++c) s[c] = __uint_as_float(r[c]);
  if (masked) {
#pragma unroll
    for (int c = 0; c < NCOL; ++c) s[c] = (c > col_limit) ? -INFINITY : s[c];
  }
  float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
  for (int c = 4; c < NCOL; c += 4) {
    mx0 = fmaxf(mx0, s[c]);
    mx1 = fmaxf(mx1, s[c + 1]);
    mx2 = fmaxf(mx2, s[c + 2]);
    mx3 = fmaxf(mx3, s[c + 3]);
  }
  const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
  float alpha = 1.0f;
  if (mx > m + kRescaleThreshold) {  // false while nothing is visible (mx = -inf)
    alpha = ex2(m - mx);             // 0 when m = -inf
    m = mx;
  }
  const float mu = (m == -INFINITY) ? 0.0f : m;

  uint32_t P[NCOL / 2];
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int i = 0; i < NCOL / 2; ++i) {
    const float p0 = ex2(fmaf(s[2 * i], sl2, -mu));
    const float p1 = ex2(fmaf(s[2 * i + 1], sl2, -mu));
    a0 += p0;
    a1 += p1;
    const uint32_t w = pack_bf16x2(p0, p1);
    P[i] = w;
    b0 += bf16lo_to_f32(w);
    b1 += bf16hi_to_f32(w);
  }
#pragma unroll
  for (int c = 0; c < NCOL / 64; ++c) tmem_st32(s_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&P[c * 32]));
  l = l * alpha + (a0 + a1);
  lr = lr * alpha + (b0 + b1);
  return alpha;
}

// Multiplies the calling thread's O row (D fp32 columns in TMEM) by alpha.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t o_taddr, float alpha) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(o_taddr + c * 32, r);
    tmem_ld_wait(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st32(o_taddr + c * 32, r);
  }
}

// Epilogue for one row: O / lr to global (bf16 or fp32) and the log-sum-exp.
template <int D>
__device__ __forceinline__ void store_row(const FwdArgs& a, uint32_t o_taddr, bool have_o, bool valid, int b,
                                          int hq, int q, float m, float l, float lr) {
  const float inv = lr > 0.f ? 1.0f / lr : 0.f;
  const size_t row = ((size_t)b * a.Hq + hq) * (size_t)a.Nq + (size_t)(valid ? q : 0);
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    if (have_o) {
      tmem_ld32(o_taddr + c * 32, r);
      tmem_ld_wait(r);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    if (valid) {
      if (a.o_f32) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + row * D + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                               __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + row * D + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv, __uint_as_float(r[8 * i + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv);
          dst[i] = w;
        }
      }
    }
  }
  if (valid && a.lse != nullptr) {
    a.lse[row] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

// ====================================================================================
// Kernel 1: two Q tiles per CTA (d = 64 or 128)
// ====================================================================================

template <int D>
struct PingPongCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int THREADS = 384;  // warp 0 TMA, warp 1 MMA, warps 4-7 and 8-11 softmax
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int NSTAGE = (D == 64) ? 8 : 4;  // K and V tiles share the ring
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NSTAGE * KV_BYTES;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;  // barriers + 1 KB alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
};

struct PingPongBars {
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(384, 1) attn_fwd_pingpong_kernel(const __grid_constant__ FwdArgs a) {
  using C = PingPongCfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PingPongBars* bars = reinterpret_cast<PingPongBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit (heaviest causal tiles first)
  int b, kvh;
  TileJob tj[2];
  {
    const int u = blockIdx.x;
    if (a.pair_heads) {
      const int per_level = a.B * (a.Hq / 2);
      const int qt = a.n_qtiles - 1 - u / per_level;
      const int rem = u % per_level;
      b = rem / (a.Hq / 2);
      const int h0 = 2 * (rem % (a.Hq / 2));
      tj[0] = make_tile<BN>(a, h0, qt * 128);
      tj[1] = make_tile<BN>(a, h0 + 1, qt * 128);
    } else {
      const int per_level = a.B * a.Hq;
      const int qp = (a.n_qtiles + 1) / 2 - 1 - u / per_level;
      const int rem = u % per_level;
      b = rem / a.Hq;
      const int h = rem % a.Hq;
      tj[0] = make_tile<BN>(a, h, (2 * qp) * 128);
      tj[1] = make_tile<BN>(a, h, (2 * qp + 1) * 128);
    }
    kvh = tj[0].hq / a.group;
  }
  const int nblk = max(tj[0].nblk, tj[1].nblk);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_done[t], 1);
    }
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ[2] = {smem_u32(smem + C::OFF_Q), smem_u32(smem + C::OFF_Q + C::Q_BYTES)};
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);

  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      tma_prefetch_map(&a.tm_q);
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
      for (int t = 0; t < 2; ++t) {
        if (tj[t].nblk == 0) continue;
        mbar_arrive_expect_tx(&bars->q_full[t], C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + c * (128 * 128), &a.tm_q, &bars->q_full[t], c * 64,
                      tj[t].q0, b * a.Hq + tj[t].hq);
      }
      const uint64_t pol = l2_policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        for (int kv = 0; kv < 2 && ok; ++kv, ++it) {
          const int st = it % C::NSTAGE;
          const int use = it / C::NSTAGE;
          if (use > 0 && !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, abort_flag, a.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->kv_full[st], C::KV_BYTES);
          const CUtensorMap* map = kv ? &a.tm_v : &a.tm_k;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_hint(smem + C::OFF_KV + st * C::KV_BYTES + c * (BN * 128), map, &bars->kv_full[st],
                             c * 64, j * BN, b * a.Hkv + kvh, pol);
        }
      }
      // drain: every copy issued must have landed before the CTA may exit
      for (int t = 0; t < 2; ++t)
        if (tj[t].nblk > 0) mbar_wait(&bars->q_full[t], 0, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < C::NSTAGE && st < it; ++st) {
        const int last_use = (it - 1 - st) / C::NSTAGE;  // index of the last fill of stage st
        mbar_wait(&bars->kv_full[st], last_use & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0 && nblk > 0) {
      bool ok = true;
      for (int t = 0; t < 2 && ok; ++t)
        if (tj[t].nblk > 0) ok = mbar_wait(&bars->q_full[t], 0, abort_flag, a.timeout_ns);
      auto stage_of = [&](int it) { return it % C::NSTAGE; };
      auto parity_of = [&](int it) { return (uint32_t)((it / C::NSTAGE) & 1); };
      // prologue: S_t(0)
      if (ok) ok = mbar_wait(&bars->kv_full[stage_of(0)], parity_of(0), abort_flag, a.timeout_ns);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t) {
          if (tj[t].nblk == 0) continue;
          issue_qk<D, BN>(tmem + (t ? C::COL_S1 : C::COL_S0), sQ[t], sKV + stage_of(0) * C::KV_BYTES);
          tc_commit(&bars->s_full[t]);
        }
        tc_commit(&bars->kv_empty[stage_of(0)]);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int itV = 2 * j + 1, itK = 2 * j + 2;
        if (!mbar_wait(&bars->kv_full[stage_of(itV)], parity_of(itV), abort_flag, a.timeout_ns)) break;
        const uint32_t sV = sKV + stage_of(itV) * C::KV_BYTES;
        const bool next = (j + 1 < nblk);
        bool k_ready = false;
        for (int t = 0; t < 2; ++t) {
          const uint32_t colS = t ? C::COL_S1 : C::COL_S0;
          const uint32_t colO = t ? C::COL_O1 : C::COL_O0;
          if (j < tj[t].nblk) {
            if (!mbar_wait(&bars->p_full[t], j & 1, abort_flag, a.timeout_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv<D, BN>(tmem + colO, tmem + colS, sV, j > 0);
            tc_commit(&bars->o_done[t]);
          }
          if (t == 1) tc_commit(&bars->kv_empty[stage_of(itV)]);
          if (next && j + 1 < tj[t].nblk) {
            if (!k_ready) {
              if (!mbar_wait(&bars->kv_full[stage_of(itK)], parity_of(itK), abort_flag, a.timeout_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
              k_ready = true;
            }
            issue_qk<D, BN>(tmem + colS, sQ[t], sKV + stage_of(itK) * C::KV_BYTES);
            tc_commit(&bars->s_full[t]);
          }
        }
        if (!ok) break;
        if (next) {
          if (!k_ready) {  // no tile used K(j+1) (cannot happen when next is true, kept for safety)
            if (!mbar_wait(&bars->kv_full[stage_of(itK)], parity_of(itK), abort_flag, a.timeout_ns)) break;
          }
          tc_commit(&bars->kv_empty[stage_of(itK)]);
        }
      }
      // every MMA must be finished before TMEM is released
      tc_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
    }
  } else if (warp >= 4) {
    // ================= softmax warpgroups: warps 4-7 own tile 0, warps 8-11 tile 1
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;       // row within the tile
    const TileJob& job = tj[t];
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (t ? C::COL_S1 : C::COL_S0);
    const uint32_t o_addr = tmem + lane_off + (t ? C::COL_O1 : C::COL_O0);
    const int q = job.q0 + r;
    const int klim = row_key_limit(a, q);
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int j = 0; j < job.nblk; ++j) {
      if (!mbar_wait(&bars->s_full[t], j & 1, abort_flag, a.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool masked = block_needs_mask<BN>(a, job, j);
      const float alpha = softmax_step<BN>(s_addr, masked, klim - j * BN, a.scale_log2, m, l, lr);
      if (__any_sync(0xffffffffu, alpha != 1.0f) && j > 0) {
        // O holds P V of blocks < j: wait for the last of those MMAs, then rescale
        if (!mbar_wait(&bars->o_done[t], (j - 1) & 1, abort_flag, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        rescale_o<D>(o_addr, alpha);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[t]);
    }
    bool have_o = job.nblk > 0;
    if (ok && have_o) {
      ok = mbar_wait(&bars->o_done[t], (job.nblk - 1) & 1, abort_flag, a.timeout_ns);
      tc_fence_after();
    }
    if (ok) store_row<D>(a, o_addr, have_o, r < job.rows, b, job.hq, q, m, l, lr);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ====================================================================================
// Kernel 2: one Q tile per CTA, S double-buffered (d = 256)
// ====================================================================================

template <int D>
struct SingleCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 64;
  static constexpr int THREADS = 256;  // warp 0 TMA, warp 1 MMA, warps 4-7 softmax
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int NSTAGE = 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NSTAGE * KV_BYTES;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 64, COL_O = 256;
};

struct SingleBars {
  uint64_t q_full;
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done;
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(256, 1) attn_fwd_single_kernel(const __grid_constant__ FwdArgs a) {
  using C = SingleCfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SingleBars* bars = reinterpret_cast<SingleBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int b, hq;
  TileJob job;
  {
    const int u = blockIdx.x;
    const int per_level = a.B * a.Hq;
    const int qt = a.n_qtiles - 1 - u / per_level;
    const int rem = u % per_level;
    b = rem / a.Hq;
    hq = rem % a.Hq;
    job = make_tile<BN>(a, hq, qt * 128);
  }
  const int kvh = hq / a.group;
  const int nblk = job.nblk;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);

  if (warp == 0) {
    if (lane == 0 && nblk > 0) {
      tma_prefetch_map(&a.tm_q);
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
      mbar_arrive_expect_tx(&bars->q_full, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d(smem + C::OFF_Q + c * (128 * 128), &a.tm_q, &bars->q_full, c * 64, job.q0, b * a.Hq + hq);
      const uint64_t pol = l2_policy_evict_last();
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int st = it % C::NSTAGE;
          const int use = it / C::NSTAGE;
          if (use > 0 && !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, abort_flag, a.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->kv_full[st], C::KV_BYTES);
          const CUtensorMap* map = kv ? &a.tm_v : &a.tm_k;
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d_hint(smem + C::OFF_KV + st * C::KV_BYTES + c * (BN * 128), map, &bars->kv_full[st],
                             c * 64, j * BN, b * a.Hkv + kvh, pol);
        }
      }
      mbar_wait(&bars->q_full, 0, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < C::NSTAGE && st < it; ++st) {
        const int last_use = (it - 1 - st) / C::NSTAGE;
        mbar_wait(&bars->kv_full[st], last_use & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nblk > 0) {
      auto stage_of = [&](int it) { return it % C::NSTAGE; };
      auto parity_of = [&](int it) { return (uint32_t)((it / C::NSTAGE) & 1); };
      auto colS = [&](int j) { return (j & 1) ? C::COL_S1 : C::COL_S0; };
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, a.timeout_ns);
      // S(0) and S(1) up front
      for (int j = 0; j < 2 && j < nblk && ok; ++j) {
        const int itK = 2 * j;
        if (!mbar_wait(&bars->kv_full[stage_of(itK)], parity_of(itK), abort_flag, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_qk<D, BN>(tmem + colS(j), sQ, sKV + stage_of(itK) * C::KV_BYTES);
        tc_commit(&bars->s_full[j & 1]);
        tc_commit(&bars->kv_empty[stage_of(itK)]);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const int itV = 2 * j + 1;
        if (!mbar_wait(&bars->kv_full[stage_of(itV)], parity_of(itV), abort_flag, a.timeout_ns)) break;
        if (!mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, abort_flag, a.timeout_ns)) break;
        tc_fence_after();
        issue_pv<D, BN>(tmem + C::COL_O, tmem + colS(j), sKV + stage_of(itV) * C::KV_BYTES, j > 0);
        tc_commit(&bars->o_done);
        tc_commit(&bars->kv_empty[stage_of(itV)]);
        if (j + 2 < nblk) {
          const int itK = 2 * (j + 2);
          if (!mbar_wait(&bars->kv_full[stage_of(itK)], parity_of(itK), abort_flag, a.timeout_ns)) break;
          tc_fence_after();
          issue_qk<D, BN>(tmem + colS(j), sQ, sKV + stage_of(itK) * C::KV_BYTES);
          tc_commit(&bars->s_full[j & 1]);
          tc_commit(&bars->kv_empty[stage_of(itK)]);
        }
      }
      tc_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + C::COL_O;
    const int q = job.q0 + r;
    const int klim = row_key_limit(a, q);
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      if (!mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, a.timeout_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_off + ((j & 1) ? C::COL_S1 : C::COL_S0);
      const bool masked = block_needs_mask<BN>(a, job, j);
      const float alpha = softmax_step<BN>(s_addr, masked, klim - j * BN, a.scale_log2, m, l, lr);
      if (__any_sync(0xffffffffu, alpha != 1.0f) && j > 0) {
        if (!mbar_wait(&bars->o_done, (j - 1) & 1, abort_flag, a.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        rescale_o<D>(o_addr, alpha);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[j & 1]);
    }
    const bool have_o = nblk > 0;
    if (ok && have_o) {
      ok = mbar_wait(&bars->o_done, (nblk - 1) & 1, abort_flag, a.timeout_ns);
      tc_fence_after();
    }
    if (ok) store_row<D>(a, o_addr, have_o, r < job.rows, b, hq, q, m, l, lr);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Writes O = 0 and lse = -inf for every row (used when Nk == 0: no key is visible).
__global__ void attn_fwd_empty_kernel(void* o, float* lse, size_t rows, int d, int o_f32) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  const size_t n = rows * (size_t)d;
  for (size_t k = i; k < n; k += (size_t)gridDim.x * blockDim.x) {
    if (o_f32)
      reinterpret_cast<float*>(o)[k] = 0.f;
    else
      reinterpret_cast<__nv_bfloat16*>(o)[k] = __float2bfloat16(0.f);
  }
  if (lse != nullptr)
    for (size_t k = i; k < rows; k += (size_t)gridDim.x * blockDim.x) lse[k] = -INFINITY;
}

}  // namespace attn
