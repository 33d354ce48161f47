// backward_sm100.cuh — gradients of exact attention (the backward pass) for sm_100a.
//
// The method: the forward pass never stores the score matrix; the backward pass
// recomputes it block by block from Q, K and the saved log-sum-exp (patricehuetz.fr,
// "Flash Attention : pourquoi ton GPU utilise 85% de VRAM", section "Ce que fait Flash
// Attention", second idea).  With P = exp(scale Q K^T - LSE) recomputed per block and
// Delta = rowsum(dO o O):
//     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// B200 design: three kernels, no atomics.
//   * delta kernel: one warp per query row, Delta in fp32.
//   * dK/dV kernel: one CTA per (batch, KV head, 128-key tile).  It walks the query
//     heads of the KV head's group and the q-tiles that see its keys, and keeps dK and
//     dV for its keys in TMEM for the whole walk (the group's sum comes for free):
//     S^T = K Q^T and dP^T = V dO^T land in TMEM (one thread per key row), the thread
//     writes P^T and dS^T back over them as bf16, and dV += P^T dO, dK += dS^T Q run
//     with A from TMEM.  Q and dO tiles stream through a two-stage TMA ring.
//   * dQ kernel: one CTA per (batch, query head, 128-row q-tile).  It walks the K/V
//     tiles its rows see: S = Q K^T and dP = dO V^T in TMEM (one thread per query row),
//     dS written back over S, dQ += dS K with A from TMEM.
//   S and dP are computed by both kernels (the dQ pass repeats two of the five
//   products) in exchange for no atomic accumulation.
//   TMEM per CTA: S, dP (128 columns each) and the accumulators (d columns each).
// Causal masking uses the forward's bottom-right alignment: key j is visible to query i
// iff j <= i + (Nk - Nq).  d = 64 or 128.
#pragma once

#include "sm100_common.cuh"

namespace attn {

struct BwdArgs {
  CUtensorMap tm_q;   // [B*Hq, Nq, d] bf16, box {64, 128, 1}
  CUtensorMap tm_do;  // same layout as Q
  CUtensorMap tm_k;   // [B*Hkv, Nk, d] bf16, box {64, 128, 1}
  CUtensorMap tm_v;
  CUtensorMap tm_dq;   // fp32 [B*Hq, Nq, d], box {32, 32, 1}: the gradients leave through TMA stores
  CUtensorMap tm_dk;   // fp32 [B*Hkv, Nk, d], same boxes
  CUtensorMap tm_dv;
  const float* lse;    // [B*Hq, Nq] natural log-sum-exp of the forward pass
  const float* delta;  // [B*Hq, Nq] rowsum(dO o O)
  float* dq;           // [B*Hq, Nq, d]
  float* dk;           // [B*Hkv, Nk, d]
  float* dv;           // [B*Hkv, Nk, d]
  int B, Hq, Hkv, Nq, Nk, group, causal, n_qtiles, n_ktiles;
  float scale, scale_log2;
  uint64_t timeout_ns;
};

// The log-sum-exp in log2 units, with +inf for rows that must give P = 0 (outside the
// sequence, or no visible key: LSE = -inf).
__device__ __forceinline__ float lse2_of(const BwdArgs& a, size_t bh, int q) {
  if (q >= a.Nq) return INFINITY;
  const float l = __ldg(&a.lse[bh * a.Nq + q]);
  return (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
}

// ---------------------------------------------------------------------------- delta

template <int D>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                             const __nv_bfloat16* __restrict__ dout,
                                                             float* __restrict__ delta, long long rows) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nwarps) {
    const __nv_bfloat162* po = reinterpret_cast<const __nv_bfloat162*>(o + r * D);
    const __nv_bfloat162* pd = reinterpret_cast<const __nv_bfloat162*>(dout + r * D);
    float acc = 0.f;
#pragma unroll
    for (int c = lane; c < D / 2; c += 32) {
      const float2 x = __bfloat1622float2(po[c]);
      const float2 y = __bfloat1622float2(pd[c]);
      acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) delta[r] = acc;
  }
}

// ------------------------------------------------------------------- shared pieces

// One 32-column chunk of a probability / gradient row: p = 2^(s sl2 - L2) where the
// column is visible, ds = p (dp - dl); both packed to bf16 pairs.
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[32], const uint32_t (&dp)[32], float sl2,
                                          const float* L2, const float* dl, int vis_lo, int vis_hi, uint32_t (&P)[16],
                                          uint32_t (&dS)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float p[2], g[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int c = i + e;
      const bool vis = c >= vis_lo && c <= vis_hi;
      const float y = fmaf(__uint_as_float(s[c]), sl2, -L2[c]);
      p[e] = vis ? ex2(y) : 0.f;
      g[e] = p[e] * (__uint_as_float(dp[c]) - dl[c]);
    }
    P[i / 2] = pack_bf16x2(p[0], p[1]);
    dS[i / 2] = pack_bf16x2(g[0], g[1]);
  }
}

// D accumulator columns of this thread's row from TMEM, times `mul`, to a global fp32
// row (or zeros when the row got no work).
template <int D>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, bool have, bool valid, float mul, float* dst) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    if (have) {
      tmem_ld32(taddr + c * 32, r);
      tmem_ld_wait(r);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    if (valid) {
      float4* out = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        out[i] = make_float4(__uint_as_float(r[4 * i]) * mul, __uint_as_float(r[4 * i + 1]) * mul,
                             __uint_as_float(r[4 * i + 2]) * mul, __uint_as_float(r[4 * i + 3]) * mul);
    }
  }
}

// Columns [C0, C0 + NC) of this thread's fp32 accumulator row r (times mul), written to
// the calling warp's rows of a staging area in the layout of TMA's 128-byte swizzled fp32
// boxes, and stored from there with TMA: chunk i (32 columns, 128 bytes a row) of 128 rows
// sits at stage + i * 16 KB, and row r's 16-byte granule g at g ^ (r % 8).  A warp store
// then writes whole rows instead of touching 32 rows per instruction.  Rows at or past
// n_rows are clipped by the tensor map; the warp stores nothing if it has none below it.
template <int C0, int NC>
__device__ __forceinline__ void store_acc_tma(uint32_t stage, int r, uint32_t taddr, bool have, float mul,
                                              const CUtensorMap* map, int row0, int n_rows, int plane) {
  const int lane = threadIdx.x & 31;
  const int quad = r >> 5;
#pragma unroll
  for (int c = C0 / 32; c < (C0 + NC) / 32; ++c) {
    uint32_t v[32];
    if (have) {
      tmem_ld32(taddr + c * 32, v);
      tmem_ld_wait(v);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0u;
    }
    const uint32_t row = stage + (uint32_t)((c - C0 / 32) * (128 * 128) + r * 128);
#pragma unroll
    for (int g = 0; g < 8; ++g)
      st_shared_v4(row + (uint32_t)((g ^ (r & 7)) << 4), __float_as_uint(__uint_as_float(v[4 * g]) * mul),
                   __float_as_uint(__uint_as_float(v[4 * g + 1]) * mul),
                   __float_as_uint(__uint_as_float(v[4 * g + 2]) * mul),
                   __float_as_uint(__uint_as_float(v[4 * g + 3]) * mul));
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && row0 + quad * 32 < n_rows) {
#pragma unroll
    for (int c = C0 / 32; c < (C0 + NC) / 32; ++c)
      tma_store_3d(map, stage + (uint32_t)((c - C0 / 32) * (128 * 128) + quad * 32 * 128), c * 32, row0 + quad * 32,
                   plane);
    bulk_commit();
    bulk_wait_all();  // the CTA exits next: the stores must have read shared memory
  }
  __syncwarp();
}

struct BwdBars {
  uint64_t fixed_full;  // the CTA's own tiles (K and V, or Q and dO) have landed
  uint64_t stage_full[2];
  uint64_t stage_empty[2];
  uint64_t s_full[2];   // half h of the step's two score-like products is in TMEM
  uint64_t p_full[2];   // P and/or dS of half h written back (4 warps)
  uint64_t o_final;     // the last accumulation is done
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
struct BwdCfg {
  // warp 0 TMA, 1 MMA, 2-3 statistics (dK/dV kernel), 4-7 and 8-11 the elementwise pass
  // of query (dK/dV) or key (dQ) half 0 and half 1 of each step
  static constexpr int THREADS = 384;
  static constexpr int T = 128;  // rows of every tile
  static constexpr int TILE_BYTES = T * D * 2;
  static constexpr int OFF_FIXED = 0;                       // two tiles
  static constexpr int OFF_RING = 2 * TILE_BYTES;           // 2 stages x two tiles
  static constexpr int OFF_STAT = OFF_RING + 4 * TILE_BYTES;  // dK/dV kernel: [stage][L2 | delta][128]
  static constexpr int OFF_BAR = OFF_STAT + 2 * 2 * 128 * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + 1 KB alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  // S and dP in two 64-column halves each (half h at +64h), then the accumulators
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_ACC0 = 256, COL_ACC1 = 256 + D;
  static constexpr int HALF_ROWS_BYTES = 64 * 128;  // offset of rows 64.. inside a 64-column chunk
};

__device__ __forceinline__ void bwd_init_bars(BwdBars* bars, int stage_full_count) {
  mbar_init(&bars->fixed_full, 1);
  for (int s = 0; s < 2; ++s) {
    mbar_init(&bars->stage_full[s], stage_full_count);
    mbar_init(&bars->stage_empty[s], 1);
  }
  for (int h = 0; h < 2; ++h) {
    mbar_init(&bars->s_full[h], 1);
    mbar_init(&bars->p_full[h], 4);
  }
  mbar_init(&bars->o_final, 1);
  mbar_init(&bars->drain, 1);
  bars->abort_flag = 0;
  fence_mbar_init();
}

// ----------------------------------------------------------------------- dK / dV

// Steps of a dK/dV CTA: (query head of the group, q-tile), q-tiles from qt_lo on.
__device__ __forceinline__ int kv_qt_lo(const BwdArgs& a, int kt) {
  if (!a.causal) return 0;
  const long long x = (long long)kt * 128 - (a.Nk - a.Nq);  // earliest query that sees key kt*128
  if (x <= 0) return 0;
  const long long t = x / 128;
  return t < a.n_qtiles ? (int)t : a.n_qtiles;
}

template <int D>
__global__ void __launch_bounds__(384, 1) attn_bwd_dkdv_kernel(const __grid_constant__ BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  float* stat = reinterpret_cast<float*>(smem + C::OFF_STAT);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // causal: the first K/V tiles are seen by the most q-tiles, so they go first (longest
  // processing time first); consecutive CTAs share a key-tile index
  const int kt = blockIdx.x / (a.B * a.Hkv);
  const int bkv = blockIdx.x % (a.B * a.Hkv);  // b * Hkv + kvh
  const int b = bkv / a.Hkv, kvh = bkv % a.Hkv;
  const int k0 = kt * 128;
  const int qt_lo = kv_qt_lo(a, kt);
  const int nqt = a.n_qtiles - qt_lo;
  const int nsteps = a.group * nqt;
  auto step_bh = [&](int j) { return (size_t)b * a.Hq + (size_t)kvh * a.group + j / nqt; };
  auto step_q0 = [&](int j) { return (qt_lo + j % nqt) * 128; };

  if (threadIdx.x == 0) bwd_init_bars(bars, 3);  // TMA + the two stats warps
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sK = smem_u32(smem + C::OFF_FIXED), sV = sK + C::TILE_BYTES;
  const uint32_t sRing = smem_u32(smem + C::OFF_RING);

  if (warp == 0) {
    // ================= TMA: K and V of the tile once, then Q and dO of every step
    if (lane == 0) {
      tma_prefetch_map(&a.tm_q);
      tma_prefetch_map(&a.tm_do);
      mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + C::OFF_FIXED + c * (128 * 128), &a.tm_k, &bars->fixed_full, c * 64, k0, bkv);
        tma_load_3d(smem + C::OFF_FIXED + C::TILE_BYTES + c * (128 * 128), &a.tm_v, &bars->fixed_full, c * 64, k0,
                    bkv);
      }
      int j = 0;
      for (; j < nsteps; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&bars->stage_empty[st], ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns)) break;
        mbar_arrive_expect_tx(&bars->stage_full[st], 2 * C::TILE_BYTES);
        uint8_t* dst = smem + C::OFF_RING + st * 2 * C::TILE_BYTES;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(dst + c * (128 * 128), &a.tm_q, &bars->stage_full[st], c * 64, step_q0(j), (int)step_bh(j));
          tma_load_3d(dst + C::TILE_BYTES + c * (128 * 128), &a.tm_do, &bars->stage_full[st], c * 64, step_q0(j),
                      (int)step_bh(j));
        }
      }
      // drain: the copies in flight must land before the CTA exits
      mbar_wait(&bars->fixed_full, 0, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < 2 && st < j; ++st) {
        const int last = j - 1 - ((j - 1 - st) & 1);  // last step that used stage st
        mbar_wait(&bars->stage_full[st], (last >> 1) & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ================= per step: L2 (log-sum-exp in log2 units) and Delta of its 128 queries
    const int t = threadIdx.x - 64;  // 0..63
    for (int j = 0; j < nsteps; ++j) {
      const int st = j & 1;
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->stage_empty[st], ((j >> 1) - 1) & 1, abort_flag,
                                                       a.timeout_ns)))
        break;
      const size_t bh = step_bh(j);
      const int q0 = step_q0(j);
      float* L2 = stat + st * 256;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = t + 64 * h;
        const int q = q0 + c;
        L2[c] = lse2_of(a, bh, q);
        L2[128 + c] = (q < a.Nq) ? __ldg(&a.delta[bh * a.Nq + q]) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->stage_full[st]);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (whole warp, one elected lane issues)
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
    };
    if (nsteps > 0) {
      const Desc dk = desc_sw128(sK, 16, 1024), dvk = desc_sw128(sV, 16, 1024);
      // Each step is split in two halves of 64 queries, so that the softmax warps work on
      // one half while the tensor core computes the other:
      //   S^T_h = K Q_h^T, dP^T_h = V dO_h^T  (64 columns each), then after p_full[h]
      //   dV += P^T_h dO_h, dK += dS^T_h Q_h  (contraction over the half's 64 queries).
      // The next step's half h overwrites P_h / dS_h only after those products were
      // issued (this thread issues in order).
      auto stage_q = [&](int j) { return sRing + (j & 1) * 2 * C::TILE_BYTES; };
      auto issue_s = [&](int j, int h) {
        const uint32_t sQ = stage_q(j) + h * C::HALF_ROWS_BYTES, sDO = sQ + C::TILE_BYTES;
        if (elect_one()) {
          tc_fence_after();
          issue_qk_rows<D, 64>(tmem + C::COL_S + 64 * h, dk, desc_sw128(sQ, 16, 1024));
          issue_qk_rows<D, 64>(tmem + C::COL_DP + 64 * h, dvk, desc_sw128(sDO, 16, 1024));
          tc_commit(&bars->s_full[h]);
        }
        __syncwarp();
      };
      auto issue_acc = [&](int j, int h) {
        const uint32_t sQ = stage_q(j) + h * C::HALF_ROWS_BYTES, sDO = sQ + C::TILE_BYTES;
        const bool acc = j > 0 || h > 0;
        if (elect_one()) {
          tc_fence_after();
          issue_pv_ts_w<D, 64>(tmem + C::COL_ACC1, tmem + C::COL_S + 64 * h, desc_sw128(sDO, 128 * 128, 1024), acc);
          issue_pv_ts_w<D, 64>(tmem + C::COL_ACC0, tmem + C::COL_DP + 64 * h, desc_sw128(sQ, 128 * 128, 1024), acc);
        }
        __syncwarp();
      };
      bool ok = wait_all(&bars->fixed_full, 0) && wait_all(&bars->stage_full[0], 0);
      if (ok) {
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int j = 0; j < nsteps && ok; ++j) {
        const bool more = j + 1 < nsteps;
        if (!wait_all(&bars->p_full[0], j & 1)) break;
        issue_acc(j, 0);
        if (more) {
          if (!wait_all(&bars->stage_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) break;
          issue_s(j + 1, 0);
        }
        if (!wait_all(&bars->p_full[1], j & 1)) break;
        issue_acc(j, 1);
        if (elect_one()) {
          tc_commit(&bars->stage_empty[j & 1]);  // Q, dO and the statistics of step j
          if (!more) tc_commit(&bars->o_final);
        }
        __syncwarp();
        if (more) issue_s(j + 1, 1);
      }
      if (elect_one()) tc_commit(&bars->drain);
      __syncwarp();
      mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
    }
  } else {
    // ================= warps 4-7 (half 0) and 8-11 (half 1): one key row per thread, the
    // half's 64 query columns of every step
    const int h = warp >= 8 ? 1 : 0;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int k = k0 + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S, tDP = tmem + lane_off + C::COL_DP;
    const int off = a.Nk - a.Nq;
    bool ok = true;
    for (int j = 0; j < nsteps && ok; ++j) {
      const int st = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->stage_full[st], (j >> 1) & 1, abort_flag, a.timeout_ns))) {
        ok = false;
        break;
      }
      const float* L2 = stat + st * 256;
      // visible query columns of this key row: q >= k - off (causal)
      const int lo = a.causal ? k - off - step_q0(j) : -1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[h], j & 1, abort_flag, a.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * h + 32 * cc;  // first query column of the chunk
        uint32_t sv[32], dp[32], P[16], dS[16];
        tmem_ld32(tS + c0, sv);
        tmem_ld32(tDP + c0, dp);
        tmem_ld_wait(sv);
        tmem_ld_wait(dp);
        bwd_chunk(sv, dp, a.scale_log2, L2 + c0, L2 + 128 + c0, lo - c0, 31, P, dS);
        tmem_st16(tS + 64 * h + 16 * cc, P);  // packed over the half's columns already read
        tmem_st16(tDP + 64 * h + 16 * cc, dS);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[h]);
    }
    ok = __all_sync(0xffffffffu, ok);
    const bool have = nsteps > 0;
    if (ok && have) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0, abort_flag, a.timeout_ns));
      tc_fence_after();
    }
    if (ok) {  // half 0's warps write dK, half 1's dV, each staged in one ring stage (free now)
      const uint32_t stage = sRing + (uint32_t)(h * 2 * C::TILE_BYTES);
      if (h == 0)
        store_acc_tma<0, D>(stage, r, tmem + lane_off + C::COL_ACC0, have, a.scale, &a.tm_dk, k0, a.Nk, bkv);
      else
        store_acc_tma<0, D>(stage, r, tmem + lane_off + C::COL_ACC1, have, 1.0f, &a.tm_dv, k0, a.Nk, bkv);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------- dQ

template <int D>
__global__ void __launch_bounds__(384, 1) attn_bwd_dq_kernel(const __grid_constant__ BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // causal: the last q-tiles see the most K/V tiles, so they go first
  const int qt = a.n_qtiles - 1 - (int)(blockIdx.x / (a.B * a.Hq));
  const int bh = blockIdx.x % (a.B * a.Hq);  // b * Hq + hq
  const int b = bh / a.Hq, hq = bh % a.Hq;
  const int bkv = b * a.Hkv + hq / a.group;
  const int q0 = qt * 128;
  const int off = a.Nk - a.Nq;
  int nsteps = a.n_ktiles;  // K/V tiles 0 .. nsteps-1
  if (a.causal) {
    const long long last = (long long)q0 + 127 + off;  // last key the tile's last row sees
    const long long n = last < 0 ? 0 : last / 128 + 1;
    nsteps = n < a.n_ktiles ? (int)n : a.n_ktiles;
  }

  if (threadIdx.x == 0) bwd_init_bars(bars, 1);
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_FIXED), sDO = sQ + C::TILE_BYTES;
  const uint32_t sRing = smem_u32(smem + C::OFF_RING);

  if (warp == 0) {
    if (lane == 0 && nsteps > 0) {
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
      mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + C::OFF_FIXED + c * (128 * 128), &a.tm_q, &bars->fixed_full, c * 64, q0, bh);
        tma_load_3d(smem + C::OFF_FIXED + C::TILE_BYTES + c * (128 * 128), &a.tm_do, &bars->fixed_full, c * 64, q0,
                    bh);
      }
      int j = 0;
      for (; j < nsteps; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&bars->stage_empty[st], ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns)) break;
        mbar_arrive_expect_tx(&bars->stage_full[st], 2 * C::TILE_BYTES);
        uint8_t* dst = smem + C::OFF_RING + st * 2 * C::TILE_BYTES;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(dst + c * (128 * 128), &a.tm_k, &bars->stage_full[st], c * 64, j * 128, bkv);
          tma_load_3d(dst + C::TILE_BYTES + c * (128 * 128), &a.tm_v, &bars->stage_full[st], c * 64, j * 128, bkv);
        }
      }
      mbar_wait(&bars->fixed_full, 0, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < 2 && st < j; ++st) {
        const int last = j - 1 - ((j - 1 - st) & 1);
        mbar_wait(&bars->stage_full[st], (last >> 1) & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 1) {
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
    };
    if (nsteps > 0) {
      const Desc dq = desc_sw128(sQ, 16, 1024), ddo = desc_sw128(sDO, 16, 1024);
      // halves of 64 keys: S_h = Q K_h^T, dP_h = dO V_h^T, then dQ += dS_h K_h
      auto stage_k = [&](int j) { return sRing + (j & 1) * 2 * C::TILE_BYTES; };
      auto issue_s = [&](int j, int h) {
        const uint32_t sK = stage_k(j) + h * C::HALF_ROWS_BYTES, sV = sK + C::TILE_BYTES;
        if (elect_one()) {
          tc_fence_after();
          issue_qk_rows<D, 64>(tmem + C::COL_S + 64 * h, dq, desc_sw128(sK, 16, 1024));
          issue_qk_rows<D, 64>(tmem + C::COL_DP + 64 * h, ddo, desc_sw128(sV, 16, 1024));
          tc_commit(&bars->s_full[h]);
        }
        __syncwarp();
      };
      auto issue_acc = [&](int j, int h) {
        const uint32_t sK = stage_k(j) + h * C::HALF_ROWS_BYTES;
        if (elect_one()) {
          tc_fence_after();
          issue_pv_ts_w<D, 64>(tmem + C::COL_ACC0, tmem + C::COL_S + 64 * h, desc_sw128(sK, 128 * 128, 1024),
                               j > 0 || h > 0);
        }
        __syncwarp();
      };
      bool ok = wait_all(&bars->fixed_full, 0) && wait_all(&bars->stage_full[0], 0);
      if (ok) {
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int j = 0; j < nsteps && ok; ++j) {
        const bool more = j + 1 < nsteps;
        if (!wait_all(&bars->p_full[0], j & 1)) break;
        issue_acc(j, 0);
        if (more) {
          if (!wait_all(&bars->stage_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) break;
          issue_s(j + 1, 0);
        }
        if (!wait_all(&bars->p_full[1], j & 1)) break;
        issue_acc(j, 1);
        if (elect_one()) {
          tc_commit(&bars->stage_empty[j & 1]);
          if (!more) tc_commit(&bars->o_final);
        }
        __syncwarp();
        if (more) issue_s(j + 1, 1);
      }
      if (elect_one()) tc_commit(&bars->drain);
      __syncwarp();
      mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
    }
  } else if (warp >= 4) {
    // ================= warps 4-7 (half 0) and 8-11 (half 1): one query row per thread,
    // the half's 64 key columns of every step
    const int h = warp >= 8 ? 1 : 0;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int q = q0 + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S, tDP = tmem + lane_off + C::COL_DP;
    const float L2 = lse2_of(a, (size_t)bh, q);
    const float dl = (q < a.Nq) ? __ldg(&a.delta[(size_t)bh * a.Nq + q]) : 0.f;
    float L2v[32], dlv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      L2v[i] = L2;
      dlv[i] = dl;
    }
    bool ok = true;
    for (int j = 0; j < nsteps && ok; ++j) {
      // visible key columns of this query row: key < Nk, and key <= q + off (causal)
      int hi = a.Nk - 1 - j * 128;
      if (a.causal) hi = min(hi, q + off - j * 128);
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[h], j & 1, abort_flag, a.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c0 = 64 * h + 32 * cc;
        uint32_t sv[32], dp[32], P[16], dS[16];
        tmem_ld32(tS + c0, sv);
        tmem_ld32(tDP + c0, dp);
        tmem_ld_wait(sv);
        tmem_ld_wait(dp);
        bwd_chunk(sv, dp, a.scale_log2, L2v, dlv, 0, hi - c0, P, dS);
        tmem_st16(tS + 64 * h + 16 * cc, dS);  // over the half's S columns already read
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[h]);
    }
    ok = __all_sync(0xffffffffu, ok);
    const bool have = nsteps > 0;
    if (ok && have) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0, abort_flag, a.timeout_ns));
      tc_fence_after();
    }
    if (ok) {  // each half's warps write half of the row's columns, staged in the (free) ring
      const uint32_t stage = sRing + (uint32_t)(h * (D / 64) * (128 * 128));
      if (h == 0)
        store_acc_tma<0, D / 2>(stage, r, tmem + lane_off + C::COL_ACC0, have, a.scale, &a.tm_dq, q0, a.Nq, bh);
      else
        store_acc_tma<D / 2, D / 2>(stage, r, tmem + lane_off + C::COL_ACC0, have, a.scale, &a.tm_dq, q0, a.Nq, bh);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
