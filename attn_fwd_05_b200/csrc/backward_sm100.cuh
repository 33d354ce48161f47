// backward_sm100.cuh — gradients of exact attention (the backward pass) for sm_100a.
//
// The method: the forward pass never stores the score matrix; the backward pass
// recomputes it block by block from Q, K and the saved log-sum-exp (patricehuetz.fr,
// "Flash Attention : pourquoi ton GPU utilise 85% de VRAM", section "Ce que fait Flash
// Attention", second idea).  With P = exp(scale Q K^T - LSE) recomputed per block and
// Delta = rowsum(dO o O):
//     dV = P^T dO,  dP = dO V^T,  dS = P o (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// B200 design: one pass over the score matrix, five products per block.
//   * delta kernel: one warp per query row, Delta in fp32; it also clears the row of dQ
//     that the main kernel accumulates into.
//   * main kernel: one CTA per (batch, KV head, 128-key tile), longest first under the
//     causal mask.  It walks the query heads of the KV head's group and the q-tiles that
//     see its keys (a step = one 128-query tile of one head) and keeps dK and dV for its
//     keys in TMEM for the whole walk, so the group's sum needs no atomics.  Per step:
//       S^T = K Q^T and dP^T = V dO^T land in TMEM (128 x 128 each, one key row per TMEM
//       lane); the elementwise warps turn S^T into P^T (bf16, written back over S^T) and
//       dP^T into dS^T (bf16, to shared memory in the 128-byte swizzled layout);
//       dV += P^T dO takes A from TMEM; dK += dS^T Q reads dS^T K-major; dQ_step = dS K
//       reads the same shared dS^T MN-major, into TMEM.  A drain warpgroup moves dQ_step
//       out of TMEM, scales it and adds it to the global dQ with TMA reduce-adds (fp32,
//       performed in L2), staged in the ring stage the step has finished with.
//   TMEM (512 columns): S^T, dP^T (128 each), dV and dK (d each).  At d = 128 dQ_step
//   takes the dP^T columns once the elementwise pass has read them; at d = 64 it has
//   columns of its own.
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
  CUtensorMap tm_dq;   // fp32 [B*Hq, Nq, d], box {32, 32, 1}: dQ is accumulated by TMA reduce-adds
  CUtensorMap tm_dk;   // fp32 [B*Hkv, Nk, d], same boxes, written by TMA stores
  CUtensorMap tm_dv;
  const float* lse;    // [B*Hq, Nq] natural log-sum-exp of the forward pass
  const float* delta;  // [B*Hq, Nq] rowsum(dO o O)
  float* dq;           // [B*Hq, Nq, d], cleared by the delta kernel
  float* dk;           // [B*Hkv, Nk, d]
  float* dv;           // [B*Hkv, Nk, d]
  int B, Hq, Hkv, Nq, Nk, group, causal, n_qtiles, n_ktiles;
  float scale, scale_log2;
  uint64_t timeout_ns;
  // failure-path testing only (-1 in every normal call): CTA dbg_stall_cta leaves the Q
  // tile of its step dbg_stall_step out, so the wait for it runs out after timeout_ns
  int dbg_stall_cta;
  int dbg_stall_step;
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
                                                             float* __restrict__ delta, float* __restrict__ dq,
                                                             long long rows) {
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
    float4* z = reinterpret_cast<float4*>(dq + r * D);
#pragma unroll
    for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) delta[r] = acc;
  }
}

// ------------------------------------------------------------------- shared pieces

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
    bulk_wait_all();  // the staging area is reused or the CTA exits next
  }
  __syncwarp();
}

// dQ_step(128 x D) = dS K: A = dS^T in shared memory read MN-major (query columns in
// 64-element blocks 16 KB apart), B = the K tile read MN-major (d columns in 64-element
// blocks 16 KB apart); k-step kk covers keys 16 kk .. 16 kk + 15, 16 rows of 128 bytes.
template <int D>
__device__ __forceinline__ void issue_ds_k(uint32_t d_tmem, Desc ds, Desc k) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint32_t off = (uint32_t)((kk * 16 * 128) >> 4);
    mma_ss_w(d_tmem, ds.lo + off, ds.hi, k.lo + off, k.hi, idesc, kk > 0 ? 1u : 0u);
  }
}

struct BwdBars {
  uint64_t fixed_full;   // K and V of the CTA's key tile have landed
  uint64_t q_full[2];    // Q of a step has landed (two-stage ring)
  uint64_t q_empty[2];   // S and dK of the step are done with it
  uint64_t do_full;      // dO of the step has landed (one stage)
  uint64_t do_empty;     // dP and dV of the step are done with it
  uint64_t s_full;       // S^T of the step is in TMEM
  uint64_t dp_full;      // dP^T of the step is in TMEM
  uint64_t p_full[2];    // P^T of query half h written over S^T (4 warps each)
  uint64_t ds_full[2];   // dS^T of query half h written over dP^T and to shared memory (4 warps each)
  uint64_t ds_free;      // dQ of the step is done with the shared dS^T
  uint64_t dq_full;      // dQ_step is in TMEM
  uint64_t dq_empty;     // the drain has read dQ_step out of TMEM (4 warps)
  uint64_t stat_full;    // LSE and Delta of the step staged
  uint64_t stat_free;    // the elementwise warps are done with them (8 warps)
  uint64_t o_final;      // the last dK / dV accumulation is done
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
struct BwdCfg {
  // warp 0 loads K, V and Q, warp 1 issues the MMAs, warp 2 stages the statistics, warp 3
  // loads dO; warps 4-7 and 8-11 run the elementwise pass of query columns 0-63 and
  // 64-127 of each step; warps 12-15 drain dQ_step to global memory
  static constexpr int THREADS = 512;
  static constexpr int TILE_BYTES = 128 * D * 2;               // one bf16 tile of 128 rows
  static constexpr int OFF_FIXED = 0;                          // K, V
  static constexpr int OFF_Q = 2 * TILE_BYTES;                 // 2 stages of Q
  static constexpr int OFF_DO = OFF_Q + 2 * TILE_BYTES;        // 1 stage of dO
  static constexpr int OFF_DS = OFF_DO + TILE_BYTES;           // dS^T: 128 keys x 128 queries, bf16
  static constexpr int OFF_STG = OFF_DS + 128 * 128 * 2;       // dQ staging: 64 columns x 128 rows, fp32
  static constexpr int OFF_STAT = OFF_STG + 2 * 128 * 128;     // L2 [128] | Delta [128] of the step
  static constexpr int OFF_BAR = OFF_STAT + 2 * 128 * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;            // + 1 KB alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = D == 128 ? COL_DP : 256 + 2 * D;
  static constexpr int HALF_ROWS_BYTES = 64 * 128;  // offset of rows 64.. inside a 64-column chunk
  // registers per thread after the split (launch: 128 x 512 threads): warps 0-3 need few,
  // the elementwise warps hold P for the step, the drain warps hold dQ_step's row
  static constexpr int REGS_CTRL = 88, REGS_EW = 144, REGS_DRAIN = 136;
  static_assert(REGS_CTRL + 2 * REGS_EW + REGS_DRAIN == 4 * 128, "register split must add up to the launch's");
  static_assert(sizeof(BwdBars) <= 256, "barrier block");
};

constexpr int kBwdKeyBand = 64;  // key tiles per band of the grid order (long sequences)

// Steps of a CTA: (query head of the group, q-tile), q-tiles from qt_lo on.
__device__ __forceinline__ int kv_qt_lo(const BwdArgs& a, int kt) {
  if (!a.causal) return 0;
  const long long x = (long long)kt * 128 - (a.Nk - a.Nq);  // earliest query that sees key kt*128
  if (x <= 0) return 0;
  const long long t = x / 128;
  return t < a.n_qtiles ? (int)t : a.n_qtiles;
}

template <int D>
__global__ void __launch_bounds__(512, 1) attn_bwd_kernel(const __grid_constant__ BwdArgs a) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + C::OFF_BAR);
  float* stat = reinterpret_cast<float*>(smem + C::OFF_STAT);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // causal: the first K/V tiles are seen by the most q-tiles, so they go first (longest
  // processing time first).  With 64 key tiles or more the key tiles are taken in bands of
  // kBwdKeyBand, and within a band one (batch, KV head) after another: the CTAs in flight
  // then belong to about two KV heads instead of all of them, and the Q, dO and dQ tiles
  // they share stay in L2 (16K causal GQA: 22.2 -> 5.7 GB of DRAM traffic per call, the
  // same time).  Fewer key tiles: one key tile a band, consecutive CTAs share it.
  const int nbkv = a.B * a.Hkv;
  const int KB = a.n_ktiles >= kBwdKeyBand ? kBwdKeyBand : 1;
  const int kband = (int)blockIdx.x / (KB * nbkv);
  const int in_band = (int)blockIdx.x % (KB * nbkv);
  const int nk = min(KB, a.n_ktiles - kband * KB);  // the last band may be shorter
  const int bkv = in_band / nk;                      // b * Hkv + kvh
  const int kt = kband * KB + in_band % nk;
  const int b = bkv / a.Hkv, kvh = bkv % a.Hkv;
  const int k0 = kt * 128;
  const int qt_lo = kv_qt_lo(a, kt);
  const int nqt = a.n_qtiles - qt_lo;
  const int nsteps = a.group * nqt;
  auto step_bh = [&](int j) { return b * a.Hq + kvh * a.group + j / nqt; };
  auto step_q0 = [&](int j) { return (qt_lo + j % nqt) * 128; };

  if (threadIdx.x == 0) {
    mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
      mbar_init(&bars->p_full[s], 4);
      mbar_init(&bars->ds_full[s], 4);
    }
    mbar_init(&bars->do_full, 1);
    mbar_init(&bars->do_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->ds_free, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_empty, 4);
    mbar_init(&bars->stat_full, 1);
    mbar_init(&bars->stat_free, 8);
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->drain, 1);
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
  const uint32_t sK = smem_u32(smem + C::OFF_FIXED), sV = sK + C::TILE_BYTES;
  const uint32_t sQ0 = smem_u32(smem + C::OFF_Q), sDO = smem_u32(smem + C::OFF_DO);
  const uint32_t sDS = smem_u32(smem + C::OFF_DS), sSTG = smem_u32(smem + C::OFF_STG);
  auto q_stage = [&](int j) { return sQ0 + (uint32_t)((j & 1) * C::TILE_BYTES); };

  if (warp < 4) {
    setmaxnreg_dec<C::REGS_CTRL>();
    if (warp == 0) {
      // ================= TMA: K and V of the tile once, then Q of every step
      if (lane == 0 && nsteps > 0) {
        tma_prefetch_map(&a.tm_q);
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
          if (j >= 2 && !mbar_wait(&bars->q_empty[st], ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns)) break;
          if (a.dbg_stall_cta == (int)blockIdx.x && j == a.dbg_stall_step) continue;  // left out (testing)
          mbar_arrive_expect_tx(&bars->q_full[st], C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + C::OFF_Q + st * C::TILE_BYTES + c * (128 * 128), &a.tm_q, &bars->q_full[st], c * 64,
                        step_q0(j), step_bh(j));
        }
        // drain: the copies in flight must land before the CTA exits
        mbar_wait(&bars->fixed_full, 0, abort_flag, a.timeout_ns, false);
        for (int st = 0; st < 2 && st < j; ++st) {
          const int last = j - 1 - ((j - 1 - st) & 1);  // last step that used stage st
          if (a.dbg_stall_cta == (int)blockIdx.x && last == a.dbg_stall_step) continue;
          mbar_wait(&bars->q_full[st], (last >> 1) & 1, abort_flag, a.timeout_ns, false);
        }
      }
    } else if (warp == 3) {
      // ================= TMA: dO of every step into its single stage
      if (lane == 0 && nsteps > 0) {
        tma_prefetch_map(&a.tm_do);
        int j = 0;
        for (; j < nsteps; ++j) {
          if (j >= 1 && !mbar_wait(&bars->do_empty, (j - 1) & 1, abort_flag, a.timeout_ns)) break;
          mbar_arrive_expect_tx(&bars->do_full, C::TILE_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + C::OFF_DO + c * (128 * 128), &a.tm_do, &bars->do_full, c * 64, step_q0(j),
                        step_bh(j));
        }
        if (j > 0) mbar_wait(&bars->do_full, (j - 1) & 1, abort_flag, a.timeout_ns, false);
      }
    } else if (warp == 1) {
      // ================= MMA issuer (whole warp, one elected lane issues).  Per step j:
      //   dV += P^T dO, S^T(j+1), dK += dS^T Q, dQ_step = dS K, dP^T(j+1)
      // so that the next step's scores are computed while the elementwise warps work.
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
      };
      if (nsteps > 0) {
        const Desc dk = desc_sw128(sK, 16, 1024), dv = desc_sw128(sV, 16, 1024);
        const Desc ddo = desc_sw128(sDO, 16, 1024);
        auto issue_s = [&](int j) {  // S^T = K Q^T
          if (elect_one()) {
            tc_fence_after();
            issue_qk_rows<D, 128>(tmem + C::COL_S, dk, desc_sw128(q_stage(j), 16, 1024));
            tc_commit(&bars->s_full);
          }
          __syncwarp();
        };
        auto issue_dp = [&]() {  // dP^T = V dO^T
          if (elect_one()) {
            tc_fence_after();
            issue_qk_rows<D, 128>(tmem + C::COL_DP, dv, ddo);
            tc_commit(&bars->dp_full);
          }
          __syncwarp();
        };
        bool ok = wait_all(&bars->fixed_full, 0) && wait_all(&bars->q_full[0], 0);
        if (ok) issue_s(0);
        ok = ok && wait_all(&bars->do_full, 0);
        if (ok) issue_dp();
        for (int j = 0; j < nsteps && ok; ++j) {
          const bool more = j + 1 < nsteps;
          const uint32_t sQ = q_stage(j);
          // dV += P^T dO, one query half at a time (A = P^T half h from TMEM)
          for (int h = 0; h < 2 && ok; ++h) {
            ok = wait_all(&bars->p_full[h], j & 1);
            if (ok && elect_one()) {
              tc_fence_after();
              issue_pv_ts_w<D, 64>(tmem + C::COL_DV, tmem + C::COL_S + 64 * h,
                                   desc_sw128(sDO + h * C::HALF_ROWS_BYTES, 128 * 128, 1024), j > 0 || h > 0);
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) tc_commit(&bars->do_empty);  // dP and dV are done with dO
          __syncwarp();
          // the S columns are free once dV has been issued (products run in issue order)
          if (more) {
            if (!wait_all(&bars->q_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) break;
            issue_s(j + 1);
          }
          // dK += dS^T Q, one query half at a time (A = dS^T half h from TMEM)
          for (int h = 0; h < 2 && ok; ++h) {
            ok = wait_all(&bars->ds_full[h], j & 1);
            if (ok && elect_one()) {
              tc_fence_after();
              issue_pv_ts_w<D, 64>(tmem + C::COL_DK, tmem + C::COL_DP + 64 * h,
                                   desc_sw128(sQ + h * C::HALF_ROWS_BYTES, 128 * 128, 1024), j > 0 || h > 0);
            }
            __syncwarp();
          }
          if (!ok) break;
          if (elect_one()) tc_commit(&bars->q_empty[j & 1]);  // S and dK are done with Q
          __syncwarp();
          // dQ_step = dS K; at d = 64 it has its own columns, which the drain must have
          // emptied of the previous step's
          if (D == 64 && j > 0 && !wait_all(&bars->dq_empty, (j - 1) & 1)) break;
          if (elect_one()) {
            tc_fence_after();
            issue_ds_k<D>(tmem + C::COL_DQ, desc_sw128(sDS, 128 * 128, 1024), desc_sw128(sK, 128 * 128, 1024));
            tc_commit(&bars->ds_free);
            tc_commit(&bars->dq_full);
            if (!more) tc_commit(&bars->o_final);
          }
          __syncwarp();
          if (more) {
            // at d = 128 dP^T of the next step goes where dQ_step is: wait for the drain
            if (D == 128 && !wait_all(&bars->dq_empty, j & 1)) break;
            if (!wait_all(&bars->do_full, (j + 1) & 1)) break;
            issue_dp();
          }
        }
        if (elect_one()) tc_commit(&bars->drain);
        __syncwarp();
        mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
      }
    } else {
      // ================= warp 2: LSE (log2 units) and Delta of each step's 128 queries
      for (int j = 0; j < nsteps; ++j) {
        const size_t bh = step_bh(j);
        const int q0 = step_q0(j);
        float l[4], d[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q = q0 + lane + 32 * i;
          l[i] = lse2_of(a, bh, q);
          d[i] = (q < a.Nq) ? __ldg(&a.delta[bh * a.Nq + q]) : 0.f;
        }
        if (j >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(&bars->stat_free, (j - 1) & 1, abort_flag, a.timeout_ns)))
          break;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          stat[lane + 32 * i] = l[i];
          stat[128 + lane + 32 * i] = d[i];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->stat_full);
      }
    }
  } else if (warp < 12) {
    setmaxnreg_inc<C::REGS_EW>();
    // ================= warps 4-7 (query half 0) and 8-11 (half 1): one key row per
    // thread, the half's 64 query columns of every step
    const int h = warp >= 8 ? 1 : 0;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int k = k0 + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::COL_S + 64 * h, tDP = tmem + lane_off + C::COL_DP + 64 * h;
    const uint32_t ds_row = sDS + (uint32_t)(h * (128 * 128) + r * 128);
    const int off = a.Nk - a.Nq;
    bool ok = true;
    for (int j = 0; j < nsteps && ok; ++j) {
      const int q0 = step_q0(j);
      // first visible query column of this key row: q >= k - off under the causal mask;
      // none for a key past the sequence (its K row is zero-filled, its P must be 0)
      const int lo = (k >= a.Nk ? (1 << 20) : (a.causal ? k - off - q0 : 0)) - 64 * h;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->stat_full, j & 1, abort_flag, a.timeout_ns) &&
                                       mbar_wait(&bars->s_full, j & 1, abort_flag, a.timeout_ns))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- P^T = 2^(s scale log2e - L2) over the visible columns; p keeps it in fp32
      uint32_t p[2][32];
      tmem_ld32(tS, p[0]);
      tmem_ld32(tS + 32, p[1]);
      tmem_ld_wait(p[0]);
      tmem_ld_wait(p[1]);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const float4* L2 = reinterpret_cast<const float4*>(stat + 64 * h + 32 * cc);
        uint32_t P[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 l = L2[i4];
          const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * i4 + e;
            const float y = fmaf(__uint_as_float(p[cc][i]), a.scale_log2, -lv[e]);
            p[cc][i] = __float_as_uint((32 * cc + i >= lo) ? ex2(y) : 0.f);
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          P[i] = pack_bf16x2(__uint_as_float(p[cc][2 * i]), __uint_as_float(p[cc][2 * i + 1]));
        tmem_st16(tS + 16 * cc, P);  // over the half's columns already read
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[h]);
      // ---- dS^T = P^T o (dP^T - Delta): bf16 over dP^T (for dK) and to shared memory
      // in the 128-byte swizzled layout (for dQ)
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&bars->dp_full, j & 1, abort_flag, a.timeout_ns) &&
                          (j == 0 || mbar_wait(&bars->ds_free, (j - 1) & 1, abort_flag, a.timeout_ns)))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dp[32];
        tmem_ld32(tDP + 32 * cc, dp);
        tmem_ld_wait(dp);
        const float4* Dl = reinterpret_cast<const float4*>(stat + 128 + 64 * h + 32 * cc);
        uint32_t dS[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 dl = Dl[i4];
          const int i = 4 * i4;
          dS[2 * i4] = pack_bf16x2(__uint_as_float(p[cc][i]) * (__uint_as_float(dp[i]) - dl.x),
                                   __uint_as_float(p[cc][i + 1]) * (__uint_as_float(dp[i + 1]) - dl.y));
          dS[2 * i4 + 1] = pack_bf16x2(__uint_as_float(p[cc][i + 2]) * (__uint_as_float(dp[i + 2]) - dl.z),
                                       __uint_as_float(p[cc][i + 3]) * (__uint_as_float(dp[i + 3]) - dl.w));
        }
        tmem_st16(tDP + 16 * cc, dS);  // over the half's columns already read
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int gg = 4 * cc + g;  // 16-byte granule of the 128-byte row
          st_shared_v4(ds_row + (uint32_t)((gg ^ (r & 7)) << 4), dS[4 * g], dS[4 * g + 1], dS[4 * g + 2],
                       dS[4 * g + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->ds_full[h]);
        mbar_arrive(&bars->stat_free);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    const bool have = nsteps > 0;
    if (ok && have) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_final, 0, abort_flag, a.timeout_ns));
      tc_fence_after();
    }
    if (ok) {
      // dK (half 0's warps) staged in the K/V tiles, dV (half 1's) in the Q stages; both
      // are free once the last products are done
      if (h == 0)
        store_acc_tma<0, D>(sK, r, tmem + lane_off + C::COL_DK, have, a.scale, &a.tm_dk, k0, a.Nk, bkv);
      else
        store_acc_tma<0, D>(sQ0, r, tmem + lane_off + C::COL_DV, have, 1.0f, &a.tm_dv, k0, a.Nk, bkv);
    }
  } else {
    setmaxnreg_inc<C::REGS_DRAIN>();
    // ================= warps 12-15: dQ_step out of TMEM (one query row per thread) into
    // registers, which frees its columns at once; then, 64 columns at a time, times scale
    // into the staging buffer and added to dQ by TMA reduce-adds that run in the
    // background of the next steps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t tQ = tmem + ((uint32_t)(quad * 32) << 16) + C::COL_DQ;
    const uint32_t stg_rows = sSTG + (uint32_t)(r * 128);
    for (int j = 0; j < nsteps; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->dq_full, j & 1, abort_flag, a.timeout_ns))) break;
      tc_fence_after();
      uint32_t v[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tQ + c * 32, v[c]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld_wait(v[c]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_empty);
      const int q0 = step_q0(j);
      const bool rows_in = q0 + quad * 32 < a.Nq;
#pragma unroll
      for (int half = 0; half < D / 64; ++half) {
        // the previous reduce-adds must have read the staging rows of this warp
        if (lane == 0) bulk_wait_read();
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t* w = v[2 * half + cc];
          const uint32_t row = stg_rows + (uint32_t)(cc * (128 * 128));
#pragma unroll
          for (int g = 0; g < 8; ++g)
            st_shared_v4(row + (uint32_t)((g ^ (r & 7)) << 4), __float_as_uint(__uint_as_float(w[4 * g]) * a.scale),
                         __float_as_uint(__uint_as_float(w[4 * g + 1]) * a.scale),
                         __float_as_uint(__uint_as_float(w[4 * g + 2]) * a.scale),
                         __float_as_uint(__uint_as_float(w[4 * g + 3]) * a.scale));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && rows_in) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc)
            tma_reduce_add_3d(&a.tm_dq, sSTG + (uint32_t)(cc * (128 * 128) + quad * 32 * 128), (2 * half + cc) * 32,
                              q0 + quad * 32, step_bh(j));
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
