// prefill_d256_sm100.cuh — exact attention forward (prefill) for d = 256 on sm_100a.
//
// The method is the one of prefill_sm100.cuh (tiles, online softmax, rescaling when the
// maximum moves; polydesk.ai glossary "FlashAttention", section "L'idée clé :
// IO-awareness").  With d = 256 one O accumulator takes half of TMEM, so this kernel
// takes one 128-row Q tile per CTA: S is double-buffered in 64-column blocks next to O,
// the next S = Q K^T runs while the softmax works, P is written back over its S block and
// P V reads it from TMEM.  The row reference moves only when the maximum grows by more
// than 2^8, and O is normalised by the sum of the bf16-rounded probabilities (see
// softmax_row64_step).
#pragma once

#include "prefill_sm100.cuh"

namespace attn {

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

// Epilogue for one row: O / lr to global (bf16 or fp32) and the log-sum-exp from l.
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
// Kernel 2: one Q tile per CTA, S double-buffered (d = 256)
// ====================================================================================

// Softmax over the calling thread's whole 64-column row of one score block (one
// warpgroup per tile; d = 256).  With d = 256 an O rescale moves 256 TMEM columns, so
// the row reference is kept until the maximum grows by more than 2^8 (p <= 256 then).
// The largest probability is then not exactly 1, so two sums are kept: lr, the sum of
// the bf16-rounded P that multiply V, normalises O (the rounding of a dominant
// probability cancels in the ratio); l, the fp32 sum, gives the log-sum-exp.
// Returns the factor for the row's O.

constexpr float kStaleMaxSlack = 8.0f;  // log2 units

template <bool LOW>
__device__ __forceinline__ float softmax_row64_step(uint32_t s_taddr, bool masked, int col_limit, int col_low,
                                                    float sl2, float& m, float& l, float& lr) {
  uint32_t r[64];
  tmem_ld32(s_taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld32(s_taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  float s[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(r[c]);
  if (masked) {
#pragma unroll
    for (int c = 0; c < 64; ++c) s[c] = (c > col_limit || (LOW && c < col_low)) ? -INFINITY : s[c];
  }
  float x0 = max3(s[0], s[1], s[2]), x1 = max3(s[3], s[4], s[5]);
#pragma unroll
  for (int c = 6; c < 62; c += 4) {
    x0 = max3(x0, s[c], s[c + 1]);
    x1 = max3(x1, s[c + 2], s[c + 3]);
  }
  const float mx = max3(x0, x1, fmaxf(s[62], s[63])) * sl2;
  float alpha = 1.0f;
  if (mx > m + kStaleMaxSlack) {  // false while nothing is visible (mx = -inf)
    alpha = ex2(m - mx);          // 0 when m = -inf
    m = mx;
  }
  const float nmu = (m == -INFINITY) ? 0.0f : -m;
  float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t P[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int i = 16 * half + k;
      float y0, y1;
      fma2(y0, y1, s[2 * i], s[2 * i + 1], sl2, sl2, nmu, nmu);
      const float p0 = ex2(y0), p1 = ex2(y1);
      add2(a0, a1, p0, p1);
      const uint32_t w = pack_bf16x2(p0, p1);
      P[k] = w;
      add2(b0, b1, bf16lo_to_f32(w), bf16hi_to_f32(w));
    }
    tmem_st16(s_taddr + 16 * half, P);
  }
  l = l * alpha + (a0 + a1);
  lr = lr * alpha + (b0 + b1);
  return alpha;
}

template <int D>
struct SingleCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 64;
  static constexpr int THREADS = 256;  // warp 0 TMA, warp 1 MMA, warps 4-7 softmax
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  // 5 stages: S(j+2) needs K(j+2) right after P V(j), and with 4 stages that tile can
  // only start loading once P V(j-1) has released its stage (225.5 KB of shared memory)
  static constexpr int NSTAGE = 5;
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
  uint64_t o_done;   // one phase per P V
  uint64_t o_final;  // one phase: the last P V is done
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
  uint32_t visible[32];  // block-sparse map row of the tile: bit mb = 128-key block mb
};

template <int D, bool MASKS>
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
    const int qt = a.causal ? a.n_qtiles - 1 - u / per_level : u % a.n_qtiles;
    const int rem = a.causal ? u % per_level : u / a.n_qtiles;
    b = rem / a.Hq;
    hq = rem % a.Hq;
    job = make_tile<BN, MASKS>(a, hq, qt * 128);
  }
  const int kvh = hq / a.group;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_final, 1);
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
  if (MASKS && warp == 2 && a.block_mask != nullptr) build_row_bitmap(a, job, bars->visible, 32);  // nkt <= 1024
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);
  const uint32_t* bits = (MASKS && a.block_mask != nullptr) ? bars->visible : nullptr;
  const int kb0 = next_visit<BN>(bits, job, job.jlo);  // first visited block
  const bool any = job.rows > 0 && kb0 < job.jhi;

  if (warp == 0) {
    if (lane == 0 && any) {
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
      for (int kb = kb0; kb < job.jhi && ok; kb = next_visit<BN>(bits, job, kb + 1)) {
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
                             c * 64, kb * BN, b * a.Hkv + kvh, pol);
        }
      }
      mbar_wait(&bars->q_full, 0, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < C::NSTAGE && st < it; ++st) {
        const int last_use = (it - 1 - st) / C::NSTAGE;
        mbar_wait(&bars->kv_full[st], last_use & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 1) {
    // Visit j: K at ring position 2j, V at 2j + 1; S(j) in TMEM block j & 1.  S(j + 2) is
    // issued right after P V(j), which freed that block.  The whole warp runs the loop and
    // one elected lane issues (see the two-tile kernel).
    if (any) {
      auto stage_of = [&](int it) { return it % C::NSTAGE; };
      auto parity_of = [&](int it) { return (uint32_t)((it / C::NSTAGE) & 1); };
      auto colS = [&](int j) { return (j & 1) ? C::COL_S1 : C::COL_S0; };
      auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
      };
      const Desc dq = desc_sw128(sQ, 16, 1024);
      const Desc dk0 = desc_sw128(sKV, 16, 1024);
      const Desc dv0 = desc_sw128(sKV, BN * 128, 1024);
      auto kdesc = [&](int it) { return Desc{dk0.lo + (uint32_t)(stage_of(it) * (C::KV_BYTES >> 4)), dk0.hi}; };
      auto vdesc = [&](int it) { return Desc{dv0.lo + (uint32_t)(stage_of(it) * (C::KV_BYTES >> 4)), dv0.hi}; };
      bool ok = wait_all(&bars->q_full, 0);
      int nq = 0;      // Q K^T issued (visits 0 .. nq-1)
      int kbq = kb0;   // block of the next Q K^T
      for (; nq < 2 && kbq < job.jhi && ok; ++nq, kbq = next_visit<BN>(bits, job, kbq + 1)) {
        const int itK = 2 * nq;
        if (!wait_all(&bars->kv_full[stage_of(itK)], parity_of(itK))) {
          ok = false;
          break;
        }
        if (elect_one()) {
          tc_fence_after();
          issue_qk_w<D, BN>(tmem + colS(nq), dq, kdesc(itK));
          tc_commit(&bars->s_full[nq & 1]);
          tc_commit(&bars->kv_empty[stage_of(itK)]);
        }
        __syncwarp();
      }
      for (int j = 0; j < nq && ok; ++j) {
        const int itV = 2 * j + 1;
        if (!wait_all(&bars->kv_full[stage_of(itV)], parity_of(itV))) break;
        if (!wait_all(&bars->p_full[j & 1], (j >> 1) & 1)) break;
        const bool last = j + 1 == nq && kbq >= job.jhi;  // that is the last visit
        if (elect_one()) {
          tc_fence_after();
          issue_pv_ts_w<D, BN>(tmem + C::COL_O, tmem + colS(j), vdesc(itV), j > 0);
          tc_commit(&bars->o_done);
          if (last) tc_commit(&bars->o_final);
          tc_commit(&bars->kv_empty[stage_of(itV)]);
        }
        __syncwarp();
        if (kbq < job.jhi) {
          const int itK = 2 * nq;  // nq == j + 2
          if (!wait_all(&bars->kv_full[stage_of(itK)], parity_of(itK))) break;
          if (elect_one()) {
            tc_fence_after();
            issue_qk_w<D, BN>(tmem + colS(nq), dq, kdesc(itK));
            tc_commit(&bars->s_full[nq & 1]);
            tc_commit(&bars->kv_empty[stage_of(itK)]);
          }
          __syncwarp();
          ++nq;
          kbq = next_visit<BN>(bits, job, kbq + 1);
        }
      }
      if (elect_one()) tc_commit(&bars->drain);
      __syncwarp();
      mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + C::COL_O;
    const int q = job.q0 + r;
    const int khi = row_key_limit(a, q);
    const int klo = MASKS ? row_key_low(a, q) : 0;
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    int j = 0;  // visits so far
    for (int kb = any ? kb0 : job.jhi; kb < job.jhi; kb = next_visit<BN>(bits, job, kb + 1), ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, a.timeout_ns))) {
        ok = false;  // warp-uniform: the TMEM accesses are per warp
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_off + ((j & 1) ? C::COL_S1 : C::COL_S0);
      const bool masked = block_needs_mask<BN, MASKS>(a, job, kb);
      const float alpha =
          softmax_row64_step<MASKS>(s_addr, masked, khi - kb * BN, klo - kb * BN, a.scale_log2, m, l, lr);
      if (__any_sync(0xffffffffu, alpha != 1.0f) && j > 0) {
        // P V(j-2) finished before S(j) (issued after it), so o_done is in phase j-1 or
        // later and its parity names P V(j-1) without ambiguity
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done, (j - 1) & 1, abort_flag, a.timeout_ns))) {
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
    const bool have_o = any;
    if (ok && have_o) {
      // o_final, not o_done: the next Q K^T runs ahead of P V here, so P V(j-2) may
      // still be in flight and o_done's parity could name an older completed phase
      ok = mbar_wait(&bars->o_final, 0, abort_flag, a.timeout_ns);
      tc_fence_after();
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok) store_row<D>(a, o_addr, have_o, r < job.rows, b, hq, q, m, l, lr);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
