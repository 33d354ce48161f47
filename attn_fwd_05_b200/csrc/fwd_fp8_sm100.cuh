// fwd_fp8_sm100.cuh — exact attention forward with FP8 (e4m3) inputs, for sm_100a.
//
// The method is the bf16 forward's (tiled online softmax, the score matrix never leaves
// the chip) with the inputs in FP8 and one scale per block of each tensor: the
// polydesk.ai glossary "FlashAttention", section on FlashAttention-3, names FP8 with
// block quantization as the way H100 approaches 1.2 PFLOPS.  Blocks: 128 rows of a head
// for Q and K (the tiles multiplied together), the whole head for V, so that a row's
// largest probability stays exactly representable when P is rounded to e4m3 (see below).
//
// B200 design (d = 128): the two-tile persistent kernel of the bf16 path with
//   * Q, K, V tiles of 128 x 128 bytes: one 128-byte swizzle row per token, brought in
//     by TMA;
//   * S = Q K^T and O += P V as tcgen05.mma kind::f8f6f4 (e4m3 x e4m3, fp32 accumulate,
//     32 elements of the contraction per instruction, twice the bf16 rate); V stays
//     [keys][d] and is read MN-major;
//   * the block scales folded into the softmax: scores s (units of the fp8 products) are
//     multiplied by scale * log2(e) * sq * sk_j, the q-tile's and the key block's scales;
//   * P = 2^(s - m) with the exact running maximum m (so P <= 1 and the row maximum is 1),
//     scaled by 256 and rounded to e4m3 into shared memory; 256 = 2^8 is exact in e4m3,
//     which keeps the largest probability exact, and pushes probabilities down to 2^-17
//     above the format's smallest subnormal;
//   * O = O_acc * sv / l' in the epilogue, l' the fp32 sum of the unrounded 256 P (the
//     factor 2^8 is added in the exponent: 2^(y + 8) = 256 2^y, exactly).
#pragma once

#include "sm100_common.cuh"

namespace attn {

struct Fp8Args {
  CUtensorMap tm_q;  // [B*Hq, Nq, 128] uint8 (e4m3), box {128, 128, 1}
  CUtensorMap tm_k;  // [B*Hkv, Nk, 128]
  CUtensorMap tm_v;
  CUtensorMap tm_o;      // bf16 O [B*Hq, Nq, 128], box {64, 32, 1} (unused for fp32 O)
  const float* q_scale;  // [B*Hq, ceil(Nq/128)]
  const float* k_scale;  // [B*Hkv, ceil(Nk/128)]
  const float* v_scale;  // [B*Hkv]
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nk, group, causal, o_f32;
  float scale_log2;  // scale * log2(e)
  int pair_heads, n_qtiles, n_ktiles, n_units;
  uint64_t timeout_ns;
};

// Instruction descriptor of tcgen05.mma kind::f8f6f4 with e4m3 A and B (format code 0)
// and an fp32 accumulator; the other fields as in idesc_bf16_f32.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f8_ss_w(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi, uint32_t b_lo,
                                            uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// S(128 x 128) = Q K^T, both K-major with 128-byte rows (d = 128 bytes): k-step kk takes
// 32 elements = 32 bytes of the row.
__device__ __forceinline__ void issue_qk_f8(uint32_t s_tmem, Desc q, Desc k) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_f8_ss_w(s_tmem, q.lo + (uint32_t)(kk * 2), q.hi, k.lo + (uint32_t)(kk * 2), k.hi, idesc, kk > 0 ? 1u : 0u);
}

// O(128 x 128) += P V: P K-major (128-byte rows of keys), V MN-major ([keys][d], 128-byte
// rows): k-step kk takes keys 32kk..32kk+31, 32 bytes of a P row and 32 rows of V.
__device__ __forceinline__ void issue_pv_f8(uint32_t o_tmem, Desc p, Desc v, bool accumulate) {
  constexpr uint32_t idesc = idesc_e4m3_f32(128, 128, 0, 1);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_f8_ss_w(o_tmem, p.lo + (uint32_t)(kk * 2), p.hi, v.lo + (uint32_t)((kk * 32 * 128) >> 4), v.hi, idesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

// Four values to e4m3 (round to nearest even, saturating), the first in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float x0, float x1, float x2, float x3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// ------------------------------------------------------------------------ quantizer

// One CTA per block of `block_rows` rows of one plane ([planes, N, d] bf16 input):
// scale = amax / 448 (1 if the block is zero), code = e4m3(x / scale); both divisions
// rounded to nearest in fp32.
__global__ void __launch_bounds__(256) attn_quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ x,
                                                                 uint8_t* __restrict__ out, float* __restrict__ scales,
                                                                 int N, int d, int block_rows, int nblk) {
  __shared__ float red[8];
  const int blk = blockIdx.x % nblk;
  const long long plane = blockIdx.x / nblk;
  const int r0 = blk * block_rows;
  const int rows = min(block_rows, N - r0);
  const size_t base = ((size_t)plane * N + r0) * d;
  const long long pairs = (long long)rows * d / 2;
  const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(x + base);
  float amax = 0.f;
  for (long long i = threadIdx.x; i < pairs; i += blockDim.x) {
    const float2 v = __bfloat1622float2(src[i]);
    amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, s));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  uint16_t* dst = reinterpret_cast<uint16_t*>(out + base);
  for (long long i = threadIdx.x; i < pairs; i += blockDim.x) {
    const float2 v = __bfloat1622float2(src[i]);
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(__fdiv_rn(v.y, sc)), "f"(__fdiv_rn(v.x, sc)));
    dst[i] = c;
  }
  if (threadIdx.x == 0) scales[plane * nblk + blk] = sc;
}

// --------------------------------------------------------------------- attention

struct Fp8Cfg {
  static constexpr int THREADS = 384;  // warp 0 TMA, 1 MMA, 2-3 idle, 4-7 / 8-11 softmax of tiles 0 / 1
  static constexpr int TILE = 128 * 128;  // bytes of a 128 x 128 e4m3 tile
  static constexpr int NSTAGE = 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = 2 * TILE;
  static constexpr int OFF_KV = 4 * TILE;
  // bf16 O of a tile leaves through TMA stores of two 64-column chunks, staged in the
  // tile's P buffer and in one more 16 KB buffer per tile
  static constexpr int OFF_X = OFF_KV + NSTAGE * TILE;
  static constexpr int OFF_BAR = OFF_X + 2 * TILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;  // + 1 KB alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 384;
};
static_assert(Fp8Cfg::SMEM <= 227 * 1024, "shared memory");

struct Fp8Bars {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t o_final[2];
  uint64_t drain;
  uint64_t kv_full[Fp8Cfg::NSTAGE];
  uint64_t kv_empty[Fp8Cfg::NSTAGE];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Fp8Bars) <= 256, "barrier area");

struct Fp8Tile {
  int hq, q0, rows, jhi;  // blocks 0 .. jhi-1 are visited
};

__device__ __forceinline__ Fp8Tile fp8_tile(const Fp8Args& a, int hq, int q0) {
  Fp8Tile t{hq, q0, 0, 0};
  if (q0 >= a.Nq) return t;
  t.rows = min(128, a.Nq - q0);
  long long nkeys = a.Nk;
  if (a.causal) {
    const long long last = (long long)q0 + t.rows - 1 + a.Nk - a.Nq;
    nkeys = last + 1 < 0 ? 0 : (last + 1 > a.Nk ? a.Nk : last + 1);
  }
  t.jhi = (int)((nkeys + 127) / 128);
  return t;
}

__device__ __forceinline__ void fp8_unit(const Fp8Args& a, int u, int& b, int& kvh, Fp8Tile (&tj)[2]) {
  if (a.pair_heads) {
    const int hp_n = a.Hq / 2;
    const int qt = a.causal ? a.n_qtiles - 1 - u / (a.B * hp_n) : u % a.n_qtiles;
    const int rem = a.causal ? u % (a.B * hp_n) : u / a.n_qtiles;
    b = rem / hp_n;
    const int h0 = 2 * (rem % hp_n);
    tj[0] = fp8_tile(a, h0, qt * 128);
    tj[1] = fp8_tile(a, h0 + 1, qt * 128);
  } else {
    const int nqp = (a.n_qtiles + 1) / 2;
    const int qp = a.causal ? nqp - 1 - u / (a.B * a.Hq) : u % nqp;
    const int rem = a.causal ? u % (a.B * a.Hq) : u / nqp;
    b = rem / a.Hq;
    const int h = rem % a.Hq;
    tj[0] = fp8_tile(a, h, 2 * qp * 128);
    tj[1] = fp8_tile(a, h, (2 * qp + 1) * 128);
  }
  kvh = tj[0].hq / a.group;
}

__global__ void __launch_bounds__(384, 1) attn_fwd_fp8_kernel(const __grid_constant__ Fp8Args a) {
  using C = Fp8Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Fp8Bars* bars = reinterpret_cast<Fp8Bars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->q_empty[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_free[t], 4);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_done[t], 1);
      mbar_init(&bars->o_final[t], 1);
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
  const uint32_t sQ = smem_u32(smem + C::OFF_Q), sP = smem_u32(smem + C::OFF_P), sKV = smem_u32(smem + C::OFF_KV);

  int b, kvh;
  Fp8Tile tj[2];
  constexpr int kDone = 0x7fffffff;
  auto tile_next = [&](int t, int kb) -> int {
    const Fp8Tile& j = t ? tj[1] : tj[0];
    return (j.rows > 0 && kb < j.jhi) ? kb : kDone;
  };
  auto union_next = [&](int kb) -> int { return min(tile_next(0, kb), tile_next(1, kb)); };
  auto snake_unit = [&](int rd) -> int {
    return rd * (int)gridDim.x + ((rd & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_map(&a.tm_q);
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
      const uint64_t pol = l2_policy_evict_last();
      int seq = 0;
      int nql[2] = {0, 0};
      auto push = [&](int kb, int kv) -> bool {
        const int st = seq % C::NSTAGE;
        const int use = seq / C::NSTAGE;
        if (use > 0 && !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, abort_flag, a.timeout_ns)) return false;
        mbar_arrive_expect_tx(&bars->kv_full[st], C::TILE);
        tma_load_3d_hint(smem + C::OFF_KV + st * C::TILE, kv ? &a.tm_v : &a.tm_k, &bars->kv_full[st], 0, kb * 128,
                         b * a.Hkv + kvh, pol);
        ++seq;
        return true;
      };
      bool ok = true;
      for (int rd = 0; rd * (int)gridDim.x < a.n_units && ok; ++rd) {
        const int u = snake_unit(rd);
        if (u >= a.n_units) continue;
        fp8_unit(a, u, b, kvh, tj);
        for (int t = 0; t < 2 && ok; ++t) {
          if (tile_next(t, 0) == kDone) continue;
          if (nql[t] > 0 && !mbar_wait(&bars->q_empty[t], (nql[t] - 1) & 1, abort_flag, a.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->q_full[t], C::TILE);
          tma_load_3d(smem + C::OFF_Q + t * C::TILE, &a.tm_q, &bars->q_full[t], 0, tj[t].q0, b * a.Hq + tj[t].hq);
          ++nql[t];
        }
        int kb = union_next(0);
        if (ok && kb != kDone) ok = push(kb, 0);
        while (ok && kb != kDone) {
          const int nk = union_next(kb + 1);
          if (nk != kDone) ok = push(nk, 0);
          if (ok) ok = push(kb, 1);
          kb = nk;
        }
      }
      for (int t = 0; t < 2; ++t)
        if (nql[t] > 0) mbar_wait(&bars->q_full[t], (nql[t] - 1) & 1, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < C::NSTAGE && st < seq; ++st)
        mbar_wait(&bars->kv_full[st], ((seq - 1 - st) / C::NSTAGE) & 1, abort_flag, a.timeout_ns, false);
    }
  } else if (warp == 1) {
    auto stage_of = [&](int seq) { return seq % C::NSTAGE; };
    auto parity_of = [&](int seq) { return (uint32_t)((seq / C::NSTAGE) & 1); };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
    };
    const Desc dq[2] = {desc_sw128(sQ, 16, 1024), desc_sw128(sQ + C::TILE, 16, 1024)};
    const Desc dp[2] = {desc_sw128(sP, 16, 1024), desc_sw128(sP + C::TILE, 16, 1024)};
    const Desc dk0 = desc_sw128(sKV, 16, 1024);
    const Desc dv0 = desc_sw128(sKV, 128 * 128, 1024);
    auto kdesc = [&](int seq) { return Desc{dk0.lo + (uint32_t)(stage_of(seq) * (C::TILE >> 4)), dk0.hi}; };
    auto vdesc = [&](int seq) { return Desc{dv0.lo + (uint32_t)(stage_of(seq) * (C::TILE >> 4)), dv0.hi}; };
    int seq = 0;
    int nqk[2] = {0, 0}, npv[2] = {0, 0}, nql[2] = {0, 0};
    bool ok = true;
    auto issue_s = [&](int kb) -> bool {
      if (!wait_all(&bars->kv_full[stage_of(seq)], parity_of(seq))) return false;
      const Desc dk = kdesc(seq);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (tile_next(t, kb) != kb) continue;
        if (nqk[t] > 0 && !wait_all(&bars->s_free[t], (nqk[t] - 1) & 1)) return false;
        const bool last = tile_next(t, kb + 1) == kDone;
        if (elect_one()) {
          tc_fence_after();
          issue_qk_f8(tmem + (t ? C::COL_S1 : C::COL_S0), dq[t], dk);
          tc_commit(&bars->s_full[t]);
          if (last) tc_commit(&bars->q_empty[t]);
        }
        __syncwarp();
        ++nqk[t];
      }
      if (elect_one()) tc_commit(&bars->kv_empty[stage_of(seq)]);
      __syncwarp();
      ++seq;
      return true;
    };
    for (int rd = 0; rd * (int)gridDim.x < a.n_units && ok; ++rd) {
      const int u = snake_unit(rd);
      if (u >= a.n_units) continue;
      fp8_unit(a, u, b, kvh, tj);
      int kb = union_next(0);
      if (kb == kDone) continue;
      int upv[2] = {0, 0};
      for (int t = 0; t < 2 && ok; ++t) {
        if (tile_next(t, 0) == kDone) continue;
        ok = wait_all(&bars->q_full[t], nql[t] & 1);
        ++nql[t];
      }
      if (ok) ok = issue_s(kb);
      while (ok && kb != kDone) {
        const int nk = union_next(kb + 1);
        if (nk != kDone && !issue_s(nk)) {
          ok = false;
          break;
        }
        if (!wait_all(&bars->kv_full[stage_of(seq)], parity_of(seq))) {
          ok = false;
          break;
        }
        const Desc dv = vdesc(seq);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || tile_next(t, kb) != kb) continue;
          if (!wait_all(&bars->p_full[t], npv[t] & 1)) {
            ok = false;
            continue;
          }
          const bool last = tile_next(t, kb + 1) == kDone;
          if (elect_one()) {
            tc_fence_after();
            issue_pv_f8(tmem + (t ? C::COL_O1 : C::COL_O0), dp[t], dv, upv[t] > 0);
            tc_commit(&bars->o_done[t]);
            if (last) tc_commit(&bars->o_final[t]);
          }
          __syncwarp();
          ++npv[t];
          ++upv[t];
        }
        if (!ok) break;
        if (elect_one()) tc_commit(&bars->kv_empty[stage_of(seq)]);
        __syncwarp();
        ++seq;
        kb = nk;
      }
    }
    if (elect_one()) tc_commit(&bars->drain);
    __syncwarp();
    mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
  } else if (warp >= 4) {
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (t ? C::COL_S1 : C::COL_S0);
    const uint32_t o_addr = tmem + lane_off + (t ? C::COL_O1 : C::COL_O0);
    const uint32_t p_row = sP + t * C::TILE + (uint32_t)r * 128u;
    const uint32_t x_tile = smem_u32(smem + C::OFF_X) + t * C::TILE;
    int k = 0, nfin = 0;
    bool fail = false;
    // this warp's last O store still reads its rows of the staging buffers (P_t, X_t)
    bool store_pending = false;
    auto settle_store = [&]() {
      if (store_pending) {
        if (lane == 0) bulk_wait_read();
        __syncwarp();
        store_pending = false;
      }
    };
    for (int rd = 0; rd * (int)gridDim.x < a.n_units && !fail; ++rd) {
      const int u = snake_unit(rd);
      if (u >= a.n_units) continue;
      fp8_unit(a, u, b, kvh, tj);
      const Fp8Tile job = t ? tj[1] : tj[0];
      const int q = job.q0 + r;
      const int khi = q + a.Nk - a.Nq;  // last visible key (causal)
      const size_t bhq = (size_t)b * a.Hq + job.hq;
      const float sq = job.rows > 0 ? __ldg(&a.q_scale[bhq * a.n_qtiles + job.q0 / 128]) : 1.f;
      const float* ks_row = a.k_scale + ((size_t)b * a.Hkv + kvh) * a.n_ktiles;
      float m = -INFINITY, l = 0.f;
      int kl = 0;
      for (int kb = tile_next(t, 0); kb != kDone; kb = tile_next(t, kb + 1), ++k, ++kl) {
        if (__any_sync(0xffffffffu, !mbar_wait(&bars->s_full[t], k & 1, abort_flag, a.timeout_ns) || *abort_flag)) {
          fail = true;
          break;
        }
        tc_fence_after();
        const float c = a.scale_log2 * sq * __ldg(&ks_row[kb]);  // log2 units per unit of the fp8 product
        uint32_t rs[128];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld32(s_addr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&rs[32 * j]));
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&rs[32 * j]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[t]);
        // mask: keys past Nk, and past the diagonal when causal
        int lim = a.Nk - 1 - kb * 128;
        if (a.causal) lim = min(lim, khi - kb * 128);
        // raw scores (units of the fp8 products); the mask only where the block needs it
        float s[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(rs[i]);
        const bool masked = lim < 127;
        if (masked) {
#pragma unroll
          for (int i = 0; i < 128; ++i) s[i] = (i > lim) ? -INFINITY : s[i];
        }
        float x0 = max3(s[0], s[1], s[2]), x1 = max3(s[3], s[4], s[5]);
#pragma unroll
        for (int i = 6; i < 126; i += 4) {
          x0 = max3(x0, s[i], s[i + 1]);
          x1 = max3(x1, s[i + 2], s[i + 3]);
        }
        const float mx = max3(x0, x1, fmaxf(s[126], s[127])) * c;  // c > 0 commutes with the max
        float alpha = 1.0f;
        if (mx > m) {
          alpha = ex2(m - mx);
          m = mx;
        }
        // p' = 256 p = 2^(s c - m + 8): the factor 2^8 rides in the exponent; l sums p'
        const float nmu = (m == -INFINITY) ? 0.0f : 8.0f - m;
        uint32_t P[32];
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float y0, y1, y2, y3, p0, p1, p2, p3;
          fma2(y0, y1, s[4 * i], s[4 * i + 1], c, c, nmu, nmu);
          fma2(y2, y3, s[4 * i + 2], s[4 * i + 3], c, c, nmu, nmu);
          // a quarter of the pairs on the FMA pipe, as in the bf16 kernel; in masked blocks a
          // hidden key gives 2^-117 (below e4m3's range, so P is 0; a row that never sees a
          // visible key is written from m = -inf)
          if ((i & 3) == 3) {
            exp2_fma2(p0, p1, y0, y1);
          } else {
            p0 = ex2(y0);
            p1 = ex2(y1);
          }
          p2 = ex2(y2);
          p3 = ex2(y3);
          add2(a0, a1, p0, p1);
          add2(a0, a1, p2, p3);
          P[i] = pack_e4m3x4(p0, p1, p2, p3);
        }
        l = l * alpha + (a0 + a1);  // in units of 256
        if (!__all_sync(0xffffffffu,
                        k == 0 || mbar_wait(&bars->o_done[t], (k - 1) & 1, abort_flag, a.timeout_ns))) {
          fail = true;
          break;
        }
        settle_store();
#pragma unroll
        for (int g = 0; g < 8; ++g)  // 16-byte granule g (keys 16g..16g+15) at g ^ (r % 8)
          st_shared_v4(p_row + (uint32_t)((g ^ (r & 7)) << 4), P[4 * g], P[4 * g + 1], P[4 * g + 2], P[4 * g + 3]);
        fence_proxy_async_smem();
        if (kl > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
          tc_fence_after();
          uint32_t ro[128];  // one TMEM round trip for the whole row
#pragma unroll
          for (int j = 0; j < 4; ++j) tmem_ld32(o_addr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&ro[32 * j]));
#pragma unroll
          for (int j = 0; j < 4; ++j) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&ro[32 * j]));
#pragma unroll
          for (int i = 0; i < 128; i += 2) {
            float u0 = __uint_as_float(ro[i]), u1 = __uint_as_float(ro[i + 1]);
            mul2(u0, u1, alpha, alpha);
            ro[i] = __float_as_uint(u0);
            ro[i + 1] = __float_as_uint(u1);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) tmem_st32(o_addr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&ro[32 * j]));
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      if (fail) break;
      const bool have_o = kl > 0;
      bool ok = true;
      if (have_o) {
        ok = mbar_wait(&bars->o_final[t], nfin & 1, abort_flag, a.timeout_ns);
        tc_fence_after();
        ++nfin;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        fail = true;
        break;
      }
      const bool valid = r < job.rows;
      const size_t row = bhq * (size_t)a.Nq + (size_t)(valid ? q : 0);
      if (m == -INFINITY) l = 0.f;  // no visible key: O = 0, LSE = -inf
      const float sv = __ldg(&a.v_scale[(size_t)b * a.Hkv + kvh]);
      const float inv = l > 0.f ? sv / l : 0.f;  // l already carries the factor 256
      if (!a.o_f32) {
        if (job.rows > quad * 32) {  // the warp has valid rows (warp-uniform)
          // P_t is free (the tile's last P V of the unit is done, or it had none): this
          // warp's 32 rows of O go to P_t (columns 0-63) and X_t (64-127), swizzled like
          // P, and TMA stores them (rows past Nq are clipped)
          settle_store();
          uint32_t ro[128];
          if (have_o) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld32(o_addr + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&ro[32 * j]));
#pragma unroll
            for (int j = 0; j < 4; ++j) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&ro[32 * j]));
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i) ro[i] = 0u;
          }
          const uint32_t xrow = x_tile + (uint32_t)r * 128u;
#pragma unroll
          for (int g = 0; g < 16; ++g) {  // 16-byte granule: 8 columns
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = pack_bf16x2(__uint_as_float(ro[8 * g + 2 * i]) * inv, __uint_as_float(ro[8 * g + 2 * i + 1]) * inv);
            st_shared_v4((g < 8 ? p_row : xrow) + (uint32_t)(((g & 7) ^ (r & 7)) << 4), w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const uint32_t off = (uint32_t)(quad * 32 * 128);
            tma_store_3d(&a.tm_o, sP + t * C::TILE + off, 0, job.q0 + quad * 32, (int)bhq);
            tma_store_3d(&a.tm_o, x_tile + off, 64, job.q0 + quad * 32, (int)bhq);
            bulk_commit();
          }
          store_pending = true;
        }
        if (valid && a.lse != nullptr) a.lse[row] = (l > 0.f) ? (m + log2f(l) - 8.0f) * kLn2 : -INFINITY;
        continue;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t ro[32];
        if (have_o) {
          tmem_ld32(o_addr + 32 * j, ro);
          tmem_ld_wait(ro);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = 0u;
        }
        if (!valid) continue;
        if (a.o_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + row * 128 + 32 * j);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(ro[4 * i]) * inv, __uint_as_float(ro[4 * i + 1]) * inv,
                                 __uint_as_float(ro[4 * i + 2]) * inv, __uint_as_float(ro[4 * i + 3]) * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + row * 128 + 32 * j);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ro[8 * i + 0]) * inv, __uint_as_float(ro[8 * i + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ro[8 * i + 2]) * inv, __uint_as_float(ro[8 * i + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ro[8 * i + 4]) * inv, __uint_as_float(ro[8 * i + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ro[8 * i + 6]) * inv, __uint_as_float(ro[8 * i + 7]) * inv);
            dst[i] = w;
          }
        }
      }
      if (valid && a.lse != nullptr) a.lse[row] = (l > 0.f) ? (m + log2f(l) - 8.0f) * kLn2 : -INFINITY;
    }
    if (lane == 0) bulk_wait_all();  // this warp's O stores are done before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace attn
