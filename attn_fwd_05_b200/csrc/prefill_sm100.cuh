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
//   * One warp issues the tcgen05 MMAs (one elected lane): S = Q K^T lands in tensor
//     memory (TMEM), the softmax warps read S from TMEM, and O += P V accumulates in
//     TMEM.
//   * Kernel "pingpong" (d = 64 or 128): two 128-row Q tiles per CTA, each with its own
//     softmax warpgroup (the FA4 page, section "Pipeline ping-pong avec double tuile
//     Query", describes two Q tiles per CTA for Blackwell).  TMEM: S0 | S1 | O0 | O1 =
//     128 + 128 + d + d columns.  P goes to shared memory, so S is free once the softmax
//     has read it and the next S = Q K^T runs during the softmax.  Persistent CTAs.
//   * d = 256 has its own kernel (prefill_d256_sm100.cuh); this file holds the two-tile
//     kernel and the tile planning both kernels share.
//   * d <= 128: the reference of each row is its exact running maximum: whenever a block
//     raises it, the row's O accumulator is rescaled in TMEM before the next P V.  The
//     row's largest probability is then exactly 1 and its bf16 rounding is exact, which
//     keeps sharply peaked rows accurate; O and the log-sum-exp are normalised by the one
//     fp32 sum of the probabilities.
#pragma once

#include "sm100_common.cuh"

namespace attn {

constexpr float kLn2 = 0.6931471805599453f;

struct FwdArgs {
  CUtensorMap tm_q;  // [B*Hq, Nq, d] bf16, box {64, 128, 1}
  CUtensorMap tm_k;  // [B*Hkv, Nk, d] bf16, box {64, BN, 1}
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // bf16 O [B*Hq, Nq, d], box {64, 32, 1}: stores of the two-tile kernel (d <= 128)
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
  // masks beyond causal: window > 0 hides keys older than `window` tokens (with causal);
  // block_mask (not null) is a [n_qtiles][nkt] map of 128x128 blocks, nonzero = visible
  int window;
  const uint8_t* block_mask;
  int nkt;  // ceil(Nk / 128)
  // failure-path testing only (-1 in every normal call): CTA dbg_stall_cta leaves its K/V
  // ring fill number dbg_stall_fill out, so the wait for it runs out after timeout_ns
  int dbg_stall_cta;
  int dbg_stall_fill;
};

// Is ring fill `fill` of this CTA the one a failure-path test leaves out?
__device__ __forceinline__ bool stalled_fill(int stall_cta, int stall_fill, int fill) {
  return stall_cta == (int)blockIdx.x && fill == stall_fill;
}

constexpr int kMaskBlock = 128;  // block size of the block-sparse map
constexpr int kUnitBand = 16;           // q-tile levels per band of the causal unit order
constexpr int kUnitBandMinTiles = 64;   // q-tiles from which the levels are banded
constexpr int kMaxVisits = 2048;  // blocks a CTA may visit under a block-sparse map

struct TileJob {
  int hq;    // query head
  int q0;    // first query row of the tile
  int rows;  // valid rows (0 if the tile lies past Nq)
  int jlo;   // first KV block the tile may visit
  int jhi;   // one past the last KV block the tile may visit (jlo >= jhi: none)
};

template <int BN, bool MASKS>
__device__ __forceinline__ TileJob make_tile(const FwdArgs& a, int hq, int q0) {
  TileJob t;
  t.hq = hq;
  t.q0 = q0;
  t.jlo = 0;
  t.jhi = 0;
  if (q0 >= a.Nq) {
    t.rows = 0;
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
  t.jhi = (int)((nkeys + BN - 1) / BN);
  if (MASKS && a.window > 0) {
    // first visible key of the tile's first row: q0 + (Nk - Nq) - window + 1
    long long first = (long long)q0 + a.Nk - a.Nq - a.window + 1;
    if (first < 0) first = 0;
    const long long jl = first / BN;
    t.jlo = (int)(jl < t.jhi ? jl : t.jhi);
  }
  return t;
}

// Does block j of this tile contain a hidden key for some row of the tile?
template <int BN, bool MASKS>
__device__ __forceinline__ bool block_needs_mask(const FwdArgs& a, const TileJob& t, int j) {
  long long hi = (long long)(j + 1) * BN;  // one past the block's last key
  if (hi > a.Nk) return true;
  if (a.causal && hi - 1 > (long long)t.q0 + a.Nk - a.Nq) return true;
  if (MASKS && a.window > 0 && (long long)j * BN < (long long)t.q0 + t.rows - 1 + a.Nk - a.Nq - a.window + 1) return true;
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

// Smallest visible key index for query row q (0 without a window).
__device__ __forceinline__ int row_key_low(const FwdArgs& a, int q) {
  if (a.window <= 0) return 0;
  long long lo = (long long)q + a.Nk - a.Nq - a.window + 1;
  if (lo < 0) lo = 0;
  if (lo > a.Nk) lo = a.Nk;
  return (int)lo;
}

// Does the tile visit KV block kb?  bits: the tile's row of the block-sparse map as a
// bitmap (bit mb = keys 128 mb .. 128 mb + 127), or null when there is none.
template <int BN>
__device__ __forceinline__ bool tile_visits(const uint32_t* bits, const TileJob& t, int kb) {
  if (kb < t.jlo || kb >= t.jhi) return false;
  if (bits == nullptr) return true;
  const int mb = kb * BN / kMaskBlock;
  return (bits[mb >> 5] >> (mb & 31)) & 1u;
}

// Smallest block >= kb the tile visits (t.jhi if none).
template <int BN>
__device__ __forceinline__ int next_visit(const uint32_t* bits, const TileJob& t, int kb) {
  if (kb < t.jlo) kb = t.jlo;
  if (bits == nullptr) return kb < t.jhi ? kb : t.jhi;
  while (kb < t.jhi) {
    const int mb = kb * BN / kMaskBlock;
    const uint32_t w = bits[mb >> 5] >> (mb & 31);
    if (w & 1u) return kb;
    const int skip = w ? __ffs(w) - 1 : 32 - (mb & 31);  // to the next set bit, or the next word
    kb = (mb + skip) * (kMaskBlock / BN);
  }
  return t.jhi;
}

// One warp writes the tile's row of the block-sparse map as a bitmap of nwords words.
__device__ __forceinline__ void build_row_bitmap(const FwdArgs& a, const TileJob& t, uint32_t* bits, int nwords) {
  const int lane = threadIdx.x & 31;
  const uint8_t* row = a.block_mask + (size_t)(t.q0 / kMaskBlock) * a.nkt;
  for (int i = 0; i < nwords; ++i) {
    const int mb = 32 * i + lane;
    const bool v = t.rows > 0 && mb < a.nkt && __ldg(&row[mb]) != 0;
    const uint32_t w = __ballot_sync(0xffffffffu, v);
    if (lane == 0) bits[i] = w;
  }
}

// ====================================================================================
// Kernel 1: two Q tiles per CTA (d = 64 or 128)
// ====================================================================================
//
// Warp roles (384 threads): warp 0 issues TMA loads, warp 1 issues the MMAs, warps 2-3
// turn a block-sparse map into per-tile bitmaps (else idle), warps 4-7 and 8-11 are the
// softmax warpgroups of tiles 0 and 1.  Each softmax thread owns one query row of its
// tile: all 128 scores of a block sit in its registers, so the row maximum needs no
// exchange between threads.  Twelve warps leave three per scheduler and up to 168
// registers a thread.
//
// P goes to shared memory (128-byte swizzled, K-major: the A operand of P V), not back
// over S.  So S_t is free as soon as the softmax has read it into registers, and the
// next S_t = Q_t K^T runs while the softmax still works on the current block: each
// tile's softmax steps follow one another without waiting for the tensor core, and
// the two tiles' softmaxes share the SM.  The MMA order per visited block u is
// S_0(u+1), S_1(u+1), P V_0(u), P V_1(u); the K/V ring is filled in the same order
// (K of block u+1 before V of block u).

template <int D>
struct PingPongCfg {
  static constexpr int BM = 128;
  static constexpr int BN = 128;
  static constexpr int THREADS = 384;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int NSTAGE = (D == 64) ? 8 : 3;  // K and V tiles share the ring
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = 2 * Q_BYTES;
  static constexpr int OFF_KV = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_BAR = OFF_KV + NSTAGE * KV_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int OFF_BITS = OFF_BAR + BAR_BYTES;  // block-sparse bitmaps [tile][64 words]
  static constexpr int BITS_WORDS = kMaxVisits / 32;
  static constexpr int SMEM = OFF_BITS + 2 * BITS_WORDS * 4;  // no alignment slack: the base is 1 KB aligned
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct PingPongBars {
  uint64_t q_full[2];
  uint64_t q_empty[2];  // the unit's last S_t = Q_t K^T is done: Q_t may be reloaded
  uint64_t s_full[2];   // S_t of the tile's next visit is in TMEM
  uint64_t s_free[2];   // the tile's softmax has read S_t (4 warps)
  uint64_t p_full[2];   // P_t is in shared memory and O_t is rescaled (4 warps)
  uint64_t o_done[2];   // one phase per P V of the tile
  uint64_t o_final[2];  // one phase: the tile's last P V is done
  uint64_t drain;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PingPongBars) <= PingPongCfg<128>::BAR_BYTES, "barrier area");

// A quarter of the probability pairs (kEmuMask) is computed on the FMA pipe (exp2_fma2)
// instead of the exp unit: per block the exp unit alone needs as many cycles as the
// tensor core, the bottleneck the FA4 page names for Blackwell (section "Softmax
// distribué et émulé").  More than a quarter costs more issue slots than it saves: the
// thread that issues the MMAs shares its scheduler with the softmax warps and is
// starved by FMA-heavy neighbours.
constexpr uint32_t kEmuMask = 0x88u;  // pairs 3 and 7 of each group of 8 (measured best of 0, 1/8, 2/8)

// p = 2^(s * sl2 + nmu) for NP pairs, packed to bf16 pairs in P; (a0 + a1) gets the
// fp32 sum.
template <uint32_t MASK, int NP>
__device__ __forceinline__ void exp_pairs(const float (&s)[2 * NP], float sl2, float nmu, uint32_t (&P)[NP],
                                          float& a0, float& a1) {
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    float y0, y1, p0, p1;
    fma2(y0, y1, s[2 * i], s[2 * i + 1], sl2, sl2, nmu, nmu);
    if ((MASK >> (i & 7)) & 1u) {
      exp2_fma2(p0, p1, y0, y1);
    } else {
      p0 = ex2(y0);
      p1 = ex2(y1);
    }
    add2(a0, a1, p0, p1);
    P[i] = pack_bf16x2(p0, p1);
  }
}

// Row r's probabilities (NP pairs: keys 0 .. 2NP-1 of the block) into the P tile,
// K-major with the 128-byte swizzle: keys 64c .. 64c+63 form chunk c (128 rows x 128
// bytes), and 16-byte granule g of row r sits at g ^ (r % 8).  A warp's store covers
// 32 rows x 16 bytes; within each group of 8 rows the granules land in distinct bank
// groups.
template <int NP>
__device__ __forceinline__ void store_p_row(uint32_t p_tile, int r, const uint32_t (&P)[NP]) {
  const uint32_t row = p_tile + (uint32_t)r * 128u;
#pragma unroll
  for (int g = 0; g < NP / 4; ++g)
    st_shared_v4(row + (uint32_t)((g >> 3) * (128 * 128)) + (uint32_t)(((g & 7) ^ (r & 7)) << 4), P[4 * g],
                 P[4 * g + 1], P[4 * g + 2], P[4 * g + 3]);
}

// Loads this thread's NCOL score columns of one block from TMEM, applies the mask and
// returns their maximum (log2 units).
template <bool LOW, int NCOL>
__device__ __forceinline__ float load_scores(uint32_t s_taddr, bool masked, int col_limit, int col_low, float sl2,
                                             float (&s)[NCOL]) {
  uint32_t r[NCOL];
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) tmem_ld32(s_taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
#pragma unroll
  for (int c = 0; c < NCOL; ++c) s[c] = __uint_as_float(r[c]);
  if (masked) {
#pragma unroll
    for (int c = 0; c < NCOL; ++c) s[c] = (c > col_limit || (LOW && c < col_low)) ? -INFINITY : s[c];
  }
  float x0 = max3(s[0], s[1], s[2]), x1 = max3(s[3], s[4], s[5]);
#pragma unroll
  for (int c = 6; c < NCOL - 2; c += 4) {
    x0 = max3(x0, s[c], s[c + 1]);
    x1 = max3(x1, s[c + 2], s[c + 3]);
  }
  return max3(x0, x1, fmaxf(s[NCOL - 2], s[NCOL - 1])) * sl2;
}

// All NC columns are loaded before the one wait: one TMEM round trip, not NC / 32.
template <int NC>
__device__ __forceinline__ void rescale_cols(uint32_t o_taddr, float alpha) {
  uint32_t r[NC];
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) tmem_ld32(o_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
#pragma unroll
  for (int i = 0; i < NC; i += 2) {
    float u0 = __uint_as_float(r[i]), u1 = __uint_as_float(r[i + 1]);
    mul2(u0, u1, alpha, alpha);
    r[i] = __float_as_uint(u0);
    r[i + 1] = __float_as_uint(u1);
  }
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) tmem_st32(o_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * c]));
}

// Epilogue for NC columns of one row: O / l to global (bf16 or fp32).
template <int NC>
__device__ __forceinline__ void store_cols(const FwdArgs& a, uint32_t o_taddr, bool have_o, bool valid,
                                           size_t elem_off, float l) {
  const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
  for (int c = 0; c < NC / 32; ++c) {
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
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + elem_off + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                               __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + elem_off + c * 32);
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
}

// Row r of O / l as bf16 into a 128-row tile in the P layout (128-byte swizzled
// 64-column chunks), from where TMA writes it to global memory: one 16-byte store per
// 8 columns, conflict-free like the P stores, instead of 32 rows' worth of scattered
// global stores per warp instruction.
template <int D>
__device__ __forceinline__ void stage_o_row(uint32_t tile, int r, uint32_t o_taddr, bool have_o, float l) {
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const uint32_t row = tile + (uint32_t)r * 128u;
  uint32_t o[D];
  if (have_o) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) tmem_ld32(o_taddr + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32 * c]));
#pragma unroll
    for (int c = 0; c < D / 32; ++c) tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&o[32 * c]));
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0u;
  }
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const uint32_t* v = o + 32 * c;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * i]) * inv, __uint_as_float(v[8 * j + 2 * i + 1]) * inv);
      const int g = (c & 1) * 4 + j;  // 16-byte granule within the 64-column chunk c / 2
      st_shared_v4(row + (uint32_t)((c >> 1) * (128 * 128)) + (uint32_t)((g ^ (r & 7)) << 4), w[0], w[1], w[2],
                   w[3]);
    }
  }
}

// Work unit u of the two-tile kernel: two 128-row Q tiles and the KV head they read.
// Causal: heaviest q-tiles first (longest-processing-time order).  Otherwise all units
// weigh about the same; consecutive units share a head so that the K/V tiles streamed at
// the same time stay in L2.
template <int BN, bool MASKS>
__device__ __forceinline__ void unit_tiles(const FwdArgs& a, int u, int& b, int& kvh, TileJob (&tj)[2]) {
  if (a.pair_heads) {
    const int hp_n = a.Hq / 2;
    int qt, rem;
    if (a.causal) {
      // Heaviest first: q-tile levels from the top.  Long sequences take the levels in
      // bands of kUnitBand, and within a band the (batch, KV head) groups one after
      // another, so that a round of CTAs streams the K/V of about two KV heads instead of
      // all of them and their re-reads stay in L2 (16K causal GQA: DRAM reads 656 -> 508
      // MB per launch, time unchanged within 1 %).  With fewer levels, one level a band.
      const int per_level = a.B * hp_n;
      const int L = a.n_qtiles >= kUnitBandMinTiles ? kUnitBand : 1;
      const int band = u / (L * per_level);
      const int in_band = u % (L * per_level);
      const int lv_hi = a.n_qtiles - 1 - band * L;
      const int nl = min(L, lv_hi + 1);  // the last band may be shorter
      const int P = a.group / 2;         // head pairs of one KV head
      const int gkv = in_band / (nl * P);
      const int r2 = in_band % (nl * P);
      qt = lv_hi - r2 / P;
      rem = gkv * P + r2 % P;
    } else {
      qt = u % a.n_qtiles;
      rem = u / a.n_qtiles;
    }
    b = rem / hp_n;
    const int h0 = 2 * (rem % hp_n);
    tj[0] = make_tile<BN, MASKS>(a, h0, qt * 128);
    tj[1] = make_tile<BN, MASKS>(a, h0 + 1, qt * 128);
  } else {
    const int nqp = (a.n_qtiles + 1) / 2;
    int qp, rem;
    if (a.causal) {
      qp = nqp - 1 - u / (a.B * a.Hq);
      rem = u % (a.B * a.Hq);
    } else {
      qp = u % nqp;
      rem = u / nqp;
    }
    b = rem / a.Hq;
    const int h = rem % a.Hq;
    tj[0] = make_tile<BN, MASKS>(a, h, (2 * qp) * 128);
    tj[1] = make_tile<BN, MASKS>(a, h, (2 * qp + 1) * 128);
  }
  kvh = tj[0].hq / a.group;
}

// Persistent: in round r CTA c takes unit r G + c (r even) or r G + G - 1 - c (r odd),
// G = gridDim.x.  Every role walks the same unit
// sequence and every barrier keeps counting across units, so the next unit's Q and K
// loads and its first S = Q K^T run while the current unit's last softmax step and
// epilogue are still going.  With a block-sparse map each CTA takes exactly one unit
// (the map row becomes bitmaps once, before the roles start).
//
// MASKS = false: causal or no mask only (window = 0, block_mask = null); that instance
// carries none of the window and block-map logic.
template <int D, bool MASKS>
__global__ void __launch_bounds__(384, 1) attn_fwd_pingpong_kernel(const __grid_constant__ FwdArgs a) {
  using C = PingPongCfg<D>;
  constexpr int BN = C::BN;
  extern __shared__ __align__(1024) uint8_t smem_pp[];
  uint8_t* smem = smem_pp;
  if (smem_u32(smem) & 1023u) {  // the layout has no slack to realign (uniform exit, nothing started)
    if (threadIdx.x == 0) latch_status(ATTN_ERR_ALIGNMENT);
    return;
  }
  PingPongBars* bars = reinterpret_cast<PingPongBars*>(smem + C::OFF_BAR);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(smem + C::OFF_BITS);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool use_bits = MASKS && a.block_mask != nullptr;

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
  int b, kvh;
  TileJob tj[2];
  if (use_bits && (warp == 2 || warp == 3)) {  // one unit per CTA here (host launch)
    unit_tiles<BN, MASKS>(a, blockIdx.x, b, kvh, tj);
    build_row_bitmap(a, warp == 3 ? tj[1] : tj[0], bitmaps + (warp - 2) * C::BITS_WORDS, C::BITS_WORDS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sP = smem_u32(smem + C::OFF_P);
  const uint32_t sKV = smem_u32(smem + C::OFF_KV);
  const uint32_t* bits0 = use_bits ? bitmaps : nullptr;
  const uint32_t* bits1 = use_bits ? bitmaps + C::BITS_WORDS : nullptr;

  // visit walk of the current unit: the union of both tiles' visited blocks, in order
  constexpr int kDone = 0x7fffffff;
  auto tile_next = [&](int t, int kb) -> int {  // kDone if the tile visits nothing >= kb
    const TileJob& j = t ? tj[1] : tj[0];
    const int n = next_visit<BN>(t ? bits1 : bits0, j, kb);
    return n < j.jhi ? n : kDone;
  };
  auto union_next = [&](int kb) -> int { return min(tile_next(0, kb), tile_next(1, kb)); };
  auto visits = [&](int t, int kb) -> bool { return tile_visits<BN>(t ? bits1 : bits0, t ? tj[1] : tj[0], kb); };
  // unit of round rd: rounds alternate direction over the CTAs, so that with the units
  // sorted heaviest first every CTA's total stays close to the mean
  auto snake_unit = [&](int rd) -> int {
    return rd * (int)gridDim.x + ((rd & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };

  if (warp == 0) {
    // ================= TMA producer.  Per unit: the Q tiles (each once the previous
    // unit's last S of that tile is done), then K(u0), and per visited block u:
    // K(next block), V(u)
    if (lane == 0) {
      tma_prefetch_map(&a.tm_q);
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
      const uint64_t pol = l2_policy_evict_last();
      int seq = 0;
      int nql[2] = {0, 0};  // Q loads of each tile so far
      auto push = [&](int kb, int kv) -> bool {
        const int st = seq % C::NSTAGE;
        const int use = seq / C::NSTAGE;
        if (use > 0 && !mbar_wait(&bars->kv_empty[st], (use - 1) & 1, abort_flag, a.timeout_ns)) return false;
        if (stalled_fill(a.dbg_stall_cta, a.dbg_stall_fill, seq)) {  // never armed, never completes
          ++seq;
          return true;
        }
        mbar_arrive_expect_tx(&bars->kv_full[st], C::KV_BYTES);
        const CUtensorMap* map = kv ? &a.tm_v : &a.tm_k;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d_hint(smem + C::OFF_KV + st * C::KV_BYTES + c * (BN * 128), map, &bars->kv_full[st], c * 64,
                           kb * BN, b * a.Hkv + kvh, pol);
        ++seq;
        return true;
      };
      bool ok = true;
      for (int rd = 0; rd * (int)gridDim.x < a.n_units && ok; ++rd) {
        const int u = snake_unit(rd);
        if (u >= a.n_units) continue;
        unit_tiles<BN, MASKS>(a, u, b, kvh, tj);
        for (int t = 0; t < 2 && ok; ++t) {
          if (tile_next(t, 0) == kDone) continue;
          if (nql[t] > 0 && !mbar_wait(&bars->q_empty[t], (nql[t] - 1) & 1, abort_flag, a.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->q_full[t], C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + C::OFF_Q + t * C::Q_BYTES + c * (128 * 128), &a.tm_q, &bars->q_full[t], c * 64,
                        tj[t].q0, b * a.Hq + tj[t].hq);
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
      // drain: every copy issued must have landed before the CTA may exit (a Q tile is
      // reloaded only after the previous load was consumed, so only the last can fly)
      for (int t = 0; t < 2; ++t)
        if (nql[t] > 0) mbar_wait(&bars->q_full[t], (nql[t] - 1) & 1, abort_flag, a.timeout_ns, false);
      for (int st = 0; st < C::NSTAGE && st < seq; ++st) {
        const int last_use = (seq - 1 - st) / C::NSTAGE;  // index of the last fill of stage st
        if (stalled_fill(a.dbg_stall_cta, a.dbg_stall_fill, st + last_use * C::NSTAGE)) continue;
        mbar_wait(&bars->kv_full[st], last_use & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer.  Consumes the ring in the producer's order.  S_t of a
    // tile's next visit waits until the tile's softmax has read S_t (s_free); P V_t(u)
    // waits for P_t (p_full).  Barrier phases count each tile's visits over all units.
    // The whole warp runs this loop (waits, descriptors, bookkeeping are warp-uniform)
    // and one elected lane issues the MMAs and commits: the issuing thread shares its
    // scheduler with busy softmax warps, so each MMA should cost it few instructions.
    auto stage_of = [&](int seq) { return seq % C::NSTAGE; };
    auto parity_of = [&](int seq) { return (uint32_t)((seq / C::NSTAGE) & 1); };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, a.timeout_ns));
    };
    const Desc dq[2] = {desc_sw128(sQ, 16, 1024), desc_sw128(sQ + C::Q_BYTES, 16, 1024)};
    const Desc dp[2] = {desc_sw128(sP, 16, 1024), desc_sw128(sP + C::P_BYTES, 16, 1024)};
    const Desc dk0 = desc_sw128(sKV, 16, 1024);
    const Desc dv0 = desc_sw128(sKV, BN * 128, 1024);
    auto kdesc = [&](int seq) { return Desc{dk0.lo + (uint32_t)(stage_of(seq) * (C::KV_BYTES >> 4)), dk0.hi}; };
    auto vdesc = [&](int seq) { return Desc{dv0.lo + (uint32_t)(stage_of(seq) * (C::KV_BYTES >> 4)), dv0.hi}; };
    int seq = 0;
    int nqk[2] = {0, 0}, npv[2] = {0, 0}, nql[2] = {0, 0};
    bool ok = true;
    // S_t(kb) = Q_t K(kb)^T for the tiles that visit kb; K(kb) is ring entry seq
    auto issue_s = [&](int kb) -> bool {
      if (!wait_all(&bars->kv_full[stage_of(seq)], parity_of(seq))) return false;
      const Desc dk = kdesc(seq);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!visits(t, kb)) continue;
        if (nqk[t] > 0 && !wait_all(&bars->s_free[t], (nqk[t] - 1) & 1)) return false;
        const bool last = tile_next(t, kb + 1) == kDone;  // the unit's last S of this tile
        if (elect_one()) {
          tc_fence_after();
          issue_qk_w<D, BN>(tmem + (t ? C::COL_S1 : C::COL_S0), dq[t], dk);
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
      unit_tiles<BN, MASKS>(a, u, b, kvh, tj);
      int kb = union_next(0);
      if (kb == kDone) continue;
      int upv[2] = {0, 0};  // P V of each tile in this unit (the first one overwrites O_t)
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
        // O_t += P_t(kb) V(kb)
        if (!wait_all(&bars->kv_full[stage_of(seq)], parity_of(seq))) {
          ok = false;
          break;
        }
        const Desc dv = vdesc(seq);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || !visits(t, kb)) continue;
          if (!wait_all(&bars->p_full[t], npv[t] & 1)) {
            ok = false;
            continue;
          }
          const bool last = tile_next(t, kb + 1) == kDone;  // the tile's last visit of the unit
          if (elect_one()) {
            tc_fence_after();
            issue_pv_w<D, BN>(tmem + (t ? C::COL_O1 : C::COL_O0), dp[t], dv, upv[t] > 0);
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
    // every MMA must be finished before TMEM is released
    if (elect_one()) tc_commit(&bars->drain);
    __syncwarp();
    mbar_wait(&bars->drain, 0, abort_flag, a.timeout_ns, false);
  } else if (warp >= 4) {
    // ================= softmax: warps 4 + 4t .. 7 + 4t own tile t, one row per thread
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;       // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;  // row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + (t ? C::COL_S1 : C::COL_S0);
    const uint32_t o_addr = tmem + lane_off + (t ? C::COL_O1 : C::COL_O0);
    const uint32_t p_tile = sP + t * C::P_BYTES;
    int k = 0;         // this tile's visits over all units (barrier phases)
    int nfin = 0;      // units in which this tile had visits (o_final phases)
    bool fail = false;  // a wait gave up (the warp decides as one)
    // this warp's last O store (bf16 O) still reads its rows of P_t: lane 0 waits for
    // that before the rows are written again
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
      unit_tiles<BN, MASKS>(a, u, b, kvh, tj);
      const TileJob job = t ? tj[1] : tj[0];  // selects, not a dynamic index (no local memory)
      const int q = job.q0 + r;
      const int khi = row_key_limit(a, q);
      const int klo = MASKS ? row_key_low(a, q) : 0;
      float m = -INFINITY, l = 0.f;
      int kl = 0;  // visits in this unit
      for (int kb = tile_next(t, 0); kb != kDone; kb = tile_next(t, kb + 1), ++k, ++kl) {
        if (__any_sync(0xffffffffu, !mbar_wait(&bars->s_full[t], k & 1, abort_flag, a.timeout_ns) || *abort_flag)) {
          fail = true;
          break;
        }
        tc_fence_after();
        float s[BN];
        const bool masked = block_needs_mask<BN, MASKS>(a, job, kb);
        const float mx = load_scores<MASKS, BN>(s_addr, masked, khi - kb * BN, klo - kb * BN, a.scale_log2, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[t]);  // S_t may be overwritten
        // exact running maximum: whenever it grows, O is rescaled before this block's P V,
        // so the row's largest probability is exactly 1 and its bf16 rounding is exact
        float alpha = 1.0f;
        if (mx > m) {           // false while nothing is visible (mx = -inf)
          alpha = ex2(m - mx);  // 0 when m = -inf
          m = mx;
        }
        const float nmu = (m == -INFINITY) ? 0.0f : -m;
        // masked blocks take the same path: a hidden key (-inf) comes out of the FMA-pipe
        // exponential as 2^-125 instead of 0, 2^-100 or less relative to any visible
        // probability of the row; while the row has seen no visible key (m = -inf) those
        // values are wiped by the factor 0 at its first visible key, and a row that never
        // sees one is written as O = 0, LSE = -inf below
        uint32_t P[BN / 2];
        float a0 = 0.f, a1 = 0.f;
        exp_pairs<kEmuMask, BN / 2>(s, a.scale_log2, nmu, P, a0, a1);
        l = l * alpha + (a0 + a1);
        // P V of the tile's previous visit (of this unit or the last) must be done: it
        // reads P_t, and O_t may be rescaled.  (Warp-uniform decision: the stores and
        // TMEM accesses below are per warp.)
        if (!__all_sync(0xffffffffu,
                        k == 0 || mbar_wait(&bars->o_done[t], (k - 1) & 1, abort_flag, a.timeout_ns))) {
          fail = true;
          break;
        }
        settle_store();
        store_p_row<BN / 2>(p_tile, r, P);
        fence_proxy_async_smem();
        if (kl > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
          tc_fence_after();
          rescale_cols<D>(o_addr, alpha);
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
        // the unit's last P V; the next unit's first P V (which overwrites O_t) waits for
        // this warp's next p_full, given after these TMEM loads
        ok = mbar_wait(&bars->o_final[t], nfin & 1, abort_flag, a.timeout_ns);
        tc_fence_after();
        ++nfin;
      }
      ok = __all_sync(0xffffffffu, ok);  // the TMEM loads of the epilogue are per warp
      if (!ok) {
        fail = true;
        break;
      }
      const bool valid = r < job.rows;
      const size_t row = ((size_t)b * a.Hq + job.hq) * (size_t)a.Nq + (size_t)(valid ? q : 0);
      if (m == -INFINITY) l = 0.f;  // no visible key: O = 0, LSE = -inf
      if (a.o_f32) {
        store_cols<D>(a, o_addr, have_o, valid, row * D, l);
      } else if (job.rows > quad * 32) {  // the warp has valid rows (warp-uniform)
        // P_t is free (the tile's last P V of the unit is done, or it had none): stage
        // this warp's 32 rows there and store them with TMA (rows past Nq are clipped)
        settle_store();
        stage_o_row<D>(p_tile, r, o_addr, have_o, l);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_store_3d(&a.tm_o, p_tile + (uint32_t)(c * (128 * 128) + quad * 32 * 128), c * 64, job.q0 + quad * 32,
                         b * a.Hq + job.hq);
          bulk_commit();
        }
        store_pending = true;
      }
      if (valid && a.lse != nullptr) a.lse[row] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
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
