// decode_sm100.cuh — one decode step over a paged KV cache, for sm_100a.
//
// The method: the new token's query attends to every cached key/value of its sequence
// (ranksignal.fr, "FlashAttention et PagedAttention : à quoi servent-elles ?", section
// "Le cache KV, ce locataire qui grossit"); the cache is stored in fixed-size pages
// found through a per-sequence table (same page, section "PagedAttention : ranger par
// pages plutôt que d'un seul tenant").  Paging changes where the data lives, not what
// is computed.
//
// The step is bound by HBM bandwidth (every cached K and V byte is read once, about
// 8 FLOP per byte), so the design streams the cache at full bandwidth:
//   * plan kernel: one CTA turns seq_lens into a prefix of work chunks per sequence.
//   * split kernel (persistent, about 3 CTAs per SM): a work item is (sequence, chunk of
//     CHUNK_TOK tokens, KV head, group of up to 16 query heads).  A producer warp walks
//     the block table and gathers 16-token pieces of K and V pages with TMA (128-byte
//     swizzled, 16-byte aligned bulk transfers) into a ring of shared-memory stages; the
//     next item's pieces are fetched while the current one is still being consumed.
//     Four consumer warps each own every fourth piece (and their own ring stages) and
//     keep their own online-softmax state.  All query heads of a KV group share one K/V read ("pack-GQA"): they form
//     the 16 rows of a warp-level bf16 MMA (m16n8k16), for Q K^T and for P V.  The work
//     is too small for the tcgen05 path to pay (M would be 8 query heads); the tensor
//     pipe only has to keep up with HBM here.
//     At the end of an item each warp writes its state as one partial (O normalised by
//     its own sum, plus its log2-sum-exp) to the workspace; the warps never wait for one
//     another (measured: a shared-memory merge of the four states at every item cost
//     about a tenth of the bandwidth).
//   * merge kernel: per (sequence, query head) the partials are combined with weights
//     exp(lse_c - lse), which is exact because the running max/sum statistics of the
//     online softmax compose associatively.
#pragma once

#include "sm100_common.cuh"

namespace attn {

constexpr int kDecTok = 16;         // tokens per piece (one MMA k-step)
constexpr int kDecWarps = 4;        // consumer warps per CTA
constexpr int kDecChunkTok = 2048;  // tokens per work item (measured: 512 -> 3.9, 1024 -> 5.0, 2048 -> 5.5 TB/s)

struct DecArgs {
  CUtensorMap tm_k;  // pool viewed as [num_pages*Hkv, page_size, d] bf16, box {64, 16, 1}
  CUtensorMap tm_v;
  const __nv_bfloat16* q;      // [S, Hq, d]
  const int32_t* block_table;  // [S, max_pages]
  const int32_t* seq_lens;     // [S]
  __nv_bfloat16* o;            // [S, Hq, d]
  float* lse;                  // [S, Hq] or null
  int* chunk_prefix;           // workspace: [S + 1]
  int4* item_map;              // workspace: [total chunks] = {sequence, chunk in sequence, sequence length, 0}
  float* part_o;               // workspace: [S * max_chunks * Hq * d]
  float* part_lse;             // workspace: [S * max_chunks * Hq]   (log2 units)
  int S, Hq, Hkv, group, n_hgroups, page_size, num_pages, max_pages, max_chunks;
  float scale_log2;
  uint64_t timeout_ns;
  // failure-path testing only (-1 in every normal call): CTA dbg_stall_cta leaves its
  // piece number dbg_stall_piece out, so the wait for it runs out after timeout_ns
  int dbg_stall_cta;
  int dbg_stall_piece;
};

// ------------------------------------------------------------------ plan

// chunk_prefix[s] = number of work chunks of sequences < s (the merge finds a sequence's
// partials by chunk index), and item_map[k] describes work chunk k (one CTA, any S).  With
// the map a work item's sequence is one load, not a search: dependent loads are slow while
// the split pass saturates HBM.
//
// The chunks are listed longest first, because the split kernel hands them out round-robin:
// every full chunk (kDecChunkTok tokens) in sequence order, then each sequence's shorter
// last chunk, longest first (ties by sequence; in sequence order beyond kPlanSortMax
// sequences), so that the last rounds get the short chunks.
constexpr int kPlanSortMax = 2048;

// Block-wide exclusive scan (every thread of the block calls it with its value): returns
// *carry plus the sum of the values of the lower threads, and adds the block's total to
// *carry.  warp_sums: 32 ints of shared memory.
__device__ __forceinline__ int plan_scan(int v, int* carry, int* warp_sums) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_sums[lane] = t;  // inclusive scan of the warp totals
  }
  __syncthreads();
  const int before = *carry + (w > 0 ? warp_sums[w - 1] : 0) + (x - v);
  __syncthreads();
  if (threadIdx.x == 0) *carry += warp_sums[nw - 1];
  __syncthreads();
  return before;
}

__global__ void attn_decode_plan_kernel(const int32_t* __restrict__ seq_lens, int S, int max_tokens,
                                        int* __restrict__ chunk_prefix, int4* __restrict__ item_map) {
  __shared__ int carry_all, carry_full, carry_part;
  __shared__ int warp_sums[32];
  __shared__ int tail_len[kPlanSortMax];  // tokens in each sequence's last, shorter chunk (0: none)
  if (threadIdx.x == 0) carry_all = carry_full = carry_part = 0;
  __syncthreads();
  // pass 1: the prefix of all chunks, and the full chunks in sequence order
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int len = 0;
    if (s < S) {
      len = seq_lens[s];
      if (len < 0 || len > max_tokens) {
        latch_status(ATTN_ERR_INVALID_ARG);
        len = 0;
      }
    }
    const int n_full = len / kDecChunkTok;
    const int tail = len % kDecChunkTok;
    const int before_all = plan_scan(n_full + (tail != 0 ? 1 : 0), &carry_all, warp_sums);
    const int before_full = plan_scan(n_full, &carry_full, warp_sums);
    if (s < S) {
      chunk_prefix[s] = before_all;
      for (int c = 0; c < n_full; ++c) item_map[before_full + c] = make_int4(s, c, len, 0);
      if (S <= kPlanSortMax) tail_len[s] = tail;
    }
  }
  __syncthreads();
  const int total_full = carry_full;
  if (threadIdx.x == 0) chunk_prefix[S] = carry_all;
  // pass 2: the shorter last chunks after the full ones
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    int len = 0;
    if (s < S) {
      len = seq_lens[s];
      if (len < 0 || len > max_tokens) len = 0;
    }
    const int tail = len % kDecChunkTok;
    int slot;
    if (S <= kPlanSortMax) {  // rank by (length descending, sequence)
      slot = 0;
      if (tail != 0)
        for (int t = 0; t < S; ++t) {
          const int o = tail_len[t];
          slot += (o > tail || (o == tail && t < s)) ? 1 : 0;
        }
    } else {
      slot = plan_scan(tail != 0 ? 1 : 0, &carry_part, warp_sums);
    }
    if (s < S && tail != 0) item_map[total_full + slot] = make_int4(s, len / kDecChunkTok, len, 0);
  }
}

// ------------------------------------------------------------------ split kernel

template <int D>
struct DecCfg {
  static constexpr int THREADS = (kDecWarps + 1) * 32;
  static constexpr int PIECE_BYTES = kDecTok * D * 2;  // 16 tokens of K (or V) for one KV head
  static constexpr int STAGE_BYTES = 2 * PIECE_BYTES;
  static constexpr int NST = (D == 256) ? 4 : 8;        // multiple of kDecWarps
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_MISC = NST * STAGE_BYTES;
  static constexpr int SMEM = OFF_MISC + 1024 + 1024;
  static constexpr int CTAS_PER_SM = (D == 256) ? 2 : 3;
};

struct DecMisc {
  uint64_t full[8];
  uint64_t empty[8];
  int32_t stage_ok[8];   // 1 = the stage holds valid K/V, 0 = its page was out of range
  int abort_flag;
};

struct DecItem {
  int s, c, kvh, hg;
  int tok0, ntok;  // first token of the chunk and tokens in it
};

__device__ __forceinline__ int4 item_info(const DecArgs& a, int f) {
  return __ldg(&a.item_map[f / (a.Hkv * a.n_hgroups)]);
}

__device__ __forceinline__ DecItem decode_item(const DecArgs& a, int f, int4 info) {
  DecItem it;
  const int rem = f % (a.Hkv * a.n_hgroups);
  it.kvh = rem / a.n_hgroups;
  it.hg = rem % a.n_hgroups;
  it.s = info.x;
  it.c = info.y;
  it.tok0 = it.c * kDecChunkTok;
  it.ntok = min(kDecChunkTok, info.z - it.tok0);
  return it;
}

template <int D>
__global__ void __launch_bounds__(DecCfg<D>::THREADS, DecCfg<D>::CTAS_PER_SM)
    attn_decode_split_kernel(const __grid_constant__ DecArgs a) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DecMisc* misc = reinterpret_cast<DecMisc*>(smem + C::OFF_MISC);
  volatile int* abort_flag = &misc->abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int n_items = __ldg(&a.chunk_prefix[a.S]) * a.Hkv * a.n_hgroups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&misc->full[s], 1);
      mbar_init(&misc->empty[s], 1);
    }
    misc->abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kDecWarps) {
    // ================= producer: gather pieces of K/V pages through the block table
    const uint64_t pol = l2_policy_evict_first();
    if (lane == 0 && a.num_pages > 0) {
      tma_prefetch_map(&a.tm_k);
      tma_prefetch_map(&a.tm_v);
    }
    // The pieces are issued group by group (32 pieces of one item).  The page ids of the
    // next group, and the item record of the item after the next, are loaded one step
    // ahead so that their latency hides behind the current group's copies.
    const int ppp = a.page_size / kDecTok;  // pieces per page
    auto group_pages = [&](const DecItem& it, int p0) -> int {
      const int p = p0 + lane;
      const int npieces = (it.ntok + kDecTok - 1) / kDecTok;
      if (p >= npieces) return -1;
      return __ldg(&a.block_table[(size_t)it.s * a.max_pages + (it.tok0 / kDecTok + p) / ppp]);
    };
    int gp = 0;  // pieces issued so far by this CTA
    bool ok = true;
    int f = blockIdx.x;
    if (f < n_items) {
      DecItem it = decode_item(a, f, item_info(a, f));
      int4 info_next = f + (int)gridDim.x < n_items ? item_info(a, f + gridDim.x) : make_int4(0, 0, 0, 0);
      int p0 = 0;
      int pages = group_pages(it, 0);
      while (ok) {
        const int npieces = (it.ntok + kDecTok - 1) / kDecTok;
        // where the next group is, and its page ids (in flight while this group issues)
        int nf = f, np0 = p0 + 32;
        DecItem nit = it;
        if (np0 >= npieces) {
          nf = f + gridDim.x;
          np0 = 0;
          if (nf < n_items) nit = decode_item(a, nf, info_next);
        }
        const bool more = nf < n_items;
        const int next_pages = more ? group_pages(nit, np0) : -1;
        const int cnt = min(32, npieces - p0);
        for (int i = 0; i < cnt; ++i) {
          const int pg = __shfl_sync(0xffffffffu, pages, i);
          const int st = gp % C::NST;
          const int use = gp / C::NST;
          const bool stall = a.dbg_stall_cta == (int)blockIdx.x && gp == a.dbg_stall_piece;
          if (lane == 0) {
            if (use > 0 && !mbar_wait(&misc->empty[st], (use - 1) & 1, abort_flag, a.timeout_ns)) ok = false;
            if (ok && !stall) {
              const bool good = pg >= 0 && pg < a.num_pages;
              misc->stage_ok[st] = good ? 1 : 0;
              if (good) {
                const int piece_in_page = ((it.tok0 / kDecTok) + p0 + i) % ppp;
                const int y = piece_in_page * kDecTok;
                const int z = pg * a.Hkv + it.kvh;
                mbar_arrive_expect_tx(&misc->full[st], C::STAGE_BYTES);
                uint8_t* dst = smem + C::OFF_RING + st * C::STAGE_BYTES;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                  tma_load_3d_hint(dst + c * (kDecTok * 128), &a.tm_k, &misc->full[st], c * 64, y, z, pol);
                  tma_load_3d_hint(dst + C::PIECE_BYTES + c * (kDecTok * 128), &a.tm_v, &misc->full[st], c * 64,
                                   y, z, pol);
                }
              } else {
                latch_status(ATTN_ERR_BAD_PAGE);
                mbar_arrive(&misc->full[st]);
              }
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          ++gp;
        }
        if (!more) break;
        if (nf != f) {
          const int nn = nf + gridDim.x;
          info_next = nn < n_items ? item_info(a, nn) : make_int4(0, 0, 0, 0);
        }
        f = nf;
        p0 = np0;
        it = nit;
        pages = next_pages;
      }
    }
    if (lane == 0) {  // drain copies still in flight
      for (int st = 0; st < C::NST && st < gp; ++st) {
        const int last_use = (gp - 1 - st) / C::NST;
        if (a.dbg_stall_cta == (int)blockIdx.x && st + last_use * C::NST == a.dbg_stall_piece) continue;
        mbar_wait(&misc->full[st], last_use & 1, abort_flag, a.timeout_ns, false);
      }
    }
  } else {
    // ================= consumers.  Piece gp of the CTA's stream goes to warp gp % 4 and
    // ring stage gp % NST, so each warp owns the stages w, w + 4, ...: every wait on a
    // stage follows the same warp's wait on that stage's previous use, which keeps the
    // phase parity unambiguous without any barrier between the warps.  Each warp keeps
    // its own online-softmax state for the item and writes it as one partial (O
    // normalised by its own sum, plus its log2-sum-exp); the merge kernel combines the
    // partials, so the warps never wait for one another.
    const int g = lane >> 2;  // row (query head within the group) of the MMA fragments
    const int t = lane & 3;
    constexpr int NT = D / 8;  // n-tiles of the P V product
    const uint32_t ring = smem_u32(smem + C::OFF_RING);
    int gp_base = 0;
    bool ok = true;
    for (int f = blockIdx.x; f < n_items && ok; f += gridDim.x) {
      const DecItem it = decode_item(a, f, item_info(a, f));
      const int npieces = (it.ntok + kDecTok - 1) / kDecTok;
      const int hq0 = it.kvh * a.group + it.hg * 16;
      const int nrows = min(16, a.group - it.hg * 16);

      // A fragments of Q (rows g and g+8), kept in registers for the whole item
      uint32_t qa[D / 16][4];
      {
        const __nv_bfloat16* qb = a.q + ((size_t)it.s * a.Hq + hq0) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int c0 = ks * 16 + 2 * t;
          qa[ks][0] = g < nrows ? *reinterpret_cast<const uint32_t*>(qb + (size_t)g * D + c0) : 0u;
          qa[ks][1] = g + 8 < nrows ? *reinterpret_cast<const uint32_t*>(qb + (size_t)(g + 8) * D + c0) : 0u;
          qa[ks][2] = g < nrows ? *reinterpret_cast<const uint32_t*>(qb + (size_t)g * D + c0 + 8) : 0u;
          qa[ks][3] = g + 8 < nrows ? *reinterpret_cast<const uint32_t*>(qb + (size_t)(g + 8) * D + c0 + 8) : 0u;
        }
      }
      float oc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g+8

      // this warp's pieces of the item: global piece indices gp with gp % 4 == warp
      for (int i = (warp - gp_base % kDecWarps + kDecWarps) % kDecWarps; i < npieces; i += kDecWarps) {
        const int gp = gp_base + i;
        const int st = gp % C::NST;
        if (!mbar_wait(&misc->full[st], (gp / C::NST) & 1, abort_flag, a.timeout_ns)) {
          ok = false;
          break;
        }
        if (misc->stage_ok[st]) {
          const uint32_t sK = ring + st * C::STAGE_BYTES;
          const uint32_t sV = sK + C::PIECE_BYTES;
          // S = Q K^T for 16 keys: two n-tiles of 8 keys
          float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int mi = lane >> 3, rr = lane & 7;
            const int key = (mi >> 1) * 8 + rr;
            const int unit = 2 * (ks & 3) + (mi & 1);
            const uint32_t addr = sK + (ks >> 2) * (kDecTok * 128) + key * 128 + ((unit ^ (key & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(addr, b0, b1, b2, b3);
            mma_16816(sc[0], qa[ks], b0, b1);
            mma_16816(sc[1], qa[ks], b2, b3);
          }
          // mask keys past the sequence end (only in the chunk's last piece)
          const int key0 = it.tok0 + i * kDecTok;
          const int len = it.tok0 + it.ntok;
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            const int k0 = key0 + n * 8 + 2 * t;
            if (k0 >= len) { sc[n][0] = -INFINITY; sc[n][2] = -INFINITY; }
            if (k0 + 1 >= len) { sc[n][1] = -INFINITY; sc[n][3] = -INFINITY; }
          }
          // online softmax, exact running max (rows g: c0,c1; rows g+8: c2,c3)
          float x0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
          float x1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
          x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 1));
          x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, 2));
          x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 1));
          x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, 2));
          const float n0 = fmaxf(m0, x0 * a.scale_log2);
          const float n1 = fmaxf(m1, x1 * a.scale_log2);
          const float al0 = (n0 == -INFINITY) ? 1.f : ex2(m0 - n0);
          const float al1 = (n1 == -INFINITY) ? 1.f : ex2(m1 - n1);
          m0 = n0;
          m1 = n1;
          const float u0 = (m0 == -INFINITY) ? 0.f : m0;
          const float u1 = (m1 == -INFINITY) ? 0.f : m1;
          float p[2][4];
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            p[n][0] = ex2(fmaf(sc[n][0], a.scale_log2, -u0));
            p[n][1] = ex2(fmaf(sc[n][1], a.scale_log2, -u0));
            p[n][2] = ex2(fmaf(sc[n][2], a.scale_log2, -u1));
            p[n][3] = ex2(fmaf(sc[n][3], a.scale_log2, -u1));
          }
          l0 = l0 * al0 + (p[0][0] + p[0][1] + p[1][0] + p[1][1]);
          l1 = l1 * al1 + (p[0][2] + p[0][3] + p[1][2] + p[1][3]);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            oc[n][0] *= al0;
            oc[n][1] *= al0;
            oc[n][2] *= al1;
            oc[n][3] *= al1;
          }
          uint32_t pa[4];
          pa[0] = pack_bf16x2(p[0][0], p[0][1]);
          pa[1] = pack_bf16x2(p[0][2], p[0][3]);
          pa[2] = pack_bf16x2(p[1][0], p[1][1]);
          pa[3] = pack_bf16x2(p[1][2], p[1][3]);
          // O += P V: V^T fragments by transposing ldmatrix, two n-tiles per load
#pragma unroll
          for (int n2 = 0; n2 < NT; n2 += 2) {
            const int mi = lane >> 3, rr = lane & 7;
            const int key = (mi & 1) * 8 + rr;
            const int dunit = n2 + (mi >> 1);  // 16-byte unit along d
            const uint32_t addr =
                sV + (dunit >> 3) * (kDecTok * 128) + key * 128 + (((dunit & 7) ^ (key & 7)) << 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(addr, b0, b1, b2, b3);
            mma_16816(oc[n2], pa, b0, b1);
            mma_16816(oc[n2 + 1], pa, b2, b3);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&misc->empty[st]);
      }
      gp_base += npieces;
      if (!ok) break;

      // ---- this warp's partial for the item: O / l (rows < nrows) and log2-sum-exp
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
      const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
      const size_t pbase = (((size_t)it.s * a.max_chunks + it.c) * kDecWarps + warp) * a.Hq + hq0;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int col = n * 8 + 2 * t;
        if (g < nrows)
          *reinterpret_cast<float2*>(a.part_o + (pbase + g) * D + col) = make_float2(oc[n][0] * i0, oc[n][1] * i0);
        if (g + 8 < nrows)
          *reinterpret_cast<float2*>(a.part_o + (pbase + g + 8) * D + col) =
              make_float2(oc[n][2] * i1, oc[n][3] * i1);
      }
      if (t == 0) {
        if (g < nrows) a.part_lse[pbase + g] = (l0 > 0.f) ? m0 + log2f(l0) : -INFINITY;
        if (g + 8 < nrows) a.part_lse[pbase + g + 8] = (l1 > 0.f) ? m1 + log2f(l1) : -INFINITY;
      }
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ merge kernel

// One warp per (sequence, query head): combine the chunk partials by their log-sum-exp.
template <int D>
__global__ void __launch_bounds__(256) attn_decode_merge_kernel(const __grid_constant__ DecArgs a) {
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= a.S * a.Hq) return;
  const int s = wid / a.Hq;
  const int h = wid % a.Hq;
  const int nch = __ldg(&a.chunk_prefix[s + 1]) - __ldg(&a.chunk_prefix[s]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) acc[i] = 0.f;
  const int np = nch * kDecWarps;  // partials: one per (chunk, consumer warp)
  const size_t p0 = (size_t)s * a.max_chunks * kDecWarps;
  float M = -INFINITY;
  for (int c = 0; c < np; ++c) M = fmaxf(M, a.part_lse[(p0 + c) * a.Hq + h]);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int c = 0; c < np; ++c) {
      const size_t pi = (p0 + c) * a.Hq + h;
      const float lc = a.part_lse[pi];
      if (lc == -INFINITY) continue;
      const float w = ex2(lc - M);
      L += w;
      const float* po = a.part_o + pi * D + lane * PER;
#pragma unroll
      for (int i = 0; i < PER; i += 2) {
        const float2 v = *reinterpret_cast<const float2*>(po + i);
        acc[i] += w * v.x;
        acc[i + 1] += w * v.y;
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  __nv_bfloat16* dst = a.o + ((size_t)s * a.Hq + h) * D + lane * PER;
#pragma unroll
  for (int i = 0; i < PER; i += 2)
    *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(acc[i] * inv, acc[i + 1] * inv);
  if (lane == 0 && a.lse != nullptr)
    a.lse[(size_t)s * a.Hq + h] = (L > 0.f) ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace attn
