// attn_api.cu — the C ABI declared in include/attn_b200.h.
//
// Host side only: argument checks, TMA tensor-map encoding, launch configuration.
// Every step of the computation runs in the kernels of prefill_sm100.cuh and
// decode_sm100.cuh.  The whole library is this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn_b200.h"
#include "backward_sm100.cuh"
#include "decode_sm100.cuh"
#include "prefill_d256_sm100.cuh"
#include "prefill_sm100.cuh"
#include "fwd_fp8_sm100.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;  // 1 s per pipeline wait
constexpr int kMaxDevices = 64;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 tensor map over [outer, rows, inner] with a {64, box_rows, 1} box, 128-byte
// swizzle and zero fill outside the tensor (rows past `rows` read as zero).
bool encode_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
               uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * 2, rows * inner * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 tensors [outer, rows, inner] with {32, 32, 1} boxes (128 bytes a row) and the
// 128-byte swizzle: the backward's gradient stores.
bool encode_3d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {inner, rows, outer};
  cuuint64_t strides[2] = {inner * 4, rows * inner * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// e4m3 tensors [outer, rows, 128 bytes]: one 128-byte swizzled row per token.
bool encode_3d_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t outer) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, rows, outer};
  cuuint64_t strides[2] = {128, rows * 128};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

// Raises the dynamic shared-memory limit of each kernel once per device.
template <typename K>
bool ensure_smem(K kernel, int bytes, int slot) {
  static std::mutex mu;
  static std::atomic<uint64_t> done[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return false;
  const uint64_t bit = 1ull << slot;
  if (done[dev].load(std::memory_order_acquire) & bit) return true;
  std::lock_guard<std::mutex> g(mu);
  if (done[dev].load() & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done[dev].fetch_or(bit, std::memory_order_release);
  return true;
}

int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load();
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev].store(v);
  }
  return v;
}

attn_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool MASKS>
attn_status launch_prefill(attn::FwdArgs& a, cudaStream_t st) {
  // shared-memory slots: 0-2 plain prefill, 3-5 decode, 6-8 masked prefill
  const int slot = (D == 64 ? 0 : (D == 128 ? 1 : 2)) + (MASKS ? 6 : 0);
  if constexpr (D <= 128) {
    using C = attn::PingPongCfg<D>;
    auto k = attn::attn_fwd_pingpong_kernel<D, MASKS>;
    if (!ensure_smem(k, C::SMEM, slot)) return ATTN_ERR_CUDA;
    const long long qp = (a.n_qtiles + 1) / 2;
    const long long units = a.pair_heads ? (long long)a.B * (a.Hq / 2) * a.n_qtiles : (long long)a.B * a.Hq * qp;
    if (units <= 0 || units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    a.n_units = (int)units;
    // persistent: one CTA per SM walks the units; with a block-sparse map, one unit per CTA
    const long long grid = a.block_mask != nullptr ? units : std::min<long long>(units, sm_count());
    k<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(a);
  } else {
    using C = attn::SingleCfg<D>;
    auto k = attn::attn_fwd_single_kernel<D, MASKS>;
    if (!ensure_smem(k, C::SMEM, slot)) return ATTN_ERR_CUDA;
    const long long units = (long long)a.B * a.Hq * a.n_qtiles;
    if (units <= 0 || units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    a.n_units = (int)units;
    k<<<(unsigned)units, C::THREADS, C::SMEM, st>>>(a);
  }
  return launch_status();
}

template <int D>
attn_status launch_bwd(attn::BwdArgs& a, const void* o, const void* dout, float* delta, cudaStream_t st) {
  using C = attn::BwdCfg<D>;
  const long long rows = (long long)a.B * a.Hq * a.Nq;
  const long long dblocks = std::min<long long>((rows + 7) / 8, (long long)sm_count() * 16);
  auto k = attn::attn_bwd_kernel<D>;
  const int slot = D == 64 ? 9 : 10;  // shared-memory slots 9-10: backward kernels
  if (!ensure_smem(k, C::SMEM, slot)) return ATTN_ERR_CUDA;
  const long long grid = (long long)a.B * a.Hkv * a.n_ktiles;
  if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  // Delta, and dQ cleared for the main kernel's reduce-adds
  attn::attn_bwd_delta_kernel<D><<<(unsigned)dblocks, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), delta, a.dq, rows);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  k<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(a);
  return launch_status();
}


template <int D>
attn_status launch_decode(attn::DecArgs& a, cudaStream_t st, long long max_items) {
  using C = attn::DecCfg<D>;
  auto ks = attn::attn_decode_split_kernel<D>;
  const int slot = D == 64 ? 3 : (D == 128 ? 4 : 5);
  if (!ensure_smem(ks, C::SMEM, slot)) return ATTN_ERR_CUDA;
  attn::attn_decode_plan_kernel<<<1, 1024, 0, st>>>(a.seq_lens, a.S, a.max_pages * a.page_size, a.chunk_prefix,
                                                    a.item_map);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  long long grid = (long long)sm_count() * C::CTAS_PER_SM;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  ks<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(a);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  const long long warps = (long long)a.S * a.Hq;
  const long long blocks = (warps * 32 + 255) / 256;
  attn::attn_decode_merge_kernel<D><<<(unsigned)blocks, 256, 0, st>>>(a);
  return launch_status();
}

struct DecodeLayout {
  size_t off_prefix, off_item_map, off_part_o, off_part_lse, total;
  int max_chunks;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool decode_layout(int S, int Hq, int d, int max_pages, int page_size, DecodeLayout* L) {
  if (S < 0 || Hq <= 0 || d <= 0 || max_pages <= 0 || page_size <= 0) return false;
  const long long max_tokens = (long long)max_pages * page_size;
  if (max_tokens > 0x7fffffffLL) return false;
  L->max_chunks = (int)((max_tokens + attn::kDecChunkTok - 1) / attn::kDecChunkTok);
  const size_t parts = (size_t)S * L->max_chunks * attn::kDecWarps * Hq;
  L->off_prefix = 0;
  L->off_item_map = align256((size_t)(S + 1) * 4);
  L->off_part_o = L->off_item_map + align256((size_t)S * L->max_chunks * 16);
  L->off_part_lse = L->off_part_o + align256(parts * d * 4);
  L->total = L->off_part_lse + align256(parts * 4);
  return true;
}

// ---------------------------------------------------------------- static decode scratch
//
// Scratch of attn_decode_paged_noalloc: a fixed array in the library's device image,
// so that the call needs no allocation.  Every device that loads the library holds it
// until the process exits.  In host code `g_decode_scratch` is only a host-side stand-in
// for the symbol; the device address comes from cudaGetSymbolAddress, once per device.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

// Device address of g_decode_scratch on the current device (looked up on the first
// call for that device), or nullptr if the lookup failed.  The address is valid for the
// primary context it was looked up in: a device reset invalidates it for the rest of the
// process.
void* static_scratch_address() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) {
      cudaGetLastError();  // reset the runtime error state so later calls are unaffected
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return 1; }

const char* attn_status_string(int s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_ALIGNMENT: return "ATTN_ERR_ALIGNMENT";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT";
    case ATTN_ERR_BAD_PAGE: return "ATTN_ERR_BAD_PAGE";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_TOO_LARGE: return "ATTN_ERR_TOO_LARGE";
    default: return "ATTN_STATUS_UNKNOWN";
  }
}

namespace {

// Failure-path testing: which ring fill of which CTA to leave out, and the wait limit.
struct DebugStall {
  int cta, fill;
  uint64_t timeout_ns;
};

attn_status fwd_common(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B, int Hq,
                       int Hkv, int Nq, int Nk, int d, float scale, int causal, int window, const uint8_t* block_mask,
                       void* stream, const DebugStall* dbg = nullptr) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_DTYPE_BF16 && o_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (q == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (Nk > 0 && (k == nullptr || v == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(o, 16) || (Nk > 0 && (!aligned(k, 16) || !aligned(v, 16))) ||
      (lse != nullptr && !aligned(lse, 4)))
    return ATTN_ERR_ALIGNMENT;
  if ((long long)B * Hq > 0x7fffffffLL || (long long)B * Hkv > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  // block-sparse map: one byte per 128 x 128 block; a CTA keeps its visited blocks in a
  // bounded shared-memory list (d <= 128) or bitmap (d = 256)
  const long long nkt = ((long long)Nk + attn::kMaskBlock - 1) / attn::kMaskBlock;
  if (block_mask != nullptr) {
    const long long max_nkt = d <= 128 ? (long long)attn::kMaxVisits : 1024;
    if (nkt > max_nkt) return ATTN_ERR_TOO_LARGE;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int o_f32 = o_dtype == ATTN_DTYPE_F32;

  if (Nk == 0) {  // no key is visible to any row
    const size_t rows = (size_t)B * Hq * Nq;
    attn::attn_fwd_empty_kernel<<<592, 256, 0, st>>>(o, lse, rows, d, o_f32);
    return launch_status();
  }

  attn::FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  const uint32_t bn = d <= 128 ? 128 : 64;
  if (!encode_3d(&a.tm_q, q, d, Nq, (uint64_t)B * Hq, 128) || !encode_3d(&a.tm_k, k, d, Nk, (uint64_t)B * Hkv, bn) ||
      !encode_3d(&a.tm_v, v, d, Nk, (uint64_t)B * Hkv, bn))
    return ATTN_ERR_CUDA;
  // bf16 O of the two-tile kernel leaves through TMA stores of 32-row boxes
  if (!o_f32 && d <= 128 && !encode_3d(&a.tm_o, o, d, Nq, (uint64_t)B * Hq, 32)) return ATTN_ERR_CUDA;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nk = Nk;
  a.group = Hq / Hkv;
  a.causal = causal;
  a.o_f32 = o_f32;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.pair_heads = (a.group % 2 == 0) ? 1 : 0;
  a.n_qtiles = (Nq + 127) / 128;
  a.timeout_ns = dbg != nullptr ? dbg->timeout_ns : kDefaultTimeoutNs;
  a.dbg_stall_cta = dbg != nullptr ? dbg->cta : -1;
  a.dbg_stall_fill = dbg != nullptr ? dbg->fill : -1;
  // a window wider than every row's visible prefix hides nothing
  a.window = ((long long)window >= (long long)Nk + 1 || window == 0) ? 0 : window;
  a.block_mask = block_mask;
  a.nkt = (int)nkt;
  const bool masks = a.window > 0 || a.block_mask != nullptr;
  switch (d) {
    case 64: return masks ? launch_prefill<64, true>(a, st) : launch_prefill<64, false>(a, st);
    case 128: return masks ? launch_prefill<128, true>(a, st) : launch_prefill<128, false>(a, st);
    default: return masks ? launch_prefill<256, true>(a, st) : launch_prefill<256, false>(a, st);
  }
}

}  // namespace

attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream) {
  return fwd_common(q, k, v, o, o_dtype, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, nullptr, stream);
}

attn_status attn_fwd_masked(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B,
                            int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int window,
                            const uint8_t* block_mask, void* stream) {
  return fwd_common(q, k, v, o, o_dtype, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window, block_mask, stream);
}

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                     int Nq, int Nk, int d, float scale, int causal, void* stream) {
  return attn_fwd_ex(q, k, v, o, ATTN_DTYPE_BF16, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

attn_status attn_quantize_fp8(const void* x, void* out, float* scales, int planes, int N, int d, int block_rows,
                              void* stream) {
  if (planes < 0 || N < 0 || d <= 0 || (d & 1) || block_rows <= 0) return ATTN_ERR_INVALID_ARG;
  if (planes == 0 || N == 0) return ATTN_OK;
  if (x == nullptr || out == nullptr || scales == nullptr) return ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(out, 2) || !aligned(scales, 4)) return ATTN_ERR_ALIGNMENT;
  const long long nblk = ((long long)N + block_rows - 1) / block_rows;
  const long long grid = (long long)planes * nblk;
  if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  attn::attn_quantize_e4m3_kernel<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(out), scales, N, d, block_rows, (int)nblk);
  return launch_status();
}

attn_status attn_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale, const void* v8,
                         const float* v_scale, void* o, int o_dtype, float* lse, int B, int Hq, int Hkv, int Nq, int Nk,
                         int d, float scale, int causal, void* stream) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (o_dtype != ATTN_DTYPE_BF16 && o_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0 || Nq == 0) return ATTN_OK;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (q8 == nullptr || q_scale == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  if (Nk > 0 && (k8 == nullptr || v8 == nullptr || k_scale == nullptr || v_scale == nullptr))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned(q8, 16) || !aligned(o, 16) || (Nk > 0 && (!aligned(k8, 16) || !aligned(v8, 16))) ||
      (lse != nullptr && !aligned(lse, 4)))
    return ATTN_ERR_ALIGNMENT;
  if ((long long)B * Hq > 0x7fffffffLL || (long long)B * Hkv > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int o_f32 = o_dtype == ATTN_DTYPE_F32;
  if (Nk == 0) {
    attn::attn_fwd_empty_kernel<<<592, 256, 0, st>>>(o, lse, (size_t)B * Hq * Nq, d, o_f32);
    return launch_status();
  }
  attn::Fp8Args a;
  std::memset(&a, 0, sizeof(a));
  if (!encode_3d_u8(&a.tm_q, q8, Nq, (uint64_t)B * Hq) || !encode_3d_u8(&a.tm_k, k8, Nk, (uint64_t)B * Hkv) ||
      !encode_3d_u8(&a.tm_v, v8, Nk, (uint64_t)B * Hkv))
    return ATTN_ERR_CUDA;
  if (!o_f32 && !encode_3d(&a.tm_o, o, 128, Nq, (uint64_t)B * Hq, 32)) return ATTN_ERR_CUDA;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nk = Nk;
  a.group = Hq / Hkv;
  a.causal = causal;
  a.o_f32 = o_f32;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.pair_heads = (a.group % 2 == 0) ? 1 : 0;
  a.n_qtiles = (Nq + 127) / 128;
  a.n_ktiles = (Nk + 127) / 128;
  a.timeout_ns = kDefaultTimeoutNs;
  const long long qp = (a.n_qtiles + 1) / 2;
  const long long units = a.pair_heads ? (long long)B * (Hq / 2) * a.n_qtiles : (long long)B * Hq * qp;
  if (units <= 0 || units > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  a.n_units = (int)units;
  using C = attn::Fp8Cfg;
  if (!ensure_smem(attn::attn_fwd_fp8_kernel, C::SMEM, 13)) return ATTN_ERR_CUDA;
  const long long grid = std::min<long long>(units, sm_count());
  attn::attn_fwd_fp8_kernel<<<(unsigned)grid, C::THREADS, C::SMEM, st>>>(a);
  return launch_status();
}

size_t attn_bwd_workspace_size(int B, int Hq, int Nq) {
  if (B < 0 || Hq < 0 || Nq < 0) return 0;
  return ((size_t)B * Hq * Nq * sizeof(float) + 255) & ~(size_t)255;
}

namespace {

attn_status bwd_common(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                       float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                       int causal, void* workspace, size_t workspace_bytes, void* stream, const DebugStall* dbg) {
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B == 0) return ATTN_OK;
  if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if ((long long)B * Hq > 0x7fffffffLL || (long long)B * Hkv > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Nq == 0 && Nk == 0) return ATTN_OK;
  if (Nq > 0 && (q == nullptr || o == nullptr || dout == nullptr || lse == nullptr || dq == nullptr))
    return ATTN_ERR_INVALID_ARG;
  if (Nk > 0 && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)) return ATTN_ERR_INVALID_ARG;
  if ((q && !aligned(q, 16)) || (k && !aligned(k, 16)) || (v && !aligned(v, 16)) || (o && !aligned(o, 16)) ||
      (dout && !aligned(dout, 16)) || (lse && !aligned(lse, 4)) || (dq && !aligned(dq, 16)) ||
      (dk && !aligned(dk, 16)) || (dv && !aligned(dv, 16)))
    return ATTN_ERR_ALIGNMENT;
  if (Nq == 0) {  // no query: no gradient reaches K or V
    const size_t bytes = (size_t)B * Hkv * Nk * d * sizeof(float);
    if (cudaMemsetAsync(dk, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, st) != cudaSuccess)
      return ATTN_ERR_CUDA;
    return ATTN_OK;
  }
  if (Nk == 0) {  // no key: every output row is zero, so is its gradient
    return cudaMemsetAsync(dq, 0, (size_t)B * Hq * Nq * d * sizeof(float), st) == cudaSuccess ? ATTN_OK
                                                                                               : ATTN_ERR_CUDA;
  }
  const size_t need = attn_bwd_workspace_size(B, Hq, Nq);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return ATTN_ERR_ALIGNMENT;

  attn::BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!encode_3d(&a.tm_q, q, d, Nq, (uint64_t)B * Hq, 128) || !encode_3d(&a.tm_do, dout, d, Nq, (uint64_t)B * Hq, 128) ||
      !encode_3d(&a.tm_k, k, d, Nk, (uint64_t)B * Hkv, 128) || !encode_3d(&a.tm_v, v, d, Nk, (uint64_t)B * Hkv, 128) ||
      !encode_3d_f32(&a.tm_dq, dq, d, Nq, (uint64_t)B * Hq) || !encode_3d_f32(&a.tm_dk, dk, d, Nk, (uint64_t)B * Hkv) ||
      !encode_3d_f32(&a.tm_dv, dv, d, Nk, (uint64_t)B * Hkv))
    return ATTN_ERR_CUDA;
  a.lse = lse;
  a.delta = static_cast<float*>(workspace);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nk = Nk;
  a.group = Hq / Hkv;
  a.causal = causal;
  a.n_qtiles = (Nq + 127) / 128;
  a.n_ktiles = (Nk + 127) / 128;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = dbg != nullptr ? dbg->timeout_ns : kDefaultTimeoutNs;
  a.dbg_stall_cta = dbg != nullptr ? dbg->cta : -1;
  a.dbg_stall_step = dbg != nullptr ? dbg->fill : -1;
  float* delta = static_cast<float*>(workspace);
  return d == 64 ? launch_bwd<64>(a, o, dout, delta, st) : launch_bwd<128>(a, o, dout, delta, st);
}

}  // namespace

attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                     float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                     int causal, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, workspace,
                    workspace_bytes, stream, nullptr);
}

size_t attn_decode_paged_workspace_size(int num_seqs, int Hq, int Hkv, int d, int max_pages_per_seq,
                                        int page_size) {
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0) return 0;
  if (d != 64 && d != 128 && d != 256) return 0;
  if (page_size != 16 && page_size != 32 && page_size != 64) return 0;
  DecodeLayout L;
  if (!decode_layout(num_seqs, Hq, d, max_pages_per_seq, page_size, &L)) return 0;
  return L.total;
}

}  // extern "C"

namespace {

// Checks of a decode call's arguments, made on the host before anything touches the
// device.  ATTN_OK with *empty set: no sequence, nothing to launch.  On ATTN_OK, *L is
// the workspace layout.
attn_status decode_check(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                         const int32_t* seq_lens, int page_size, const void* o, const float* lse, int num_seqs,
                         int Hq, int Hkv, int d, int num_pages, int max_pages_per_seq, float scale, bool* empty,
                         DecodeLayout* L) {
  *empty = false;
  if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || num_pages < 0 || max_pages_per_seq <= 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (page_size != 16 && page_size != 32 && page_size != 64) return ATTN_ERR_UNSUPPORTED;
  if (num_seqs == 0) {
    *empty = true;
    return ATTN_OK;
  }
  if (q == nullptr || o == nullptr || block_table == nullptr || seq_lens == nullptr) return ATTN_ERR_INVALID_ARG;
  if (num_pages > 0 && (k_pool == nullptr || v_pool == nullptr)) return ATTN_ERR_INVALID_ARG;
  if (!aligned(q, 4) || !aligned(o, 4) || !aligned(block_table, 4) || !aligned(seq_lens, 4) ||
      (lse != nullptr && !aligned(lse, 4)) || (num_pages > 0 && (!aligned(k_pool, 16) || !aligned(v_pool, 16))))
    return ATTN_ERR_ALIGNMENT;
  if ((long long)num_pages * Hkv > 0x7fffffffLL || (long long)num_seqs * Hq > 0x7fffffffLL)
    return ATTN_ERR_INVALID_ARG;
  if (!decode_layout(num_seqs, Hq, d, max_pages_per_seq, page_size, L)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

attn_status decode_common(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                          const int32_t* seq_lens, int page_size, void* o, float* lse, int num_seqs, int Hq, int Hkv,
                          int d, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                          size_t workspace_bytes, void* stream, const DebugStall* dbg) {
  DecodeLayout L;
  bool empty = false;
  const attn_status chk = decode_check(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv,
                                       d, num_pages, max_pages_per_seq, scale, &empty, &L);
  if (chk != ATTN_OK || empty) return chk;
  if (workspace == nullptr || workspace_bytes < L.total) return ATTN_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return ATTN_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  attn::DecArgs a;
  std::memset(&a, 0, sizeof(a));
  // an empty pool still needs a valid descriptor; no page id can then be in range
  const void* kp = num_pages > 0 ? k_pool : q;
  const void* vp = num_pages > 0 ? v_pool : q;
  const uint64_t outer = num_pages > 0 ? (uint64_t)num_pages * Hkv : 1;
  const uint64_t rows = num_pages > 0 ? (uint64_t)page_size : 1;
  if (num_pages > 0) {
    if (!encode_3d(&a.tm_k, kp, d, rows, outer, attn::kDecTok) || !encode_3d(&a.tm_v, vp, d, rows, outer, attn::kDecTok))
      return ATTN_ERR_CUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.chunk_prefix = reinterpret_cast<int*>(ws + L.off_prefix);
  a.item_map = reinterpret_cast<int4*>(ws + L.off_item_map);
  a.part_o = reinterpret_cast<float*>(ws + L.off_part_o);
  a.part_lse = reinterpret_cast<float*>(ws + L.off_part_lse);
  a.S = num_seqs;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.group = Hq / Hkv;
  a.n_hgroups = (a.group + 15) / 16;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.max_pages = max_pages_per_seq;
  a.max_chunks = L.max_chunks;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = dbg != nullptr ? dbg->timeout_ns : kDefaultTimeoutNs;
  a.dbg_stall_cta = dbg != nullptr ? dbg->cta : -1;
  a.dbg_stall_piece = dbg != nullptr ? dbg->fill : -1;
  const long long max_items = (long long)num_seqs * L.max_chunks * Hkv * a.n_hgroups;
  if (max_items > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  switch (d) {
    case 64: return launch_decode<64>(a, st, max_items);
    case 128: return launch_decode<128>(a, st, max_items);
    default: return launch_decode<256>(a, st, max_items);
  }
}

}  // namespace

extern "C" {

attn_status attn_decode_paged(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                              const int32_t* seq_lens, int page_size, void* o, float* lse, int num_seqs, int Hq,
                              int Hkv, int d, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return decode_common(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv, d, num_pages,
                       max_pages_per_seq, scale, workspace, workspace_bytes, stream, nullptr);
}

attn_status attn_decode_paged_noalloc(const void* q, const void* k_pool, const void* v_pool,
                                      const int32_t* block_table, const int32_t* seq_lens, int page_size, void* o,
                                      float* lse, int num_seqs, int Hq, int Hkv, int d, int num_pages,
                                      int max_pages_per_seq, float scale, void* stream) {
  // Every argument check of attn_decode_paged comes first, so that a rejected call never
  // touches the device (not even the symbol lookup of the first call).
  DecodeLayout L;
  bool empty = false;
  const attn_status chk = decode_check(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv,
                                       d, num_pages, max_pages_per_seq, scale, &empty, &L);
  if (chk != ATTN_OK || empty) return chk;
  if (L.total > kStaticScratchBytes) return ATTN_ERR_TOO_LARGE;
  void* scratch = static_scratch_address();
  if (scratch == nullptr) return ATTN_ERR_CUDA;
  return decode_common(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv, d, num_pages,
                       max_pages_per_seq, scale, scratch, kStaticScratchBytes, stream, nullptr);
}

size_t attn_decode_paged_noalloc_max_scratch(void) { return kStaticScratchBytes; }

attn_status attn_debug_watchdog(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  attn::attn_watchdog_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return launch_status();
}

attn_status attn_debug_fwd_stall(const void* q, const void* k, const void* v, void* o, int o_dtype, float* lse, int B,
                                 int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, int stall_cta,
                                 int stall_fill, uint64_t timeout_ns, void* stream) {
  if (d > 128) return ATTN_ERR_UNSUPPORTED;  // the two-tile kernel's producer carries the switch
  if (stall_cta < 0 || stall_fill < 0 || timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  const DebugStall dbg{stall_cta, stall_fill, timeout_ns};
  return fwd_common(q, k, v, o, o_dtype, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, nullptr, stream, &dbg);
}

attn_status attn_debug_bwd_stall(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                 const float* lse, float* dq, float* dk, float* dv, int B, int Hq, int Hkv, int Nq,
                                 int Nk, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                                 int stall_cta, int stall_step, uint64_t timeout_ns, void* stream) {
  if (stall_cta < 0 || stall_step < 0 || timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  const DebugStall dbg{stall_cta, stall_step, timeout_ns};
  return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, workspace,
                    workspace_bytes, stream, &dbg);
}

attn_status attn_debug_decode_stall(const void* q, const void* k_pool, const void* v_pool, const int32_t* block_table,
                                    const int32_t* seq_lens, int page_size, void* o, float* lse, int num_seqs, int Hq,
                                    int Hkv, int d, int num_pages, int max_pages_per_seq, float scale, void* workspace,
                                    size_t workspace_bytes, int stall_cta, int stall_piece, uint64_t timeout_ns,
                                    void* stream) {
  if (stall_cta < 0 || stall_piece < 0 || timeout_ns == 0 || timeout_ns > 10000000000ull) return ATTN_ERR_INVALID_ARG;
  const DebugStall dbg{stall_cta, stall_piece, timeout_ns};
  return decode_common(q, k_pool, v_pool, block_table, seq_lens, page_size, o, lse, num_seqs, Hq, Hkv, d, num_pages,
                       max_pages_per_seq, scale, workspace, workspace_bytes, stream, &dbg);
}

attn_status attn_debug_exp2(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const int threads = 256;
  const int blocks = (int)(((long long)n + 2 * threads - 1) / (2 * threads));
  attn::attn_exp2_poly_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

attn_status attn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(attn::g_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  return static_cast<attn_status>(v);
}

}  // extern "C"
