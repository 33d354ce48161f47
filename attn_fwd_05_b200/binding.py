"""ctypes binding of libattn_b200.so: argument marshalling only.

Each function here has the name of a C entry point of include/attn_b200.h.  It checks
that torch tensors have the dtype, device and layout the C side expects, reads their
sizes and device addresses, and calls the C function on the given (default: current)
CUDA stream.  All computation happens in the library's kernels.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None
_LOCK = threading.Lock()

ATTN_OK = 0
STATUS_NAMES = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_ALIGNMENT",
                4: "ATTN_ERR_CUDA", 5: "ATTN_ERR_DEVICE_TIMEOUT", 6: "ATTN_ERR_BAD_PAGE",
                7: "ATTN_ERR_WORKSPACE", 8: "ATTN_ERR_TOO_LARGE"}
DTYPE_BF16, DTYPE_F32 = 0, 1

# exported symbol -> (restype, argtypes); mirrors include/attn_b200.h
_P = ctypes.c_void_p
_I = ctypes.c_int
SIGNATURES = {
    "attn_abi_version": (_I, []),
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "attn_fwd_ex": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "attn_fwd_masked": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _I, _P, _P]),
    "attn_quantize_fp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P]),
    "attn_bwd_workspace_size": (ctypes.c_size_t, [_I, _I, _I]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P,
                      ctypes.c_size_t, _P]),
    "attn_decode_paged_workspace_size": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "attn_decode_paged": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P,
                               ctypes.c_size_t, _P]),
    "attn_decode_paged_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                                       _P]),
    "attn_decode_paged_noalloc_max_scratch": (ctypes.c_size_t, []),
    "attn_debug_watchdog": (_I, [ctypes.c_uint64, _P]),
    "attn_debug_exp2": (_I, [_P, _P, _I, _P]),
    "attn_debug_fwd_stall": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, _I, _I,
                                  ctypes.c_uint64, _P]),
    "attn_debug_bwd_stall": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I,
                                  _P, ctypes.c_size_t, _I, _I, ctypes.c_uint64, _P]),
    "attn_debug_decode_stall": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P,
                                     ctypes.c_size_t, _I, _I, ctypes.c_uint64, _P]),
    "attn_get_device_status": (_I, [_P]),
    "attn_status_string": (ctypes.c_char_p, [_I]),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def library_path() -> str:
    return os.path.join(_HERE, "libattn_b200.so")


def load_library() -> ctypes.CDLL:
    """Loads the CUDA library; raises RuntimeError if it is missing or cannot be loaded."""
    global _LIB
    with _LOCK:
        if _LIB is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is not built: run `python -m attn_fwd_05_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _LIB = lib
    return _LIB


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, where)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int | None = None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")
    return t.data_ptr()


def _fwd_shapes(q, k, v, o, lse):
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, Hkv, Nk, d] with q's B and d")
    if tuple(o.shape) != (B, Hq, Nq, d):
        raise ValueError("o must be [B, Hq, Nq, d]")
    if lse is not None and tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be [B, Hq, Nq]")
    if o.dtype == torch.bfloat16:
        odt = DTYPE_BF16
    elif o.dtype == torch.float32:
        odt = DTYPE_F32
    else:
        raise TypeError("o must be bf16 or fp32")
    ptrs = (_dev(q, "q", torch.bfloat16, 4), _dev(k, "k", torch.bfloat16, 4), _dev(v, "v", torch.bfloat16, 4),
            _dev(o, "o", o.dtype, 4), odt, None if lse is None else _dev(lse, "lse", torch.float32, 3))
    return ptrs, (B, Hq, Hkv, Nq, Nk, d)


def attn_fwd_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor | None,
                causal: bool, scale: float, stream=None) -> None:
    """Prefill forward; o is bf16 or fp32 [B, Hq, Nq, d], lse fp32 [B, Hq, Nq] or None."""
    lib = load_library()
    ptrs, dims = _fwd_shapes(q, k, v, o, lse)
    st = lib.attn_fwd_ex(*ptrs, *dims, float(scale), int(bool(causal)), _stream(stream))
    _check(st, "attn_fwd_ex")


def attn_fwd_masked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor | None,
                    causal: bool, scale: float, window: int = 0, block_mask: torch.Tensor | None = None,
                    stream=None) -> None:
    """Prefill forward with a sliding window (window > 0, needs causal) and/or a
    block-sparse map: uint8 [ceil(Nq/128), ceil(Nk/128)] on the device, nonzero =
    the 128 x 128 block pair attends."""
    lib = load_library()
    ptrs, dims = _fwd_shapes(q, k, v, o, lse)
    bm = None
    if block_mask is not None:
        Nq, Nk = dims[3], dims[4]
        want = ((Nq + 127) // 128, (Nk + 127) // 128)
        if tuple(block_mask.shape) != want:
            raise ValueError(f"block_mask must be {want}")
        bm = _dev(block_mask, "block_mask", torch.uint8, 2)
    st = lib.attn_fwd_masked(*ptrs, *dims, float(scale), int(bool(causal)), int(window), bm, _stream(stream))
    _check(st, "attn_fwd_masked")


def attn_fwd(q, k, v, o, lse, causal: bool, scale: float, stream=None) -> None:
    """Prefill forward with bf16 output (see attn_fwd_ex)."""
    if o.dtype != torch.bfloat16:
        raise TypeError("attn_fwd writes bf16 o; use attn_fwd_ex for fp32")
    attn_fwd_ex(q, k, v, o, lse, causal, scale, stream)


def attn_quantize_fp8(x: torch.Tensor, block_rows: int, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Block e4m3 quantization of a bf16 [..., N, d] tensor: returns (codes uint8 [..., N, d],
    scales fp32 [..., ceil(N / block_rows)])."""
    lib = load_library()
    *lead, N, d = x.shape
    planes = 1
    for n in lead:
        planes *= n
    nblk = (N + block_rows - 1) // block_rows
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scales = torch.empty((*lead, nblk), dtype=torch.float32, device=x.device)
    st = lib.attn_quantize_fp8(_dev(x, "x", torch.bfloat16), out.data_ptr(), scales.data_ptr(), planes, N, d,
                               block_rows, _stream(stream))
    _check(st, "attn_quantize_fp8")
    return out, scales


def attn_fwd_fp8(q8, q_scale, k8, k_scale, v8, v_scale, o, lse, causal: bool, scale: float, stream=None) -> None:
    """FP8 forward: e4m3 q8 [B, Hq, Nq, 128], k8/v8 [B, Hkv, Nk, 128] (uint8 tensors) with fp32
    scales q_scale [B, Hq, ceil(Nq/128)], k_scale [B, Hkv, ceil(Nk/128)], v_scale [B, Hkv]."""
    lib = load_library()
    B, Hq, Nq, d = q8.shape
    Hkv, Nk = k8.shape[1], k8.shape[2]
    if tuple(k8.shape) != (B, Hkv, Nk, d) or tuple(v8.shape) != tuple(k8.shape):
        raise ValueError("k8 and v8 must be [B, Hkv, Nk, d]")
    if tuple(q_scale.shape) != (B, Hq, (Nq + 127) // 128) or tuple(k_scale.shape) != (B, Hkv, (Nk + 127) // 128) \
            or tuple(v_scale.shape) != (B, Hkv):
        raise ValueError("scale shapes must be [B, Hq, ceil(Nq/128)], [B, Hkv, ceil(Nk/128)], [B, Hkv]")
    if tuple(o.shape) != (B, Hq, Nq, d):
        raise ValueError("o must be [B, Hq, Nq, d]")
    odt = DTYPE_BF16 if o.dtype == torch.bfloat16 else DTYPE_F32 if o.dtype == torch.float32 else None
    if odt is None:
        raise TypeError("o must be bf16 or fp32")
    st = lib.attn_fwd_fp8(_dev(q8, "q8", torch.uint8, 4), _dev(q_scale, "q_scale", torch.float32, 3),
                          _dev(k8, "k8", torch.uint8, 4), _dev(k_scale, "k_scale", torch.float32, 3),
                          _dev(v8, "v8", torch.uint8, 4), _dev(v_scale, "v_scale", torch.float32, 2),
                          _dev(o, "o", o.dtype, 4), odt, None if lse is None else _dev(lse, "lse", torch.float32, 3),
                          B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)), _stream(stream))
    _check(st, "attn_fwd_fp8")


def attn_bwd_workspace_size(B: int, Hq: int, Nq: int) -> int:
    return int(load_library().attn_bwd_workspace_size(B, Hq, Nq))


def _bwd_args(q, k, v, o, do, lse, dq, dk, dv, causal, scale, workspace):
    lib = load_library()
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if tuple(k.shape) != (B, Hkv, Nk, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k and v must be [B, Hkv, Nk, d] with q's B and d")
    for name, t in (("o", o), ("do", do), ("dq", dq)):
        if tuple(t.shape) != (B, Hq, Nq, d):
            raise ValueError(f"{name} must be [B, Hq, Nq, d]")
    for name, t in (("dk", dk), ("dv", dv)):
        if tuple(t.shape) != (B, Hkv, Nk, d):
            raise ValueError(f"{name} must be [B, Hkv, Nk, d]")
    if tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be [B, Hq, Nq]")
    need = lib.attn_bwd_workspace_size(B, Hq, Nq)
    if workspace is None:
        workspace = torch.empty(max(int(need), 16), dtype=torch.uint8, device=q.device)
    return (_dev(q, "q", torch.bfloat16, 4), _dev(k, "k", torch.bfloat16, 4), _dev(v, "v", torch.bfloat16, 4),
            _dev(o, "o", torch.bfloat16, 4), _dev(do, "do", torch.bfloat16, 4),
            _dev(lse, "lse", torch.float32, 3), _dev(dq, "dq", torch.float32, 4),
            _dev(dk, "dk", torch.float32, 4), _dev(dv, "dv", torch.float32, 4),
            B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
            _dev(workspace, "workspace", torch.uint8, 1), workspace.numel())


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, do: torch.Tensor,
             lse: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor, causal: bool, scale: float,
             workspace: torch.Tensor | None = None, stream=None) -> None:
    """Backward pass: fp32 dq [B, Hq, Nq, d], dk and dv [B, Hkv, Nk, d] from the bf16 inputs, the
    forward's bf16 o and fp32 lse, and the bf16 upstream gradient do [B, Hq, Nq, d]."""
    args = _bwd_args(q, k, v, o, do, lse, dq, dk, dv, causal, scale, workspace)
    _check(load_library().attn_bwd(*args, _stream(stream)), "attn_bwd")


def attn_decode_paged_workspace_size(num_seqs: int, Hq: int, Hkv: int, d: int, max_pages_per_seq: int,
                                     page_size: int) -> int:
    return int(load_library().attn_decode_paged_workspace_size(num_seqs, Hq, Hkv, d, max_pages_per_seq,
                                                               page_size))


def attn_decode_paged(q, k_pool, v_pool, block_table, seq_lens, page_size: int, o, lse, scale: float,
                      workspace: torch.Tensor, stream=None) -> None:
    """One decode step over a paged KV cache (shapes as in include/attn_b200.h)."""
    lib = load_library()
    S, Hq, d = q.shape
    num_pages, Hkv, ps, d2 = k_pool.shape
    if ps != page_size or d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("pools must be [num_pages, Hkv, page_size, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S:
        raise ValueError("block_table must be [num_seqs, max_pages_per_seq]")
    max_pages = block_table.shape[1]
    st = lib.attn_decode_paged(
        _dev(q, "q", torch.bfloat16, 3), _dev(k_pool, "k_pool", torch.bfloat16, 4),
        _dev(v_pool, "v_pool", torch.bfloat16, 4), _dev(block_table, "block_table", torch.int32, 2),
        _dev(seq_lens, "seq_lens", torch.int32, 1), page_size, _dev(o, "o", torch.bfloat16, 3),
        None if lse is None else _dev(lse, "lse", torch.float32, 2), S, Hq, Hkv, d, num_pages, max_pages,
        float(scale), _dev(workspace, "workspace", workspace.dtype), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "attn_decode_paged")


def attn_decode_paged_noalloc(q, k_pool, v_pool, block_table, seq_lens, page_size: int, o, lse, scale: float,
                              stream=None) -> None:
    """attn_decode_paged without a workspace: the library's static scratch is used.

    For callers that must not allocate device memory; raises AttnError with
    ATTN_ERR_TOO_LARGE when the sizes need more scratch than the library holds.
    """
    lib = load_library()
    S, Hq, d = q.shape
    num_pages, Hkv, ps, d2 = k_pool.shape
    if ps != page_size or d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("pools must be [num_pages, Hkv, page_size, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S:
        raise ValueError("block_table must be [num_seqs, max_pages_per_seq]")
    st = lib.attn_decode_paged_noalloc(
        _dev(q, "q", torch.bfloat16, 3), _dev(k_pool, "k_pool", torch.bfloat16, 4),
        _dev(v_pool, "v_pool", torch.bfloat16, 4), _dev(block_table, "block_table", torch.int32, 2),
        _dev(seq_lens, "seq_lens", torch.int32, 1), page_size, _dev(o, "o", torch.bfloat16, 3),
        None if lse is None else _dev(lse, "lse", torch.float32, 2), S, Hq, Hkv, d, num_pages,
        block_table.shape[1], float(scale), _stream(stream))
    _check(st, "attn_decode_paged_noalloc")


def attn_get_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the first fault a kernel latched."""
    return int(load_library().attn_get_device_status(_stream(stream)))


def attn_debug_watchdog(timeout_ns: int, stream=None) -> None:
    _check(load_library().attn_debug_watchdog(int(timeout_ns), _stream(stream)), "attn_debug_watchdog")


def attn_debug_fwd_stall(q, k, v, o, lse, causal: bool, scale: float, stall_cta: int, stall_fill: int,
                         timeout_ns: int, stream=None) -> None:
    """attn_fwd_ex with one K/V ring fill left out in one CTA and pipeline waits limited to
    timeout_ns: exercises the kernel's timeout wind-down (testing only)."""
    lib = load_library()
    ptrs, dims = _fwd_shapes(q, k, v, o, lse)
    st = lib.attn_debug_fwd_stall(*ptrs, *dims, float(scale), int(bool(causal)), int(stall_cta), int(stall_fill),
                                  int(timeout_ns), _stream(stream))
    _check(st, "attn_debug_fwd_stall")


def attn_debug_bwd_stall(q, k, v, o, do, lse, dq, dk, dv, causal: bool, scale: float, stall_cta: int,
                         stall_step: int, timeout_ns: int, workspace: torch.Tensor | None = None, stream=None) -> None:
    """attn_bwd with the Q tile of one step left out in one CTA of the gradient kernel and
    pipeline waits limited to timeout_ns (testing only)."""
    args = _bwd_args(q, k, v, o, do, lse, dq, dk, dv, causal, scale, workspace)
    st = load_library().attn_debug_bwd_stall(*args, int(stall_cta), int(stall_step), int(timeout_ns), _stream(stream))
    _check(st, "attn_debug_bwd_stall")


def attn_debug_decode_stall(q, k_pool, v_pool, block_table, seq_lens, page_size: int, o, lse, scale: float,
                            workspace: torch.Tensor, stall_cta: int, stall_piece: int, timeout_ns: int,
                            stream=None) -> None:
    """attn_decode_paged with one K/V piece left out in one CTA of the split kernel and
    pipeline waits limited to timeout_ns (testing only)."""
    lib = load_library()
    S, Hq, d = q.shape
    num_pages, Hkv, ps, d2 = k_pool.shape
    if ps != page_size or d2 != d or tuple(v_pool.shape) != tuple(k_pool.shape):
        raise ValueError("pools must be [num_pages, Hkv, page_size, d]")
    if block_table.dim() != 2 or block_table.shape[0] != S:
        raise ValueError("block_table must be [num_seqs, max_pages_per_seq]")
    st = lib.attn_debug_decode_stall(
        _dev(q, "q", torch.bfloat16, 3), _dev(k_pool, "k_pool", torch.bfloat16, 4),
        _dev(v_pool, "v_pool", torch.bfloat16, 4), _dev(block_table, "block_table", torch.int32, 2),
        _dev(seq_lens, "seq_lens", torch.int32, 1), page_size, _dev(o, "o", torch.bfloat16, 3),
        None if lse is None else _dev(lse, "lse", torch.float32, 2), S, Hq, Hkv, d, num_pages,
        block_table.shape[1], float(scale), _dev(workspace, "workspace", workspace.dtype),
        workspace.numel() * workspace.element_size(), int(stall_cta), int(stall_piece), int(timeout_ns),
        _stream(stream))
    _check(st, "attn_debug_decode_stall")


def attn_debug_exp2(x: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """y = 2^x by the kernel's FMA-pipe polynomial (fp32 device tensors)."""
    n = x.numel()
    if y.numel() != n:
        raise ValueError("x and y must have the same size")
    _check(load_library().attn_debug_exp2(_dev(x, "x", torch.float32), _dev(y, "y", torch.float32), n,
                                          _stream(stream)), "attn_debug_exp2")


def attn_status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()
