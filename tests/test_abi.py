"""The C ABI: the library builds for sm_100a, loads, exports every entry point the
header declares, and its host-side argument checks return the documented codes
before anything reaches the GPU (so these run without a device)."""

import ctypes
import os
import re
import subprocess

import pytest

from attn_fwd_05_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "attn_b200.h")

OK, INVALID, UNSUPPORTED, ALIGN, CUDA, TIMEOUT, BAD_PAGE, WORKSPACE = range(8)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[a-z_ *0-9]*?\b(attn_[a-z_]+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("attn_fwd", "attn_fwd_ex", "attn_decode_paged", "attn_decode_paged_workspace_size",
                     "attn_get_device_status", "attn_status_string"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert name in binding.SIGNATURES, name
        getattr(lib, name)


def test_library_builds_for_sm100a_only():
    # one -gencode, for the sm_100a architecture-specific target (tcgen05 and TMA need it)
    flags = build.NVCC_FLAGS
    gencodes = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]
    assert not any(f.startswith("-arch") for f in flags)


def test_status_strings(lib):
    assert lib.attn_status_string(OK) == b"ATTN_OK"
    assert lib.attn_status_string(BAD_PAGE) == b"ATTN_ERR_BAD_PAGE"
    assert lib.attn_status_string(99) == b"ATTN_STATUS_UNKNOWN"
    assert lib.attn_abi_version() == 1


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=4, Hkv=2, Nq=16, Nk=16, d=128, scale=0.1,
        causal=0, odt=0):
    return lib.attn_fwd_ex(q, k, v, o, odt, lse, B, Hq, Hkv, Nq, Nk, d, ctypes.c_float(scale), causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), INVALID), (dict(Nq=-3), INVALID), (dict(Nk=-1), INVALID),
    (dict(Hq=3, Hkv=2), INVALID), (dict(Hkv=0), INVALID),
    (dict(d=96), UNSUPPORTED), (dict(d=512), UNSUPPORTED),
    (dict(scale=0.0), INVALID), (dict(scale=-1.0), INVALID), (dict(scale=float("nan")), INVALID),
    (dict(scale=float("inf")), INVALID),
    (dict(causal=2), INVALID), (dict(odt=5), INVALID),
    (dict(q=None), INVALID), (dict(o=None), INVALID), (dict(k=None), INVALID),
    (dict(q=FAKE + 8), ALIGN), (dict(v=FAKE + 2), ALIGN), (dict(o=FAKE + 4), ALIGN), (dict(lse=FAKE + 2), ALIGN),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert fwd(lib, **kw) == code


def test_fwd_empty_work_is_a_noop(lib):
    # nothing to compute: returns before touching any pointer or the device
    assert fwd(lib, Nq=0, q=None, o=None) == OK
    assert fwd(lib, B=0, q=None, o=None) == OK


def fwd_masked(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, Hq=4, Hkv=2, Nq=16, Nk=16, d=128, scale=0.1,
               causal=1, window=0, block_mask=None, odt=0):
    return lib.attn_fwd_masked(q, k, v, o, odt, lse, B, Hq, Hkv, Nq, Nk, d, ctypes.c_float(scale), causal,
                               window, block_mask, None)


TOO_LARGE = 8


@pytest.mark.parametrize("kw,code", [
    (dict(window=-1), INVALID), (dict(window=8, causal=0), INVALID), (dict(causal=3), INVALID),
    (dict(block_mask=FAKE, Nk=2048 * 128 + 1), TOO_LARGE), (dict(block_mask=FAKE, d=256, Nk=1024 * 128 + 1), TOO_LARGE),
    (dict(d=80), UNSUPPORTED), (dict(q=None), INVALID), (dict(k=FAKE + 4), ALIGN),
])
def test_fwd_masked_rejects_bad_arguments(lib, kw, code):
    assert fwd_masked(lib, **kw) == code


def test_fwd_masked_empty_work_is_a_noop(lib):
    assert fwd_masked(lib, Nq=0, q=None, o=None, window=4) == OK


def dec(lib, q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, ps=16, o=FAKE, lse=None, S=4, Hq=8, Hkv=2, d=128,
        npages=10, maxp=8, scale=0.1, ws=FAKE, wsb=1 << 30):
    return lib.attn_decode_paged(q, kp, vp, bt, sl, ps, o, lse, S, Hq, Hkv, d, npages, maxp,
                                 ctypes.c_float(scale), ws, wsb, None)


@pytest.mark.parametrize("kw,code", [
    (dict(S=-1), INVALID), (dict(Hq=6, Hkv=4), INVALID), (dict(maxp=0), INVALID), (dict(npages=-1), INVALID),
    (dict(ps=8), UNSUPPORTED), (dict(ps=48), UNSUPPORTED), (dict(d=80), UNSUPPORTED),
    (dict(scale=0.0), INVALID), (dict(bt=None), INVALID), (dict(sl=None), INVALID), (dict(kp=None), INVALID),
    (dict(kp=FAKE + 8), ALIGN), (dict(bt=FAKE + 2), ALIGN), (dict(ws=FAKE + 16), ALIGN),
    (dict(ws=None), WORKSPACE), (dict(wsb=100), WORKSPACE),
])
def test_decode_rejects_bad_arguments(lib, kw, code):
    assert dec(lib, **kw) == code


def test_decode_empty_batch_is_a_noop(lib):
    assert dec(lib, S=0, q=None, o=None) == OK


def test_workspace_size(lib):
    f = lib.attn_decode_paged_workspace_size
    # 64 sequences, 64 query heads, d = 128, up to 2048 pages of 16 tokens: 16 chunks of 2048
    # tokens, one partial per (chunk, consumer warp) of each query head
    n = f(64, 64, 8, 128, 2048, 16)
    parts = 64 * 16 * 4 * 64
    item_map = 64 * 16 * 16  # one 16-byte record per chunk
    assert n >= parts * 128 * 4 + parts * 4 + 65 * 4 + item_map
    assert n < parts * 129 * 4 + item_map + 4096
    assert f(64, 64, 8, 96, 2048, 16) == 0    # unsupported head dimension
    assert f(64, 60, 8, 128, 2048, 16) == 0   # Hq not a multiple of Hkv
    assert f(64, 64, 8, 128, 2048, 24) == 0   # unsupported page size
    assert f(64, 64, 8, 128, 2048, 16) <= f(64, 64, 8, 128, 4096, 16)
