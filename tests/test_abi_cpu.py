"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fa143.h declares, and rejects bad arguments with the
documented status codes before any CUDA call (pointers here are never
dereferenced)."""
import ctypes
import os
import re

import pytest

import exact_attention_143_b200 as fa
from exact_attention_143_b200 import build as fa_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fa143.h")


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s*(fa_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def test_header_declarations_found():
    names = declared_functions()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string",
            "fa_get_device_error"} <= set(names)


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(fa.EXPORTED) == set(declared_functions())


def test_status_strings(lib):
    for code in range(7):
        assert lib.fa_status_string(code)
    assert lib.fa_status_string(99) == b"unknown status"


def _strides(*s):
    return (ctypes.c_int64 * 3)(*s)


def call_fwd(lib, q=0x10000, k=0x20000, v=0x30000, o=0x40000, lse=0x50000, B=1, Nq=128,
             Nk=128, Hq=2, Hkv=2, d=64, qs=None, ks=None, vs=None, os_=None, dtype=0, scale=0.125,
             causal=0, wl=-1, wr=-1):
    qs = qs or _strides(Nq * Hq * d, Hq * d, d)
    ks = ks or _strides(Nk * Hkv * d, Hkv * d, d)
    vs = vs or _strides(Nk * Hkv * d, Hkv * d, d)
    os_ = os_ or _strides(Nq * Hq * d, Hq * d, d)
    return lib.fa_fwd(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, qs, ks, vs, os_, dtype, scale,
                      causal, wl, wr, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(lse=0), fa.FA_ERR_INVALID_ARG),
    (dict(B=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=-3), fa.FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARG),
    (dict(wl=-2), fa.FA_ERR_INVALID_ARG),
    (dict(wr=-5), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(dtype=2), fa.FA_ERR_UNSUPPORTED),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=512), fa.FA_ERR_UNSUPPORTED),
    (dict(q=0x10008), fa.FA_ERR_ALIGNMENT),
    (dict(qs=_strides(128 * 2 * 64, 2 * 64 + 4, 64)), fa.FA_ERR_ALIGNMENT),
    (dict(o=0x10000), fa.FA_ERR_INVALID_ARG),      # output aliases q
    (dict(lse=0x30010), fa.FA_ERR_INVALID_ARG),    # lse inside v
])
def test_fwd_rejects(lib, kw, code):
    assert call_fwd(lib, **kw) == code


def test_bwd_workspace_size(lib):
    n = lib.fa_bwd_workspace_size(2, 100, 4, 64)
    assert n >= 2 * 100 * 4 * 64 * 4 + 2 * 2 * 4 * 100 * 4
    assert lib.fa_bwd_workspace_size(0, 100, 4, 64) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 8, 1, 64, dtype=torch.float16)
    with pytest.raises(RuntimeError):
        fa.fa_fwd(q, q, q)


def test_varlen_rejects_bad_offsets_arguments(lib):
    st = (ctypes.c_int64 * 2)(256, 64)
    args = lambda cu_q, cu_k, B, mq, mk, tq, tk: lib.fa_fwd_varlen(  # noqa: E731
        0x10000, 0x20000, 0x30000, 0x40000, 0x50000, cu_q, cu_k, B, mq, mk, tq, tk, 4, 4, 64,
        st, st, st, st, 0, 0.125, 1, -1, -1, None)
    assert args(0, 0x60000, 2, 10, 10, 20, 20) == fa.FA_ERR_INVALID_ARG      # no offsets
    assert args(0x60002, 0x60000, 2, 10, 10, 20, 20) == fa.FA_ERR_ALIGNMENT  # misaligned
    assert args(0x60000, 0x60000, 2, 30, 10, 20, 20) == fa.FA_ERR_INVALID_ARG  # max > total
    assert args(0x60000, 0x60000, 0, 10, 10, 20, 20) == fa.FA_ERR_INVALID_ARG  # no sequences


@pytest.mark.parametrize("p", [-0.1, 1.0, 1.5, 0.999, float("nan")])
def test_dropout_rejects_bad_probability(lib, p):
    # p outside [0, 1), or so close to 1 that round(256 (1 - p)) is 0: rejected
    # before any CUDA call, by the dense and the packed-batch entry points alike
    st3 = _strides(128 * 2 * 64, 2 * 64, 64)
    rc = lib.fa_fwd_dropout(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 1, 128, 128, 2, 2, 64,
                            st3, st3, st3, st3, 0, 0.125, 0, -1, -1, p, 7, 0, None)
    assert rc == fa.FA_ERR_INVALID_ARG
    st2 = (ctypes.c_int64 * 2)(256, 64)
    rc = lib.fa_fwd_varlen_dropout(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x60000,
                                   2, 10, 10, 20, 20, 4, 4, 64, st2, st2, st2, st2, 0, 0.125, 1,
                                   -1, -1, p, 7, 0, None)
    assert rc == fa.FA_ERR_INVALID_ARG
