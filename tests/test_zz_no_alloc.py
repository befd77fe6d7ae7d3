"""The no-allocation backward entry point, fa_bwd_noalloc (GPU).

Some callers cannot call cudaMalloc (a plugin inside a host framework that
owns all device memory and offers no workspace, or a latency-critical loop
where an allocation's implicit synchronisation is not allowed).  For them the
library keeps a fixed scratch array of its own.  This test calls that entry
point through the C ABI twice in a row and checks each result against the
ordinary fa_bwd (which takes a caller-allocated workspace), within the
gradient tolerance of the other GPU tests.  At the edge of the built-in
scratch, a problem whose workspace is exactly the scratch size runs and
matches fa_bwd, and one a single token longer is refused on the host.  It
lives in its own file, named to be collected last, so a stopping run has
executed every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
from seeded_inputs import make_qkv
from tests.parity import check_grad, to64

pytestmark = pytest.mark.gpu



def scratch_bytes():
    """The built-in scratch size of the loaded library (FA_BWD_NOALLOC_SCRATCH_BYTES)."""
    return int(fa.load_library().fa_bwd_noalloc_scratch_bytes())


def _strides(t):
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def call_noalloc(lib, do, q, k, v, o, lse, dq, dk, dv, scale, causal):
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    code = 1 if q.dtype == torch.bfloat16 else 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, Nq, Nk, Hq, Hkv, d, _strides(q), _strides(k),
                              _strides(v), _strides(o), _strides(do), _strides(dq),
                              _strides(dk), _strides(dv), code, scale, int(causal), -1, -1,
                              stream)


def test_noalloc_matches_fa_bwd_on_two_calls():
    lib = fa.load_library()
    B, N, Hq, Hkv, d = 2, 777, 8, 2, 128
    assert fa.bwd_workspace_size(B, N, Hq, d) <= scratch_bytes()
    q, k, v, do = (t.cuda() for t in make_qkv(B, N, N, Hq, Hkv, d, torch.bfloat16, 23, True))
    scale = d ** -0.5
    o, lse = fa.fa_fwd(q, k, v, softmax_scale=scale, causal=True)
    dq_ref, dk_ref, dv_ref = fa.fa_bwd(do, q, k, v, o, lse, softmax_scale=scale, causal=True)
    torch.cuda.synchronize()
    refs = [to64(t) for t in (dq_ref, dk_ref, dv_ref)]
    for _ in range(2):
        dq, dk, dv = torch.full_like(q, 7.0), torch.full_like(k, 7.0), torch.full_like(v, 7.0)
        rc = call_noalloc(lib, do, q, k, v, o, lse, dq, dk, dv, scale, True)
        assert rc == fa.FA_OK, fa.status_string(rc)
        torch.cuda.synchronize()
        assert fa.get_device_error() == fa.FA_OK
        for got, ref, name in zip((dq, dk, dv), refs, ("dQ", "dK", "dV")):
            check_grad(got, ref, name)
        # dK and dV are summed without atomics: identical to the workspace path
        assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)


def largest_fitting_length(limit, d):
    """The longest single-head sequence whose backward workspace fits `limit`."""
    lo, hi = 1, 1 << 24
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if fa.bwd_workspace_size(1, mid, 1, d) <= limit:
            lo = mid
        else:
            hi = mid - 1
    return lo


def test_noalloc_at_the_scratch_limit():
    # one head, d = 64: the longest sequence whose workspace fits the scratch
    # array runs and matches fa_bwd (for the 64 MiB array the workspace is
    # exactly the array's size); one more token is refused on the host
    # before anything touches the pointers
    lib = fa.load_library()
    limit, d = scratch_bytes(), 64
    N = largest_fitting_length(limit, d)
    assert fa.bwd_workspace_size(1, N, 1, d) <= limit < fa.bwd_workspace_size(1, N + 1, 1, d)
    q, k, v, do = (t.cuda() for t in make_qkv(1, N, N, 1, 1, d, torch.float16, 24, True))
    scale = d ** -0.5
    o, lse = fa.fa_fwd(q, k, v, softmax_scale=scale, causal=True)
    dq_ref, dk_ref, dv_ref = fa.fa_bwd(do, q, k, v, o, lse, softmax_scale=scale, causal=True)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = call_noalloc(lib, do, q, k, v, o, lse, dq, dk, dv, scale, True)
    assert rc == fa.FA_OK, fa.status_string(rc)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    check_grad(dq, to64(dq_ref), "dQ")
    assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), 1, N + 1, N + 1, 1, 1, d, _strides(q), _strides(k),
                            _strides(v), _strides(o), _strides(do), _strides(dq), _strides(dk),
                            _strides(dv), 0, scale, 1, -1, -1, stream)
    assert rc == fa.FA_ERR_WORKSPACE


def test_noalloc_rejects_sizes_far_beyond_scratch():
    lib = fa.load_library()
    q, k, v, do = (t.cuda() for t in make_qkv(1, 64, 64, 1, 1, 128, torch.bfloat16, 24, True))
    o, lse = fa.fa_fwd(q, k, v)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # claim a sequence length whose workspace exceeds the built-in array; the
    # size check refuses it on the host before anything touches the pointers
    Nbig = 600000
    assert fa.bwd_workspace_size(1, Nbig, 1, 128) > scratch_bytes()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), 1, Nbig, Nbig, 1, 1, 128, _strides(q), _strides(k),
                            _strides(v), _strides(o), _strides(do), _strides(dq), _strides(dk),
                            _strides(dv), 1, 0.088, 1, -1, -1, stream)
    assert rc == fa.FA_ERR_WORKSPACE
