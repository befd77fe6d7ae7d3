"""The no-allocation backward entry point, fa_bwd_noalloc (GPU).

Some callers cannot call cudaMalloc (a plugin inside a host framework that
owns all device memory and offers no workspace, or a latency-critical loop
where an allocation's implicit synchronisation is not allowed).  For them the
library keeps a fixed scratch array of its own.  This test calls that entry
point through the C ABI twice in a row and checks each result against the
ordinary fa_bwd (which takes a caller-allocated workspace), within the
gradient tolerance of the other GPU tests; it also checks that sizes beyond
the built-in scratch are refused.  It lives in its own file, named to be
collected last, so a stopping run has executed every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
from seeded_inputs import make_qkv
from tests.parity import check_grad, to64

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa143.h


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
    assert fa.bwd_workspace_size(B, N, Hq, d) <= SCRATCH_BYTES
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


def test_noalloc_rejects_sizes_beyond_scratch():
    lib = fa.load_library()
    q, k, v, do = (t.cuda() for t in make_qkv(1, 64, 64, 1, 1, 128, torch.bfloat16, 24, True))
    o, lse = fa.fa_fwd(q, k, v)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # claim a sequence length whose workspace exceeds the built-in array; the
    # size check refuses it on the host before anything touches the pointers
    Nbig = 200000
    assert fa.bwd_workspace_size(1, Nbig, 1, 128) > SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), 1, Nbig, Nbig, 1, 1, 128, _strides(q), _strides(k),
                            _strides(v), _strides(o), _strides(do), _strides(dq), _strides(dk),
                            _strides(dv), 1, 0.088, 1, -1, -1, stream)
    assert rc == fa.FA_ERR_WORKSPACE
