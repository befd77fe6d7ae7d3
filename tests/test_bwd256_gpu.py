"""GPU parity of the head_dim 256 backward against the fp64 oracle (C ABI).

The pages list head dimensions up to 256 ("Что такое FlashAttention…", section
"Версии, оборудование и первоисточники").  The d = 256 backward splits d into
two halves over the grid and steps through 32 queries at a time; these cases
cover ragged lengths, every mask shape, Nq != Nk, GQA, both dtypes, a packed
variable-length batch and one head of the full-size d = 256 workload.  Bar: per
tensor, max|g - g_ref| / max|g_ref| <= 1e-2.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import WORKLOADS, make_qkv, make_workload_inputs
from tests.parity import check_grad, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_case(B, Nq, Nk, Hq, Hkv, dtype, causal, window, seed, scale=None):
    d = 256
    q, k, v, do = make_qkv(B, Nq, Nk, Hq, Hkv, d, dtype, seed, with_dout=True)
    scale = d ** -0.5 if scale is None else scale
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, softmax_scale=scale, causal=causal, window_size=window)
    dq, dk, dv = fa.fa_bwd(dod, qd, kd, vd, o, lse, softmax_scale=scale, causal=causal,
                           window_size=window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), scale,
                                                  causal, window)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


MASKS = [(False, (-1, -1)), (True, (-1, -1)), (False, (37, 0)), (False, (-1, 5)),
         (False, (0, 0)), (True, (256, 256)), (True, (130, -1))]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "c%d_w%d_%d" % (m[0], *m[1]))
def test_d256_bwd_masks_ragged(dtype, mask):
    # 300 rows: two key tiles (the second ragged) and ten 32-query blocks
    causal, window = mask
    run_case(2, 300, 300, 4, 2, dtype, causal, window, seed=25)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 200), (77, 77), (200, 333), (333, 200),
                                   (129, 129), (256, 256)])
@pytest.mark.parametrize("causal", [False, True])
def test_d256_bwd_lengths(Nq, Nk, causal):
    run_case(1, Nq, Nk, 2, 1, torch.bfloat16, causal, (-1, -1), seed=26)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 1), (6, 2)])
def test_d256_bwd_gqa(Hq, Hkv):
    run_case(2, 160, 160, Hq, Hkv, torch.bfloat16, True, (-1, -1), seed=27, scale=0.07)


def test_d256_bwd_varlen():
    lens = [300, 1, 129, 64]
    g = torch.Generator().manual_seed(28)
    tot = sum(lens)
    q = torch.randn(tot, 4, 256, generator=g).to(torch.bfloat16)
    k = torch.randn(tot, 2, 256, generator=g).to(torch.bfloat16)
    v = torch.randn(tot, 2, 256, generator=g).to(torch.bfloat16)
    do = torch.randn(tot, 4, 256, generator=g).to(torch.bfloat16)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    qd, kd, vd, dod, cud = (t.to(DEV) for t in (q, k, v, do, cu))
    o, lse = fa.fa_fwd_varlen(qd, kd, vd, cud, cud, max(lens), max(lens), softmax_scale=0.0625,
                              causal=True)
    dq, dk, dv = fa.fa_bwd_varlen(dod, qd, kd, vd, o, lse, cud, cud, max(lens), max(lens),
                                  softmax_scale=0.0625, causal=True)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    for bi in range(len(lens)):
        a, e = int(cu[bi]), int(cu[bi + 1])
        gq, gk, gv, _, _ = oracle.attention_bwd(to64(q[a:e])[None], to64(k[a:e])[None],
                                                to64(v[a:e])[None], to64(do[a:e])[None], 0.0625,
                                                True)
        check_grad(dq[a:e][None], gq, "dQ[seq %d]" % bi)
        check_grad(dk[a:e][None], gk, "dK[seq %d]" % bi)
        check_grad(dv[a:e][None], gv, "dV[seq %d]" % bi)


def test_d256_bwd_full_size_one_head():
    """The d = 256 benchmark workload (2 x 4096, 16 heads, causal, bf16) at full
    size; the oracle differentiates one (batch, head) of it."""
    w = WORKLOADS["fwd_2x4096_h16_d256_bf16_causal"]
    q, k, v, do = make_workload_inputs(w, with_dout=True)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, softmax_scale=w.softmax_scale, causal=True)
    dq, dk, dv = fa.fa_bwd(dod, qd, kd, vd, o, lse, softmax_scale=w.softmax_scale, causal=True)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    b, h = 1, 11
    sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
    dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(to64(q[sl]), to64(k[sl]), to64(v[sl]),
                                                  to64(do[sl]), w.softmax_scale, True)
    check_grad(dq[sl], dq_r, "dQ")
    check_grad(dk[sl], dk_r, "dK")
    check_grad(dv[sl], dv_r, "dV")
