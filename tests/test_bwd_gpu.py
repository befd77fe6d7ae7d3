"""GPU parity of the backward kernels against the fp64 oracle (through the C ABI).

The GPU backward consumes the GPU forward's own O and LSE, as a training step
would; the oracle differentiates its own fp64 definition.  Bar: per tensor,
max|g - g_ref| / max|g_ref| <= 1e-2.
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


def run_case(B, Nq, Nk, Hq, Hkv, d, dtype, causal, window, seed, scale=None):
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
    return dq, dk, dv


MASKS = [(False, (-1, -1)), (True, (-1, -1)), (False, (37, 0)), (False, (-1, 5)),
         (False, (0, 0)), (True, (256, 256)), (True, (130, -1))]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "c%d_w%d_%d" % (m[0], *m[1]))
def test_masks_ragged(d, dtype, mask):
    causal, window = mask
    run_case(2, 300, 300, 4, 2, d, dtype, causal, window, seed=15)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 200), (77, 77), (200, 333), (333, 200),
                                   (129, 129), (256, 256), (511, 640)])
@pytest.mark.parametrize("causal", [False, True])
def test_lengths(Nq, Nk, causal):
    run_case(1, Nq, Nk, 2, 1, 64, torch.bfloat16, causal, (-1, -1), seed=16)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (8, 1), (6, 2)])
def test_gqa(Hq, Hkv):
    run_case(2, 260, 260, Hq, Hkv, 128, torch.bfloat16, True, (-1, -1), seed=17)


@pytest.mark.parametrize("scale", [0.0, -0.125, 0.5])
def test_scales(scale):
    run_case(1, 150, 150, 2, 2, 64, torch.float16, True, (-1, -1), seed=18, scale=scale)


def test_dk_dv_deterministic_and_gqa_sum():
    q, k, v, do = make_qkv(1, 384, 384, 8, 2, 128, torch.bfloat16, 19, with_dout=True)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    dq1, dk1, dv1 = fa.fa_bwd(dod, qd, kd, vd, o, lse, causal=True)
    dq2, dk2, dv2 = fa.fa_bwd(dod, qd, kd, vd, o, lse, causal=True)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)  # no atomics on dK / dV
    # the shared kv head's gradient equals the sum over its group (repeated heads)
    kr, vr = kd.repeat_interleave(4, dim=2), vd.repeat_interleave(4, dim=2)
    o_r, lse_r = fa.fa_fwd(qd, kr, vr, causal=True)
    _, dk_r, dv_r = fa.fa_bwd(dod, qd, kr, vr, o_r, lse_r, causal=True)
    dk_sum = dk_r.float().view(1, 384, 2, 4, 128).sum(3)
    dv_sum = dv_r.float().view(1, 384, 2, 4, 128).sum(3)
    assert (dk1.float() - dk_sum).abs().max() <= 1e-2 * dk_sum.abs().max()
    assert (dv1.float() - dv_sum).abs().max() <= 1e-2 * dv_sum.abs().max()


def test_strided_outputs():
    B, N, H, d = 1, 200, 2, 64
    q, k, v, do = make_qkv(B, N, N, H, H, d, torch.float16, 20, with_dout=True)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    pad = lambda: torch.zeros(B, N, H, d + 64, dtype=torch.float16, device=DEV)[..., :d]  # noqa
    dq, dk, dv = fa.fa_bwd(dod, qd, kd, vd, o, lse, causal=True, dq=pad(), dk=pad(), dv=pad())
    dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), d ** -0.5,
                                                  True)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


def test_workspace_too_small_rejected():
    q, k, v, do = (t.to(DEV) for t in make_qkv(1, 64, 64, 2, 2, 64, torch.float16, 21, True))
    o, lse = fa.fa_fwd(q, k, v)
    ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(do, q, k, v, o, lse, workspace=ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE


def test_full_size_long_context_one_head():
    """16384-token causal fwd+bwd at full size (the launch configuration the
    benchmark times); the oracle differentiates one query/kv head of it."""
    w = WORKLOADS["fwdbwd_1x16384_h16_d128_bf16_causal"]
    q, k, v, do = make_workload_inputs(w)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, softmax_scale=w.softmax_scale, causal=True)
    dq, dk, dv = fa.fa_bwd(dod, qd, kd, vd, o, lse, softmax_scale=w.softmax_scale, causal=True)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()
    h = 5
    sl = slice(h, h + 1)
    dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(to64(q[:, :, sl]), to64(k[:, :, sl]),
                                                  to64(v[:, :, sl]), to64(do[:, :, sl]),
                                                  w.softmax_scale, True)
    check_grad(dq[:, :, sl], dq_r, "dQ")
    check_grad(dk[:, :, sl], dk_r, "dK")
    check_grad(dv[:, :, sl], dv_r, "dV")
