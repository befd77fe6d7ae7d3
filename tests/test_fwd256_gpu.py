"""GPU parity of the head_dim 256 forward against the fp64 oracle.

d = 256 runs its own kernel (one 128-row query tile per CTA, 64-key K/V
tiles); the cases mirror the d = 64 / 128 forward tests: every mask on ragged
lengths, key counts around the 64-key tile, GQA, Nq != Nk, a packed
variable-length batch, and the full-size workload on sampled rows.  The
backward does not take d = 256 and must say so.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
from tests.parity import check_lse, check_o, to64
from tests.test_fwd_gpu import MASKS

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_case(B, Nq, Nk, Hq, Hkv, dtype, causal, window, seed, scale=None):
    q, k, v = make_qkv(B, Nq, Nk, Hq, Hkv, 256, dtype, seed)
    scale = 256 ** -0.5 if scale is None else scale
    o, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=scale, causal=causal,
                       window_size=window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_ref, lse_ref = oracle.attention_fwd(to64(q), to64(k), to64(v), scale, causal, window)
    check_o(o, o_ref, dtype)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "c%d_w%d_%d" % (m[0], *m[1]))
def test_d256_masks_ragged(dtype, mask):
    causal, window = mask
    run_case(2, 300, 300, 2, 1, dtype, causal, window, seed=70)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 65), (63, 63), (64, 64), (65, 65), (129, 300),
                                   (300, 129), (511, 700)])
@pytest.mark.parametrize("causal", [False, True])
def test_d256_lengths(Nq, Nk, causal):
    run_case(1, Nq, Nk, 2, 2, torch.bfloat16, causal, (-1, -1), seed=71)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 1), (6, 2)])
def test_d256_gqa_and_scale(Hq, Hkv):
    run_case(1, 200, 200, Hq, Hkv, torch.float16, True, (-1, -1), seed=72, scale=-0.04)


def test_d256_varlen():
    lens = [300, 1, 129, 64]
    g = torch.Generator().manual_seed(73)
    tot = sum(lens)
    q = torch.randn(tot, 4, 256, generator=g).to(torch.bfloat16)
    k = torch.randn(tot, 2, 256, generator=g).to(torch.bfloat16)
    v = torch.randn(tot, 2, 256, generator=g).to(torch.bfloat16)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    o, lse = fa.fa_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV), cu.to(DEV), max(lens),
                              max(lens), softmax_scale=0.0625, causal=True)
    torch.cuda.synchronize()
    for bi in range(len(lens)):
        a, e = int(cu[bi]), int(cu[bi + 1])
        o_ref, lse_ref = oracle.attention_fwd(to64(q[a:e])[None], to64(k[a:e])[None],
                                              to64(v[a:e])[None], 0.0625, True)
        check_o(o[a:e][None], o_ref, torch.bfloat16, "O[seq %d]" % bi)
        check_lse(lse[:, a:e][None], lse_ref, "LSE[seq %d]" % bi)


def test_d256_dropout_backward_unsupported():
    # the head_dim 256 backward has no dropout variant
    q, k, v = (t.to(DEV) for t in make_qkv(1, 64, 64, 2, 2, 256, torch.bfloat16, 74))
    o, lse = fa.fa_fwd(q, k, v)
    with pytest.raises(fa.FAError) as e:
        fa.fa_bwd(torch.ones_like(o), q, k, v, o, lse, dropout_p=0.1, seed=1)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED


def test_d256_full_size_sampled_rows():
    w = WORKLOADS["fwd_2x4096_h16_d256_bf16_causal"]
    q, k, v = make_workload_inputs(w, with_dout=False)
    o, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=w.softmax_scale,
                       causal=w.causal, window_size=w.window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    rows = sample_rows(w.batch, w.q_heads, w.seqlen_q, 48, w.seed)
    o_ref, lse_ref = oracle.attention_fwd_rows(to64(q), to64(k), to64(v), rows, w.softmax_scale,
                                               w.causal, w.window)
    og = torch.stack([o[b, i, h] for b, h, i in rows])
    lg = torch.stack([lse[b, h, i] for b, h, i in rows])
    check_o(og, o_ref, w.dtype)
    check_lse(lg, lse_ref)
