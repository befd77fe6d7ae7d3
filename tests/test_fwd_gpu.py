"""GPU parity of the forward kernel against the fp64 oracle (through the C ABI).

Small cases compare every element; the full-size workloads compare sampled
rows the oracle computes one by one, in the launch configuration the
benchmark times.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
from tests.parity import check_lse, check_o, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_case(B, Nq, Nk, Hq, Hkv, d, dtype, causal, window, seed, scale=None):
    q, k, v = make_qkv(B, Nq, Nk, Hq, Hkv, d, dtype, seed)
    scale = d ** -0.5 if scale is None else scale
    o, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=scale, causal=causal,
                       window_size=window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_ref, lse_ref = oracle.attention_fwd(to64(q), to64(k), to64(v), scale, causal, window)
    check_o(o, o_ref, dtype)
    check_lse(lse, lse_ref)
    return o, lse


def test_tiny_workload():
    w = WORKLOADS["tiny_128_d64_fp16"]
    run_case(w.batch, w.seqlen_q, w.seqlen_k, w.q_heads, w.kv_heads, w.head_dim, w.dtype,
             w.causal, w.window, w.seed)


MASKS = [(False, (-1, -1)), (True, (-1, -1)), (False, (37, 0)), (False, (-1, 5)),
         (False, (0, 0)), (False, (100, 50)), (True, (256, 256)), (True, (130, -1))]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "c%d_w%d_%d" % (m[0], *m[1]))
def test_masks_ragged(d, dtype, mask):
    # 300 rows: two 256-row blocks, the second ragged; keys not a tile multiple
    causal, window = mask
    run_case(2, 300, 300, 4, 2, d, dtype, causal, window, seed=5)


@pytest.mark.parametrize("Nq,Nk", [(1, 1), (1, 200), (77, 77), (200, 333), (333, 200),
                                   (129, 129), (256, 256), (511, 640)])
@pytest.mark.parametrize("causal", [False, True])
def test_lengths(Nq, Nk, causal):
    # Nq > Nk with causal leaves the first Nq - Nk rows without keys: O = 0, LSE = -inf
    run_case(1, Nq, Nk, 2, 1, 64, torch.float16, causal, (-1, -1), seed=6)


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)], ids=["d64", "d128"])
@pytest.mark.parametrize("window", [(-1, -1), (130, -1)], ids=["causal", "causal_w130"])
def test_causal_full_grid_ragged(d, dtype, window):
    # 2 x 40 heads x two 256-row blocks = 160 CTAs, enough to fill the SMs, so
    # the kernel keeps two 128-row query tiles per CTA (smaller causal problems
    # take one); the second block is ragged (rows 256-299)
    run_case(2, 300, 300, 40, 8, d, dtype, True, window, seed=9)


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)], ids=["d64", "d128"])
@pytest.mark.parametrize("Hq,Hkv,causal,window", [
    (8, 2, True, (200, 0)),      # G = 4, sliding window: head-pair work tiles
    (8, 2, False, (150, 100)),   # G = 4, two-sided window
    (16, 4, True, (384, 0)),     # G = 4, the widest window that pairs heads
    (6, 2, True, (200, 0)),      # G = 3 (odd): one head per work tile
], ids=["g4_causal_w200", "g4_w150_100", "g4_causal_w384", "g3_causal_w200"])
def test_gqa_window(d, dtype, Hq, Hkv, causal, window):
    # 700 rows: five 128-row blocks plus a ragged one
    run_case(2, 700, 700, Hq, Hkv, d, dtype, causal, window, seed=12)


@pytest.mark.parametrize("d,dtype", [(64, torch.float16), (128, torch.bfloat16)], ids=["d64", "d128"])
@pytest.mark.parametrize("Nq,Nk", [(333, 200), (200, 333), (1, 129)])
def test_gqa_window_unequal_lengths(d, dtype, Nq, Nk):
    # head-pair work tiles where some query tiles see no key at all (Nq > Nk
    # with a causal window leaves the first Nq - Nk rows empty)
    run_case(1, Nq, Nk, 4, 2, d, dtype, True, (100, 0), seed=13)


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (8, 1), (6, 2)])
def test_gqa(Hq, Hkv):
    run_case(2, 260, 260, Hq, Hkv, 128, torch.bfloat16, True, (-1, -1), seed=7)


@pytest.mark.parametrize("scale", [0.0, -0.125, 0.5])
def test_scales(scale):
    run_case(1, 150, 150, 2, 2, 64, torch.float16, True, (-1, -1), seed=8, scale=scale)


def test_mqa_matches_repeated_heads():
    q, k, v = make_qkv(1, 300, 300, 8, 2, 64, torch.bfloat16, 9)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = fa.fa_fwd(q, k, v, causal=True)
    o2, l2 = fa.fa_fwd(q, k.repeat_interleave(4, dim=2), v.repeat_interleave(4, dim=2),
                       causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_strided_inputs_and_deterministic():
    # q, k, v as views into one packed [B, N, 3, H, d] buffer; O into a padded buffer
    B, N, H, d = 2, 200, 4, 64
    g = torch.Generator().manual_seed(10)
    qkv = torch.randn(B, N, 3, H, d, generator=g).to(torch.float16)
    qkv_d = qkv.to(DEV)
    q, k, v = qkv_d[:, :, 0], qkv_d[:, :, 1], qkv_d[:, :, 2]
    out = torch.zeros(B, N, H, d + 64, dtype=torch.float16, device=DEV)[..., :d]
    o, lse = fa.fa_fwd(q, k, v, causal=True, out=out)
    o2, lse2 = fa.fa_fwd(q.contiguous(), k.contiguous(), v.contiguous(), causal=True)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    o3, lse3 = fa.fa_fwd(q, k, v, causal=True)
    assert torch.equal(o2, o3) and torch.equal(lse2, lse3)
    o_ref, lse_ref = oracle.attention_fwd(to64(qkv[:, :, 0]), to64(qkv[:, :, 1]),
                                          to64(qkv[:, :, 2]), d ** -0.5, True)
    check_o(o, o_ref, torch.float16)
    check_lse(lse, lse_ref)


def test_misaligned_pointer_rejected():
    q = torch.zeros(1 * 64 * 2 * 64 + 1, dtype=torch.float16, device=DEV)[1:].view(1, 64, 2, 64)
    k = torch.zeros(1, 64, 2, 64, dtype=torch.float16, device=DEV)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, k, k)
    assert e.value.status == fa.FA_ERR_ALIGNMENT


FULL = ["fwd_2x2048_h8_d64_fp16", "fwd_2x2048_h8_d64_fp16_causal",
        "fwd_4x4096_h32_d64_fp16_causal", "fwd_2x4096_h32kv8_d128_bf16_causal_win256",
        "fwdbwd_1x16384_h16_d128_bf16_causal"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_workload_inputs(w, with_dout=False)
    o, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=w.softmax_scale,
                       causal=w.causal, window_size=w.window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    rows = sample_rows(w.batch, w.q_heads, w.seqlen_q, 192, w.seed)
    o_ref, lse_ref = oracle.attention_fwd_rows(to64(q), to64(k), to64(v), rows,
                                               w.softmax_scale, w.causal, w.window)
    o_cpu = o.cpu()
    lse_cpu = lse.cpu()
    o_rows = np.stack([to64(o_cpu[b, i, h]) for b, h, i in rows])
    lse_rows = np.array([float(lse_cpu[b, h, i]) for b, h, i in rows])
    check_o(o_rows, o_ref, w.dtype)
    check_lse(lse_rows, lse_ref)
    # property at full size: every row's output is a convex combination of V rows
    assert torch.isfinite(o).all()
    vmax = v.abs().amax().item()
    assert o.abs().amax().item() <= vmax * (1 + 1e-2)
