"""GPU parity of the FP8 (e4m3) forward against the fp64 oracle.

The oracle computes exact attention of the dequantised inputs
(descale * e4m3 value, widened exactly to fp64).  The kernel's scores are exact
in fp32, but P is rounded to e4m3 before P V; the tolerance is derived from
that rounding (see fp8_error_model) and checked three ways:
  * every element lies within the worst-case bound of the rounding;
  * the RMS error does not exceed the rounding model's RMS prediction;
  * the error has no component along O itself (a scale or normalisation
    mistake would show up there long before it broke the worst-case bound).
The LSE is computed from unrounded probabilities and keeps the 16-bit bar.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import FP8_WORKLOADS, make_fp8_inputs
from tests.parity import check_lse, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
REL = 2.0 ** -4      # largest relative rounding error of a normal e4m3 value
SMALL_P = 2.0 ** -12  # below this P may land among e4m3's subnormals (P' < 2^-6)
SUB_ABS = 2.0 ** -16  # their absolute error, in units of the normalised P


def fp8_inputs(B, Nq, Nk, Hq, Hkv, d, descales, seed):
    """The e4m3 tensors and the exact fp64 values they stand for (descale x e4m3)."""
    q8, k8, v8 = make_fp8_inputs(B, Nq, Nk, Hq, Hkv, d, descales, seed)
    deq = [t.to(torch.float64).numpy() * float(s) for t, s in zip((q8, k8, v8), descales)]
    return (q8, k8, v8, *deq)


def fp8_error_model(q, k, v, scale, causal, window, b, h):
    """Worst-case bound and model RMS of the error of O[b, :, h, :].

    A P' >= 2^-6 (normal) carries a relative rounding error of at most 2^-4,
    modelled as uniform; a smaller one an absolute error of at most 2^-10 in
    P' units, i.e. 2^-16 of the normalised P since P' >= 2^6 P."""
    G = q.shape[2] // k.shape[2]
    P = oracle.attention_probs(q, k, b, h, scale, causal, window)  # [Nq, Nk]
    V = v[b, :, h // G, :]
    big = P >= SMALL_P
    small = (P > 0) & ~big
    absV = np.abs(V)
    bound = (REL + 1e-4) * (P @ absV) + SUB_ABS * (small.astype(np.float64) @ absV)
    var = ((np.where(big, P, 0.0) ** 2) * REL ** 2 / 3.0) @ (V ** 2) + \
        (small.astype(np.float64) * SUB_ABS ** 2 / 3.0) @ (V ** 2)
    return bound, var


def check_fp8(o_gpu, o_ref, parts):
    """parts: list of (index tuple into O [B,Nq,Hq,d], bound, var) covering the
    checked elements."""
    o = to64(o_gpu)
    errs, refs, preds = [], [], []
    for idx, bound, var in parts:
        e = o[idx] - o_ref[idx]
        r = o_ref[idx]
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -30))) - 8)
        lim = bound + half_ulp + 1e-4 * np.abs(r) + 1e-6
        assert np.isfinite(o[idx]).all(), "O has non-finite values"
        bad = np.abs(e) > lim
        assert not bad.any(), "%d elements beyond the e4m3 rounding bound (max excess %g)" % (
            int(bad.sum()), float((np.abs(e) - lim).max()))
        errs.append(e.ravel())
        refs.append(r.ravel())
        preds.append((var + (2 * half_ulp) ** 2 / 12.0).ravel())
    e, r, pv = np.concatenate(errs), np.concatenate(refs), np.concatenate(preds)
    rms, rms_model = np.sqrt(np.mean(e ** 2)), np.sqrt(np.mean(pv))
    assert rms <= 1.25 * rms_model, "RMS error %g above the rounding model's %g" % (rms, rms_model)
    eps = float(np.dot(e, r) / max(np.dot(r, r), 1e-30))
    assert abs(eps) <= 2e-3, "error correlates with O (scale %g)" % eps
    return {"rms": float(rms), "rms_model": float(rms_model), "scale_err": eps}


CASES = [
    # B, Nq, Nk, Hq, Hkv, d, causal, window, (descale_q, descale_k, descale_v)
    (2, 512, 512, 4, 4, 64, False, (-1, -1), (1.0, 1.0, 1.0)),
    (1, 700, 700, 4, 2, 128, True, (-1, -1), (1.0, 1.0, 1.0)),
    (1, 640, 640, 2, 2, 64, True, (64, 0), (0.5, 2.0, 1.5)),
    (1, 300, 900, 2, 1, 128, False, (-1, -1), (1.25, 0.75, 0.5)),
    (1, 129, 129, 2, 2, 128, False, (5, 5), (1.0, 1.0, 1.0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%d_q%d_k%d_d%d_c%d" % (c[0], c[1], c[2],
                                                                               c[5], c[6]))
def test_fp8_matches_oracle(case):
    B, Nq, Nk, Hq, Hkv, d, causal, window, ds = case
    q8, k8, v8, q64, k64, v64 = fp8_inputs(B, Nq, Nk, Hq, Hkv, d, ds, seed=60)
    scale = d ** -0.5
    o, lse = fa.fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), softmax_scale=scale,
                           causal=causal, window_size=window, descale_q=ds[0], descale_k=ds[1],
                           descale_v=ds[2])
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_ref, lse_ref = oracle.attention_fwd(q64, k64, v64, scale, causal, window)
    parts = []
    for b in range(B):
        for h in range(Hq):
            bound, var = fp8_error_model(q64, k64, v64, scale, causal, window, b, h)
            parts.append(((b, slice(None), h, slice(None)), bound, var))
    check_fp8(o, o_ref, parts)
    check_lse(lse, lse_ref)


def test_fp8_rejects_bad_inputs():
    q8, k8, v8 = make_fp8_inputs(1, 128, 128, 2, 2, 64, (1.0, 1.0, 1.0), seed=61)
    with pytest.raises(TypeError):  # 16-bit inputs go to fa_fwd
        fa.fa_fwd_fp8(q8.to(DEV).to(torch.bfloat16), k8.to(DEV), v8.to(DEV))
    qs = torch.zeros((1, 128, 2, 72), dtype=torch.float8_e4m3fn, device=DEV)[..., :64]
    with pytest.raises(fa.FAError) as e:  # row stride 72 bytes: not a multiple of 16
        fa.fa_fwd_fp8(qs, k8.to(DEV), v8.to(DEV))
    assert e.value.status == fa.FA_ERR_ALIGNMENT


def test_fp8_workload_full_size_sampled():
    # the pages' FP8 example shape at full size, in the launch configuration the
    # bench times; three (batch, head) slices are checked against the oracle
    w = FP8_WORKLOADS["fwd_fp8_2x4096_h32_d64_e4m3"]
    q8, k8, v8, q64, k64, v64 = fp8_inputs(w.batch, w.seqlen, w.seqlen, w.q_heads, w.kv_heads,
                                           w.head_dim, w.descales, w.seed)
    o, lse = fa.fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), softmax_scale=w.softmax_scale,
                           causal=w.causal, descale_q=w.descales[0], descale_k=w.descales[1],
                           descale_v=w.descales[2])
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    parts = []
    o_ref = np.zeros(o.shape, np.float64)
    for b, h in [(0, 0), (1, 17), (1, 31)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ob, lb = oracle.attention_fwd(q64[sl], k64[b:b + 1, :, h:h + 1], v64[b:b + 1, :, h:h + 1],
                                      w.softmax_scale, w.causal)
        o_ref[b, :, h, :] = ob[0, :, 0, :]
        check_lse(lse[b:b + 1, h:h + 1], lb, "LSE[%d,%d]" % (b, h))
        bound, var = fp8_error_model(q64, k64, v64, w.softmax_scale, w.causal, (-1, -1), b, h)
        parts.append(((b, slice(None), h, slice(None)), bound, var))
    check_fp8(o, o_ref, parts)


def test_fp8_long_causal_full_size_sampled_blocks():
    # the 16384-token causal d = 128 shape the bench times (where 2 of every 8
    # exponential pairs take the FMA-pipe exp2); two 128-row query blocks of two
    # heads are checked: a block's rows see keys [0, last row], so the oracle and
    # the error model run on that block against its key prefix (bottom-right
    # causal alignment keeps the same visibility)
    w = FP8_WORKLOADS["fwd_fp8_1x16384_h16_d128_e4m3_causal"]
    q8, k8, v8, q64, k64, v64 = fp8_inputs(w.batch, w.seqlen, w.seqlen, w.q_heads, w.kv_heads,
                                           w.head_dim, w.descales, w.seed)
    o, lse = fa.fa_fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), softmax_scale=w.softmax_scale,
                           causal=w.causal, descale_q=w.descales[0], descale_k=w.descales[1],
                           descale_v=w.descales[2])
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    for h in (3, 14):
        for r0 in (8064, 16256):
            r1 = r0 + 128
            qs = q64[:, r0:r1, h:h + 1]
            ks, vs = k64[:, :r1, h:h + 1], v64[:, :r1, h:h + 1]
            ob, lb = oracle.attention_fwd(qs, ks, vs, w.softmax_scale, True)
            check_lse(lse_cpu[:, h:h + 1, r0:r1], lb, "LSE[h %d, rows %d:%d]" % (h, r0, r1))
            bound, var = fp8_error_model(qs, ks, vs, w.softmax_scale, True, (-1, -1), 0, 0)
            check_fp8(o_cpu[:, r0:r1, h:h + 1], ob, [((0, slice(None), 0, slice(None)), bound, var)])
