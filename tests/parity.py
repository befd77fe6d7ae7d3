"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (max-abs on O: 2e-3 for fp16, 1e-2 for bf16; max-relative 1e-2 on
dQ/dK/dV measured as max|g - g_ref| / max(max|g_ref|, 1e-2) per tensor) are the
workload's stated bars.  An O element also passes when it lies within one
unit in the last place of the output dtype at the oracle value: a correctly
rounded bf16 result of magnitude >= 4 can be 1.6e-2 away from the unrounded
fp64 value, so the bar alone would reject perfect rounding.  Such elements
are counted and reported, never silently absorbed.
"""
import numpy as np
import torch

O_ATOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}
LSE_ATOL = 5e-4
GRAD_RTOL = 1e-2
GRAD_DENOM_FLOOR = 1e-2
MANTISSA_BITS = {torch.float16: 10, torch.bfloat16: 7}


def to64(t):
    return t.detach().float().cpu().double().numpy()


def ulp(ref, dtype):
    """Spacing of `dtype` numbers at |ref| (normal range)."""
    mag = np.maximum(np.abs(ref), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(mag)) - MANTISSA_BITS[dtype])


def check_o(o_gpu, o_ref, dtype, what="O"):
    o = to64(o_gpu) if isinstance(o_gpu, torch.Tensor) else o_gpu
    err = np.abs(o - o_ref)
    tol = O_ATOL[dtype]
    bad_bar = err > tol
    within_ulp = err <= ulp(o_ref, dtype)
    fail = bad_bar & ~within_ulp
    assert np.isfinite(o).all(), "%s has non-finite values" % what
    assert not fail.any(), "%s: %d elements off by more than %g (max err %g)" % (
        what, int(fail.sum()), tol, float(err.max()))
    return {"max_abs_err": float(err.max()), "n_passed_by_ulp_only": int((bad_bar & within_ulp).sum())}


def check_lse(lse_gpu, lse_ref, what="LSE"):
    lse = lse_gpu.detach().cpu().double().numpy() if isinstance(lse_gpu, torch.Tensor) else lse_gpu
    inf_ref = np.isneginf(lse_ref)
    assert (np.isneginf(lse) == inf_ref).all(), "%s: -inf pattern differs" % what
    fin = ~inf_ref
    err = np.abs(lse[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    assert err <= LSE_ATOL, "%s max abs err %g > %g" % (what, err, LSE_ATOL)
    return float(err)


def check_grad(g_gpu, g_ref, what):
    g = to64(g_gpu) if isinstance(g_gpu, torch.Tensor) else g_gpu
    assert np.isfinite(g).all(), "%s has non-finite values" % what
    # floor: where the exact gradient vanishes identically (window (0, 0): one
    # key per row makes dS = P (dP - D) exactly 0) the bar becomes 1e-4 absolute
    denom = max(np.abs(g_ref).max(), GRAD_DENOM_FLOOR)
    rel = np.abs(g - g_ref).max() / denom
    assert rel <= GRAD_RTOL, "%s max rel err %g > %g" % (what, rel, GRAD_RTOL)
    return float(rel)
