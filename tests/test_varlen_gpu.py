"""GPU parity of the variable-length (packed, no padding) forward and backward.

Each sequence of a packed batch is compared with the fp64 oracle run on that
sequence alone; lengths are ragged (not tile multiples), include a
one-token sequence, and queries and keys may differ in length.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from tests.parity import check_grad, check_lse, check_o, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def packed_inputs(lens_q, lens_k, Hq, Hkv, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    tq, tk = sum(lens_q), sum(lens_k)
    q = torch.randn(tq, Hq, d, generator=g).to(dtype)
    k = torch.randn(tk, Hkv, d, generator=g).to(dtype)
    v = torch.randn(tk, Hkv, d, generator=g).to(dtype)
    do = torch.randn(tq, Hq, d, generator=g).to(dtype)
    cu_q = torch.tensor([0] + list(np.cumsum(lens_q)), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(np.cumsum(lens_k)), dtype=torch.int32)
    return q, k, v, do, cu_q, cu_k


CASES = [
    # lens_q, lens_k, Hq, Hkv, d, dtype, causal, window
    ([300, 1, 129, 512, 77], None, 4, 2, 64, torch.float16, True, (-1, -1)),
    ([300, 1, 129, 512, 77], None, 4, 2, 128, torch.bfloat16, False, (-1, -1)),
    ([200, 333, 64], [333, 200, 64], 2, 1, 64, torch.bfloat16, True, (-1, -1)),
    ([257, 380], None, 8, 2, 128, torch.bfloat16, True, (100, 0)),
    # head-pair work tiles (even GQA group, short window) with Nq != Nk per sequence
    ([150, 700, 33], [400, 650, 33], 4, 2, 64, torch.float16, False, (60, 30)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "q%s_d%d_c%d" % (len(c[0]), c[4], c[6]))
def test_varlen_matches_per_sequence_oracle(case):
    lens_q, lens_k, Hq, Hkv, d, dtype, causal, window = case
    lens_k = lens_k or lens_q
    q, k, v, do, cu_q, cu_k = packed_inputs(lens_q, lens_k, Hq, Hkv, d, dtype, 40)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    cqd, ckd = cu_q.to(DEV), cu_k.to(DEV)
    scale = d ** -0.5
    o, lse = fa.fa_fwd_varlen(qd, kd, vd, cqd, ckd, max(lens_q), max(lens_k), softmax_scale=scale,
                              causal=causal, window_size=window)
    dq, dk, dv = fa.fa_bwd_varlen(dod, qd, kd, vd, o, lse, cqd, ckd, max(lens_q), max(lens_k),
                                  softmax_scale=scale, causal=causal, window_size=window)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    for bi in range(len(lens_q)):
        q0, q1 = int(cu_q[bi]), int(cu_q[bi + 1])
        k0, k1 = int(cu_k[bi]), int(cu_k[bi + 1])
        sq, sk, sv, sdo = (to64(t)[None] for t in (q[q0:q1], k[k0:k1], v[k0:k1], do[q0:q1]))
        o_ref, lse_ref = oracle.attention_fwd(sq, sk, sv, scale, causal, window)
        check_o(o[q0:q1][None], o_ref, dtype, "O[seq %d]" % bi)
        check_lse(lse[:, q0:q1][None], lse_ref, "LSE[seq %d]" % bi)
        dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(sq, sk, sv, sdo, scale, causal, window)
        check_grad(dq[q0:q1][None], dq_r, "dQ[seq %d]" % bi)
        check_grad(dk[k0:k1][None], dk_r, "dK[seq %d]" % bi)
        check_grad(dv[k0:k1][None], dv_r, "dV[seq %d]" % bi)


def test_varlen_single_sequence_equals_dense():
    q, k, v, do, cu_q, cu_k = packed_inputs([777], [777], 4, 4, 128, torch.bfloat16, 41)
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    o1, l1 = fa.fa_fwd_varlen(qd, kd, vd, cu_q.to(DEV), cu_k.to(DEV), 777, 777, causal=True)
    o2, l2 = fa.fa_fwd(qd[None], kd[None], vd[None], causal=True)
    assert torch.equal(o1, o2[0]) and torch.equal(l1, l2[0])


def test_varlen_benchmark_workload_sampled_sequences():
    """The packed batch the benchmark times (8 sequences, 512-4096 tokens, d 128,
    causal), in that launch configuration; the oracle checks one head of two of
    its sequences (forward and backward)."""
    from seeded_inputs import VARLEN_WORKLOADS, make_varlen_inputs
    w = VARLEN_WORKLOADS["varlen_8seq_512to4096_h16_d128_bf16_causal"]
    q, k, v, do, cu, lens = make_varlen_inputs(w)
    qd, kd, vd, dod, cud = (t.to(DEV) for t in (q, k, v, do, cu))
    mx = max(lens)
    o, lse = fa.fa_fwd_varlen(qd, kd, vd, cud, cud, mx, mx, softmax_scale=w.softmax_scale,
                              causal=True)
    dq, dk, dv = fa.fa_bwd_varlen(dod, qd, kd, vd, o, lse, cud, cud, mx, mx,
                                  softmax_scale=w.softmax_scale, causal=True)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    h = 3
    for bi in (1, 6):  # the longest and the shortest sequence
        a, z = int(cu[bi]), int(cu[bi + 1])
        sl = (slice(a, z), slice(h, h + 1))
        sq, sk, sv, sdo = (to64(t[sl])[None] for t in (q, k, v, do))
        o_ref, lse_ref = oracle.attention_fwd(sq, sk, sv, w.softmax_scale, True)
        check_o(o[sl][None], o_ref, w.dtype)
        check_lse(lse[h:h + 1, a:z][None], lse_ref)
        dq_r, dk_r, dv_r, _, _ = oracle.attention_bwd(sq, sk, sv, sdo, w.softmax_scale, True)
        check_grad(dq[sl][None], dq_r, "dQ")
        check_grad(dk[sl][None], dk_r, "dK")
        check_grad(dv[sl][None], dv_r, "dV")
