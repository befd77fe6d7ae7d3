"""GPU parity of the forward and backward with dropout against the fp64 oracle.

The kernels and the oracle draw the keep bits independently from Philox4x32-10
(pinned to its published known-answer vectors on the oracle side); a single
differing bit moves O by a whole term, so the O and gradient bars below also
check that every keep bit agrees.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import WORKLOADS, make_qkv, make_workload_inputs, sample_rows
from tests.parity import check_grad, check_lse, check_o, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"

CASES = [
    # B, Nq, Nk, Hq, Hkv, d, dtype, causal, window, p, seed, offset
    (2, 300, 300, 4, 2, 64, torch.float16, False, (-1, -1), 0.1, 1234, 0),
    (1, 257, 257, 4, 4, 128, torch.bfloat16, True, (-1, -1), 0.5, 0xDEADBEEF12345678, 7),
    (1, 200, 333, 2, 1, 64, torch.bfloat16, False, (40, 20), 0.25, 99, 3),
    (2, 129, 129, 2, 2, 128, torch.float16, True, (-1, -1), 0.3, 5, 1),
    # enough heads to fill the SMs, so the causal forward keeps two query tiles
    # per CTA (the smaller causal cases above take one)
    (2, 300, 300, 40, 8, 64, torch.float16, True, (-1, -1), 0.2, 77, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "d%d_p%g_c%d" % (c[5], c[9], c[7]))
def test_dropout_fwd_bwd_match_oracle(case):
    B, Nq, Nk, Hq, Hkv, d, dtype, causal, window, p, seed, offset = case
    q, k, v, do = make_qkv(B, Nq, Nk, Hq, Hkv, d, dtype, 80, with_dout=True)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    scale = d ** -0.5
    kw = dict(softmax_scale=scale, causal=causal, window_size=window, dropout_p=p, seed=seed,
              offset=offset)
    o, lse = fa.fa_fwd(qd, kd, vd, **kw)
    dq, dk, dv = fa.fa_bwd(dod, qd, kd, vd, o, lse, **kw)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    T = oracle.dropout_keep_threshold(p)
    o_ref, lse_ref = oracle.attention_fwd_dropout(to64(q), to64(k), to64(v), scale, T, seed,
                                                  offset, causal, window)
    check_o(o, o_ref, dtype)
    check_lse(lse, lse_ref)
    # the backward from the kernel's own O (D = rowsum(dO o O) uses it)
    gq, gk, gv, _, _ = oracle.attention_bwd_dropout(to64(q), to64(k), to64(v), to64(do), scale,
                                                    T, seed, offset, causal, window)
    check_grad(dq, gq, "dQ")
    check_grad(dk, gk, "dK")
    check_grad(dv, gv, "dV")


def test_dropout_seed_and_offset_matter():
    q, k, v = (t.to(DEV) for t in make_qkv(1, 128, 128, 2, 2, 64, torch.bfloat16, 81))
    a, la = fa.fa_fwd(q, k, v, dropout_p=0.2, seed=1, offset=0)
    b, lb = fa.fa_fwd(q, k, v, dropout_p=0.2, seed=1, offset=0)
    c, _ = fa.fa_fwd(q, k, v, dropout_p=0.2, seed=2, offset=0)
    e, _ = fa.fa_fwd(q, k, v, dropout_p=0.2, seed=1, offset=1)
    plain, lp = fa.fa_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)                 # deterministic for one seed and offset
    assert not torch.equal(a, c) and not torch.equal(a, e)
    assert torch.equal(la, lp)               # LSE ignores dropout
    z, _ = fa.fa_fwd(q, k, v, dropout_p=1e-4, seed=3)  # T = 256: nothing dropped
    assert torch.equal(z, plain)


def test_dropout_rejects_p_near_one():
    q, k, v = (t.to(DEV) for t in make_qkv(1, 64, 64, 1, 1, 64, torch.bfloat16, 82))
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd(q, k, v, dropout_p=0.999)
    assert e.value.status == fa.FA_ERR_INVALID_ARG


def test_dropout_full_size_rows_past_8192():
    # the benchmark's dropout workload (16384 tokens, 16 heads, d 128, bf16,
    # causal, p = 0.1): rows above 2^13 and keys up to 16383 exercise the
    # high bits of the generator's row and column counters, which the small
    # cases above never reach
    w = WORKLOADS["fwdbwd_1x16384_h16_d128_bf16_causal"]
    q, k, v = make_workload_inputs(w, with_dout=False)
    p, seed, offset = 0.1, 1234, 0
    o, lse = fa.fa_fwd(q.to(DEV), k.to(DEV), v.to(DEV), softmax_scale=w.softmax_scale,
                       causal=True, dropout_p=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    rows = sample_rows(w.batch, w.q_heads, w.seqlen_q, 48, w.seed + 100)
    extra = np.array([[0, h, i] for h, i in ((0, 8191), (1, 8192), (5, 12345), (15, 16383),
                                             (7, 16256), (9, 10240))])
    rows = np.unique(np.concatenate([rows, extra]), axis=0)
    assert (rows[:, 2] > 8192).sum() >= 20
    T = oracle.dropout_keep_threshold(p)
    o_ref, lse_ref = oracle.attention_fwd_rows_dropout(to64(q), to64(k), to64(v), rows,
                                                       w.softmax_scale, T, seed, offset, True)
    o_cpu, lse_cpu = o.cpu(), lse.cpu()
    o_rows = np.stack([to64(o_cpu[b, i, h]) for b, h, i in rows])
    lse_rows = np.array([float(lse_cpu[b, h, i]) for b, h, i in rows])
    check_o(o_rows, o_ref, w.dtype)
    check_lse(lse_rows, lse_ref)


VARLEN_CASES = [
    # lengths q, lengths k, Hq, Hkv, d, dtype, causal, p, seed, offset.  The
    # causal one-token sequence has one key per row, so its exact dQ and dK
    # vanish; p = 0.5 (multiplier 2) keeps O = 2 V exact in fp16, so D = dP
    # holds exactly on the GPU as well (at p = 0.2 the multiplier 256 / 205
    # rounds O, and dQ becomes rounding noise of about 1e-3 on a zero).
    ([300, 1, 129, 64], [300, 1, 129, 64], 4, 2, 64, torch.float16, True, 0.5, 4321, 5),
    ([130, 257, 1, 77], [200, 40, 3, 128], 4, 4, 128, torch.bfloat16, False, 0.1, 2 ** 40 + 9, 0),
]


@pytest.mark.parametrize("case", VARLEN_CASES, ids=lambda c: "d%d_c%d" % (c[4], c[6]))
def test_dropout_varlen_matches_dense_slot(case):
    """Packed sequences with dropout.  Sequence b draws the keep bits a dense
    batch draws at batch index b with positions counted from the start of the
    sequence, so the oracle runs a dense batch of b + 1 slots whose slot b
    holds sequence b (the others are zeros) and slot b is compared."""
    lq, lk, Hq, Hkv, d, dtype, causal, p, seed, offset = case
    seqs = [make_qkv(1, nq, nk, Hq, Hkv, d, dtype, 90 + b, with_dout=True)
            for b, (nq, nk) in enumerate(zip(lq, lk))]
    q, k, v, do = (torch.cat([s[i][0] for s in seqs]) for i in range(4))
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32, device=DEV)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32, device=DEV)
    scale = d ** -0.5
    kw = dict(softmax_scale=scale, causal=causal, dropout_p=p, seed=seed, offset=offset)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    o, lse = fa.fa_fwd_varlen(qd, kd, vd, cu_q, cu_k, max(lq), max(lk), **kw)
    dq, dk, dv = fa.fa_bwd_varlen(dod, qd, kd, vd, o, lse, cu_q, cu_k, max(lq), max(lk), **kw)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    T = oracle.dropout_keep_threshold(p)
    for b, (nq, nk) in enumerate(zip(lq, lk)):
        def slot(t, n):
            full = torch.zeros((b + 1, n) + tuple(t.shape[2:]), dtype=t.dtype)
            full[b] = t[0]
            return to64(full)
        sq, sk, sv, sdo = seqs[b]
        o_ref, lse_ref = oracle.attention_fwd_dropout(slot(sq, nq), slot(sk, nk), slot(sv, nk),
                                                      scale, T, seed, offset, causal)
        r0, r1, c0, c1 = sum(lq[:b]), sum(lq[:b + 1]), sum(lk[:b]), sum(lk[:b + 1])
        check_o(o[r0:r1], o_ref[b], dtype, "O of sequence %d" % b)
        check_lse(lse[:, r0:r1], lse_ref[b], "LSE of sequence %d" % b)
        gq, gk, gv, _, _ = oracle.attention_bwd_dropout(slot(sq, nq), slot(sk, nk), slot(sv, nk),
                                                        slot(sdo, nq), scale, T, seed, offset,
                                                        causal)
        check_grad(dq[r0:r1], gq[b], "dQ of sequence %d" % b)
        check_grad(dk[c0:c1], gk[b], "dK of sequence %d" % b)
        check_grad(dv[c0:c1], gv[b], "dV of sequence %d" % b)
