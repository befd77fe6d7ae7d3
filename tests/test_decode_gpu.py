"""GPU parity of decode against a paged KV cache (fa_fwd_paged).

Every case is compared with the fp64 oracle's paged entry point, which reads
the cache through the same block table.  The caches hold NaN in every row and
page a sequence does not own, so a kernel that let such a row reach the
output would fail.  Cases cover ragged lengths around the page and tile sizes,
one-key and empty sequences, more queries than keys, pages smaller than,
equal to and larger than a 128-key tile, GQA groups up to the 128-row limit,
windows, and forced and automatic key splits.
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa
import oracle
from seeded_inputs import PAGED_WORKLOADS, make_paged_inputs
from tests.parity import check_lse, check_o, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
F16, BF16 = torch.float16, torch.bfloat16

CASES = [
    # B, Nq, Hq, Hkv, d, dtype, page, lens, causal, window, num_splits
    (5, 1, 32, 8, 128, BF16, 16, [1, 15, 16, 17, 700], True, (-1, -1), 0),
    (5, 1, 32, 8, 128, BF16, 16, [1, 15, 16, 17, 700], True, (-1, -1), 1),
    (5, 1, 32, 8, 128, BF16, 16, [1, 15, 16, 17, 700], True, (-1, -1), 3),
    (3, 4, 8, 8, 64, F16, 8, [4, 300, 129], True, (-1, -1), 0),
    (3, 4, 8, 2, 64, F16, 32, [2, 300, 129], True, (20, -1), 2),
    (2, 16, 16, 2, 128, BF16, 256, [1000, 37], False, (-1, -1), 0),
    (2, 1, 4, 4, 128, BF16, 128, [0, 513], True, (-1, -1), 0),
    (4, 2, 8, 4, 64, BF16, 64, [64, 65, 127, 1280], False, (5, 5), 4),
    (2, 3, 6, 3, 128, F16, 16, [2049, 1], True, (-1, -1), 0),
]


def _ids(c):
    return "B%d_q%d_h%d-%d_d%d_p%d_s%d" % (c[0], c[1], c[2], c[3], c[4], c[6], c[10])


def run_case(B, Nq, Hq, Hkv, d, dtype, page, lens, causal, window, num_splits, seed=50):
    q, kc, vc, bt, sl = make_paged_inputs(B, Nq, Hq, Hkv, d, dtype, page, lens, seed)
    scale = d ** -0.5
    o, lse = fa.fa_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV),
                             softmax_scale=scale, causal=causal, window_size=window,
                             num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    o_ref, lse_ref = oracle.attention_fwd_paged(to64(q), to64(kc), to64(vc), bt.numpy(),
                                                sl.numpy(), scale, causal, window)
    return o, lse, o_ref, lse_ref


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_decode_matches_oracle(case):
    o, lse, o_ref, lse_ref = run_case(*case)
    check_o(o, o_ref, case[5])
    check_lse(lse, lse_ref)


def test_split_counts_agree():
    # the same problem under 1, 2, 7 and automatic splits
    base = (3, 1, 16, 4, 128, BF16, 16, [1500, 1, 640], True, (-1, -1))
    outs = []
    for ns in (1, 2, 7, 0):
        o, lse, o_ref, lse_ref = run_case(*base, ns)
        check_o(o, o_ref, BF16)
        check_lse(lse, lse_ref)
        outs.append(to64(o))
    for x in outs[1:]:
        assert np.abs(x - outs[0]).max() <= 2 * 2.0 ** -7 * max(1.0, np.abs(outs[0]).max())


def test_noncontiguous_q_and_o():
    B, Nq, Hq, Hkv, d, page = 2, 2, 8, 2, 64, 16
    q, kc, vc, bt, sl = make_paged_inputs(B, Nq, Hq, Hkv, d, F16, page, [333, 90], 51)
    qd = torch.zeros((B, Nq, Hq, 2 * d), dtype=F16, device=DEV)[..., :d]
    qd.copy_(q.to(DEV))
    out = torch.zeros((B, Nq, Hq, 2 * d), dtype=F16, device=DEV)[..., d:]
    o, lse = fa.fa_fwd_paged(qd, kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV),
                             softmax_scale=0.125, causal=True, out=out)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_fwd_paged(to64(q), to64(kc), to64(vc), bt.numpy(),
                                                sl.numpy(), 0.125, True)
    check_o(o, o_ref, F16)
    check_lse(lse, lse_ref)


def test_rejects_unsupported_shapes():
    q, kc, vc, bt, sl = make_paged_inputs(1, 17, 8, 1, 64, BF16, 16, [40], 52)  # 8 x 17 rows
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV))
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
    q, kc, vc, bt, sl = make_paged_inputs(1, 1, 8, 1, 64, BF16, 12, [40], 52)  # page not 2^k
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV))
    assert e.value.status == fa.FA_ERR_INVALID_ARG
    q, kc, vc, bt, sl = make_paged_inputs(1, 1, 8, 1, 64, BF16, 16, [4000], 52)
    ws = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV), num_splits=4,
                        workspace=ws)
    assert e.value.status == fa.FA_ERR_WORKSPACE


def test_decode_workload_full_size_sampled():
    # the benchmarked decode workload, in the launch configuration the bench
    # times; a sample of sequences (shortest, longest and random) is checked
    # against the oracle on a cache holding just that sequence's pages
    w = PAGED_WORKLOADS["decode_128seq_512to8192_h32kv8_d128_bf16_page16"]
    lens = w.lengths()
    q, kc, vc, bt, sl = make_paged_inputs(w.n_seqs, w.Nq, w.q_heads, w.kv_heads, w.head_dim,
                                          w.dtype, w.page_size, lens, w.seed)
    o, lse = fa.fa_fwd_paged(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV),
                             softmax_scale=w.softmax_scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.get_device_error() == fa.FA_OK
    rng = np.random.default_rng(7)
    picks = sorted({int(np.argmin(lens)), int(np.argmax(lens))} |
                   set(rng.choice(w.n_seqs, 4, replace=False).tolist()))
    for b in picks:
        n_pages = (lens[b] + w.page_size - 1) // w.page_size
        pages = bt[b, :n_pages].long()
        sub_bt = np.arange(n_pages, dtype=np.int32)[None]
        o_ref, lse_ref = oracle.attention_fwd_paged(to64(q[b:b + 1]), to64(kc[pages]),
                                                    to64(vc[pages]), sub_bt, [lens[b]],
                                                    w.softmax_scale, w.causal)
        check_o(o[b:b + 1], o_ref, w.dtype, "O[seq %d]" % b)
        check_lse(lse[b:b + 1], lse_ref, "LSE[seq %d]" % b)
