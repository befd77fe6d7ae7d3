"""Pins of the fp64 CPU oracle to things other than itself (CPU only).

Each check below ties the oracle to a source independent of its code:
  * a pure-Python brute force with exact summation (math.fsum) on tiny inputs;
  * torch's fp64 scaled_dot_product_attention (a library routine) with masks
    built from tril/triu rather than the oracle's index arithmetic;
  * closed forms (Q = 0, causal row 0, a single visible key, scale 0, a
    hand-derived 2-token example stored under tests/golden/);
  * invariants of the softmax (rows sum to 1, P >= 0, LSE bounds);
  * the MQA/GQA equivalence to repeated KV heads;
  * the 8-token / 2x2-block walkthrough of the explainer page
    ("Что такое FlashAttention…", section "Учебный вход: схема 8×8 и
    блоки 2×2"): 16 blocks visited in row-major order, each loaded, attended
    and folded into the output with correct normalisation, must equal full
    attention;
  * central finite differences and fp64 torch autograd for the backward;
  * for dropout, the generator's published known-answer vectors, a brute
    force whose mask is decoded in Python from the generator's words, the
    keep rate, and central finite differences of the dropout forward;
  * for the paged KV cache, equality with the (pinned) contiguous definition
    on the gathered keys, through a permuted page table with unrelated
    values in every row and page the sequence does not own.
A mutation test then plants plausible mistakes in copies of the oracle's C
source and checks that these pins catch every one of them.
"""
import itertools
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

MASKS = [
    (False, (-1, -1)),
    (True, (-1, -1)),
    (False, (2, 1)),
    (False, (1, -1)),
    (False, (-1, 0)),
    (True, (3, 3)),
    (False, (0, 0)),
]


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- references

def visible_matrix(Nq, Nk, causal, window):
    """Boolean [Nq, Nk] visibility built from tril/triu (bottom-right aligned)."""
    ones = torch.ones(Nq, Nk, dtype=torch.bool)
    off = Nk - Nq
    m = ones.clone()
    if causal:
        m &= ones.tril(diagonal=off)
    wl, wr = window
    if wl >= 0:
        m &= ones.triu(diagonal=off - wl)
    if wr >= 0:
        m &= ones.tril(diagonal=off + wr)
    return m


def brute_force_fwd(q, k, v, tau, causal, window):
    """Per-element loops, exact sums.  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    vis = visible_matrix(Nq, Nk, causal, window).numpy()
    o = np.zeros((B, Nq, Hq, d))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b, h, i in itertools.product(range(B), range(Hq), range(Nq)):
        g = h * Hkv // Hq
        js = [j for j in range(Nk) if vis[i, j]]
        if not js:
            continue
        s = {j: tau * math.fsum(q[b, i, h, c] * k[b, j, g, c] for c in range(d)) for j in js}
        m = max(s.values())
        z = math.fsum(math.exp(s[j] - m) for j in js)
        lse[b, h, i] = m + math.log(z)
        for c in range(d):
            o[b, i, h, c] = math.fsum(math.exp(s[j] - m) / z * v[b, j, g, c] for j in js)
    return o, lse


def torch_reference(q, k, v, tau, causal, window, dout=None):
    """fp64 torch: explicit softmax with a boolean mask; autograd for grads."""
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    G = q.shape[2] // k.shape[2]
    kk = tk.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vv = tv.repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    qq = tq.permute(0, 2, 1, 3)
    vis = visible_matrix(q.shape[1], k.shape[1], causal, window)
    s = (qq @ kk.transpose(-1, -2)) * tau
    s = s.masked_fill(~vis, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    p = torch.softmax(s, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)  # rows with no visible key
    o = (p @ vv).permute(0, 2, 1, 3)
    grads = None
    if dout is not None:
        (o * torch.tensor(dout)).sum().backward()
        grads = (tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())
    return o.detach().numpy(), lse.detach().numpy(), grads


def sdpa_reference(q, k, v, tau, causal, window):
    G = q.shape[2] // k.shape[2]
    tq = torch.tensor(q).permute(0, 2, 1, 3)
    tk = torch.tensor(k).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    tv = torch.tensor(v).repeat_interleave(G, dim=2).permute(0, 2, 1, 3)
    vis = visible_matrix(q.shape[1], k.shape[1], causal, window)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=vis, scale=tau)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- pin checks
# Each takes an Oracle instance so the mutation test can run it on a mutant.

def check_bruteforce(orc):
    for (Nq, Nk), (Hq, Hkv), (causal, window) in itertools.product(
            [(5, 5), (7, 11), (11, 7)], [(4, 4), (4, 2), (4, 1)], MASKS):
        d = 3
        q = rand((2, Nq, Hq, d), 1)
        k = rand((2, Nk, Hkv, d), 2)
        v = rand((2, Nk, Hkv, d), 3)
        o, lse = orc.attention_fwd(q, k, v, 0.7, causal, window)
        ob, lseb = brute_force_fwd(q, k, v, 0.7, causal, window)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse), np.isinf(lseb))
        fin = np.isfinite(lseb)
        np.testing.assert_allclose(lse[fin], lseb[fin], rtol=0, atol=1e-12)


def check_library_fwd(orc):
    for (causal, window), (Hq, Hkv) in itertools.product(MASKS, [(4, 4), (6, 2), (3, 1)]):
        Nq = Nk = 24
        q = rand((2, Nq, Hq, 16), 11)
        k = rand((2, Nk, Hkv, 16), 12)
        v = rand((2, Nk, Hkv, 16), 13)
        o, lse = orc.attention_fwd(q, k, v, 0.25, causal, window)
        np.testing.assert_allclose(o, sdpa_reference(q, k, v, 0.25, causal, window),
                                   rtol=0, atol=1e-12)
        _, lse_t, _ = torch_reference(q, k, v, 0.25, causal, window)
        np.testing.assert_allclose(lse, lse_t, rtol=0, atol=1e-12)


def check_golden(orc):
    with open(os.path.join(GOLDEN, "two_token_closed_form.json")) as f:
        gd = json.load(f)
    ev = lambda s: eval(s, {"__builtins__": {}}, {"e": math.e, "log": math.log})  # noqa: E731
    q = np.array(gd["q"]).reshape(1, 2, 1, 1)
    k = np.array(gd["k"]).reshape(1, 2, 1, 1)
    v = np.array(gd["v"]).reshape(1, 2, 1, 1)
    for causal in (False, True):
        ref = gd["causal" if causal else "noncausal"]
        o, lse = orc.attention_fwd(q, k, v, gd["scale"], causal)
        np.testing.assert_allclose(o.ravel(), [ev(s) for s in ref["o"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse.ravel(), [ev(s) for s in ref["lse"]], rtol=0, atol=1e-14)
    ref = gd["noncausal"]
    dq, dk, dv, _, _ = orc.attention_bwd(q, k, v, np.ones_like(q), gd["scale"], False)
    np.testing.assert_allclose(dq.ravel(), [ev(s) for s in ref["dq"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk.ravel(), [ev(s) for s in ref["dk"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv.ravel(), [ev(s) for s in ref["dv"]], rtol=0, atol=1e-14)


def check_closed_forms(orc):
    B, N, H, d = 2, 9, 3, 5
    k = rand((B, N, H, d), 21)
    v = rand((B, N, H, d), 22)
    q = rand((B, N, H, d), 23)
    # Q = 0: every visible key scores 0, so O_i is the plain mean of visible V rows
    # and LSE_i = log(#visible), for any scale.
    for causal, window in MASKS:
        vis = visible_matrix(N, N, causal, window).numpy()
        o, lse = orc.attention_fwd(np.zeros_like(q), k, v, 3.0, causal, window)
        for i in range(N):
            js = np.nonzero(vis[i])[0]
            np.testing.assert_allclose(o[:, i], v[:, js].mean(axis=1), rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[:, :, i], math.log(len(js)), rtol=0, atol=1e-13)
    # causal row 0 sees only key 0: O_0 = V_0 and LSE_0 = scale * q_0 . k_0
    o, lse = orc.attention_fwd(q, k, v, 0.6, True)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], 0.6 * np.einsum("bhc,bhc->bh", q[:, 0], k[:, 0]),
                               rtol=0, atol=1e-13)
    # window (0, 0): exactly one visible key per row, O_i = V_i
    o, _ = orc.attention_fwd(q, k, v, 0.6, False, (0, 0))
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
    # scale 0: uniform weights, O_i = mean of V over all keys
    o, lse = orc.attention_fwd(q, k, v, 0.0, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape),
                               rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, math.log(N), rtol=0, atol=1e-13)


def check_invariants(orc):
    q = rand((1, 13, 2, 8), 31) * 2
    k = rand((1, 17, 1, 8), 32) * 2
    for causal, window in MASKS:
        vis = visible_matrix(13, 17, causal, window).numpy()
        for h in range(2):
            p = orc.attention_probs(q, k, 0, h, 0.5, causal, window)
            assert (p >= 0).all()
            assert (p[~vis] == 0).all()
            rows = vis.any(axis=1)
            np.testing.assert_allclose(p[rows].sum(axis=1), 1.0, rtol=0, atol=1e-12)
            assert (p[~rows] == 0).all()
        _, lse = orc.attention_fwd(q, k, k, 0.5, causal, window)
        s = 0.5 * np.einsum("ihc,jc->hij", q[0], k[0, :, 0])
        for h, i in itertools.product(range(2), range(13)):
            js = np.nonzero(vis[i])[0]
            if len(js) == 0:
                assert lse[0, h, i] == -np.inf
                continue
            mx = s[h, i, js].max()
            assert mx - 1e-12 <= lse[0, h, i] <= mx + math.log(len(js)) + 1e-12


def check_mqa_equivalence(orc):
    for G, (causal, window) in itertools.product([2, 4, 8], MASKS[:4]):
        Hkv = 2
        q = rand((2, 12, Hkv * G, 6), 41)
        k = rand((2, 12, Hkv, 6), 42)
        v = rand((2, 12, Hkv, 6), 43)
        do = rand((2, 12, Hkv * G, 6), 44)
        kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
        o, lse = orc.attention_fwd(q, k, v, 0.4, causal, window)
        o2, lse2 = orc.attention_fwd(q, kr, vr, 0.4, causal, window)
        np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)
        dq, dk, dv, _, _ = orc.attention_bwd(q, k, v, do, 0.4, causal, window)
        dq2, dk2, dv2, _, _ = orc.attention_bwd(q, kr, vr, do, 0.4, causal, window)
        np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
        # a shared kv head collects the gradients of every query head in its group
        np.testing.assert_allclose(dk, dk2.reshape(2, 12, Hkv, G, 6).sum(axis=3), rtol=0,
                                   atol=1e-13)
        np.testing.assert_allclose(dv, dv2.reshape(2, 12, Hkv, G, 6).sum(axis=3), rtol=0,
                                   atol=1e-13)


def walkthrough_replay(q, k, v, tau, causal, block=2):
    """The explainer page's 8-token, 2x2-block traversal, replayed in fp64.

    Blocks of the 8x8 score grid (A..P) are visited in row-major order.  For
    each block the Q rows and K/V rows are "loaded", the block's scores are
    computed, and the running output of those Q rows is updated with correct
    normalisation (a running max and running sum per row).  Blocks that a
    causal mask hides completely are skipped.  One head, [N, d] arrays.
    """
    N, d = q.shape
    nb = N // block
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    acc = np.zeros((N, d))
    visited = []
    for bi in range(nb):
        rows = slice(bi * block, (bi + 1) * block)
        for bj in range(nb):
            cols = slice(bj * block, (bj + 1) * block)
            if causal and bj > bi:
                continue
            visited.append("ABCDEFGHIJKLMNOP"[bi * nb + bj])
            s = tau * q[rows] @ k[cols].T
            if causal:
                ii = np.arange(rows.start, rows.stop)[:, None]
                jj = np.arange(cols.start, cols.stop)[None, :]
                s = np.where(jj <= ii, s, -np.inf)
            m_new = np.maximum(m[rows], s.max(axis=1))
            alpha = np.exp(m[rows] - m_new)
            p = np.exp(s - m_new[:, None])
            l[rows] = alpha * l[rows] + p.sum(axis=1)
            acc[rows] = alpha[:, None] * acc[rows] + p @ v[cols]
            m[rows] = m_new
    return acc / l[:, None], m + np.log(l), visited


def check_walkthrough(orc):
    q, k, v = rand((8, 4), 51), rand((8, 4), 52), rand((8, 4), 53)
    for causal in (False, True):
        o_t, lse_t, visited = walkthrough_replay(q, k, v, 0.5, causal)
        assert len(visited) == (10 if causal else 16)
        o, lse = orc.attention_fwd(q[None, :, None], k[None, :, None], v[None, :, None], 0.5,
                                   causal)
        np.testing.assert_allclose(o[0, :, 0], o_t, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, 0], lse_t, rtol=0, atol=1e-13)


def check_backward(orc):
    # central finite differences of L = sum(dO * O) on the fp64 oracle itself
    for (Hq, Hkv), (causal, window) in itertools.product([(2, 2), (4, 2)],
                                                         [(False, (-1, -1)), (True, (-1, -1)),
                                                          (False, (2, 1)), (True, (3, -1))]):
        Nq, Nk, d = 5, 7, 3
        q = rand((1, Nq, Hq, d), 61)
        k = rand((1, Nk, Hkv, d), 62)
        v = rand((1, Nk, Hkv, d), 63)
        do = rand((1, Nq, Hq, d), 64)
        dq, dk, dv, lse, D = orc.attention_bwd(q, k, v, do, 0.8, causal, window)
        o, lse_f = orc.attention_fwd(q, k, v, 0.8, causal, window)
        np.testing.assert_allclose(D, np.einsum("bihc,bihc->bhi", do, o), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(lse, lse_f)

        def loss(qq, kk, vv):
            return float((orc.attention_fwd(qq, kk, vv, 0.8, causal, window)[0] * do).sum())

        eps = 1e-5
        for arr, grad, idx in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(arr)
            for pos in np.ndindex(arr.shape):
                args_p = [q.copy(), k.copy(), v.copy()]
                args_m = [q.copy(), k.copy(), v.copy()]
                args_p[idx][pos] += eps
                args_m[idx][pos] -= eps
                num[pos] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            scale = max(np.abs(num).max(), 1e-3)
            assert np.abs(num - grad).max() / scale < 1e-6, (idx, causal, window)
    # fp64 torch autograd on the materialised definition (library routine)
    for (Hq, Hkv), (causal, window) in itertools.product([(4, 4), (4, 1)], MASKS):
        q = rand((2, 10, Hq, 8), 71)
        k = rand((2, 14, Hkv, 8), 72)
        v = rand((2, 14, Hkv, 8), 73)
        do = rand((2, 10, Hq, 8), 74)
        dq, dk, dv, _, _ = orc.attention_bwd(q, k, v, do, 0.3, causal, window)
        _, _, (tdq, tdk, tdv) = torch_reference(q, k, v, 0.3, causal, window, dout=do)
        np.testing.assert_allclose(dq, tdq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, tdk, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, tdv, rtol=0, atol=1e-12)


def check_empty_rows(orc):
    # Nq > Nk with bottom-right causal alignment: the first Nq - Nk rows see no key
    q = rand((1, 6, 2, 4), 81)
    k = rand((1, 3, 2, 4), 82)
    v = rand((1, 3, 2, 4), 83)
    do = rand((1, 6, 2, 4), 84)
    o, lse = orc.attention_fwd(q, k, v, 0.5, True)
    assert (o[0, :3] == 0).all() and np.isneginf(lse[0, :, :3]).all()
    assert np.isfinite(lse[0, :, 3:]).all()
    np.testing.assert_allclose(o[0, 3], v[0, 0], rtol=0, atol=1e-14)  # sees key 0 only
    dq, dk, dv, _, _ = orc.attention_bwd(q, k, v, do, 0.5, True)
    assert (dq[0, :3] == 0).all()


def scatter_to_pages(k, v, P, extra_pages, seed):
    """Paged caches [pages, P, Hkv, d] holding k/v [B, N, Hkv, d] in a random
    page order; rows past N and the spare pages hold unrelated values, and
    every block-table entry (used or not) names a valid page."""
    B, N, Hkv, d = k.shape
    per_seq = (N + P - 1) // P
    n_pages = B * per_seq + extra_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)
    kc = 50.0 * rng.standard_normal((n_pages, P, Hkv, d))
    vc = 50.0 * rng.standard_normal((n_pages, P, Hkv, d))
    bt = np.zeros((B, per_seq + 2), np.int32)
    for b in range(B):
        for pg in range(per_seq + 2):
            bt[b, pg] = perm[b * per_seq + pg] if pg < per_seq else perm[(-1 - pg) % n_pages]
        for j in range(N):
            kc[bt[b, j // P], j % P] = k[b, j]
            vc[bt[b, j // P], j % P] = v[b, j]
    return kc, vc, bt


def check_paged(orc):
    # a paged cache read through its block table equals the contiguous
    # definition on the gathered keys, for every mask and GQA grouping
    for (causal, window), (Hq, Hkv), P in itertools.product(MASKS, [(4, 4), (4, 2)], [4, 8]):
        B, Nq, N, d = 3, 3, 13, 5
        q, k, v = rand((B, Nq, Hq, d), 121), rand((B, N, Hkv, d), 122), rand((B, N, Hkv, d), 123)
        kc, vc, bt = scatter_to_pages(k, v, P, 3, 124)
        o, lse = orc.attention_fwd_paged(q, kc, vc, bt, [N] * B, 0.6, causal, window)
        oc, lsec = orc.attention_fwd(q, k, v, 0.6, causal, window)
        np.testing.assert_allclose(o, oc, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse), np.isinf(lsec))
        fin = np.isfinite(lsec)
        np.testing.assert_allclose(lse[fin], lsec[fin], rtol=0, atol=1e-12)
    # ragged lengths: each sequence is its own problem, aligned bottom-right
    # against its own length; an empty sequence gives O = 0 and LSE = -inf
    B, Nq, N, Hq, Hkv, d, P = 4, 2, 21, 4, 2, 6, 8
    q, k, v = rand((B, Nq, Hq, d), 131), rand((B, N, Hkv, d), 132), rand((B, N, Hkv, d), 133)
    kc, vc, bt = scatter_to_pages(k, v, P, 2, 134)
    lens = [21, 1, 0, 9]
    o, lse = orc.attention_fwd_paged(q, kc, vc, bt, lens, 0.4, True, (4, -1))
    for b, n in enumerate(lens):
        if n == 0:
            assert (o[b] == 0).all() and np.isneginf(lse[b]).all()
            continue
        ob, lseb = orc.attention_fwd(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], 0.4, True,
                                     (4, -1))
        np.testing.assert_allclose(o[b:b + 1], ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b:b + 1], lseb, rtol=0, atol=1e-12)


def check_philox_kat(orc):
    # the generator behind dropout against its authors' known-answer vectors
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for vec in kat["vectors"]:
        ctr = [int(x, 16) for x in vec["counter"]]
        key = [int(x, 16) for x in vec["key"]]
        assert orc.philox4x32_10(ctr, key) == [int(x, 16) for x in vec["out"]]


def dropout_mask_bruteforce(orc, seed, offset, B, Hq, Nq, Nk, T):
    """Keep mask [B, Hq, Nq, Nk] decoded here from the (KAT-pinned) generator:
    counter (j // 4, i // 4, b Hq + h, offset), key = seed split in two words,
    byte j % 4 of word i % 4, kept iff below T."""
    m = np.zeros((B, Hq, Nq, Nk), bool)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for b in range(B):
        for h in range(Hq):
            for ib in range(0, Nq, 4):
                for jb in range(0, Nk, 4):
                    w = orc.philox4x32_10([jb // 4, ib // 4, b * Hq + h, offset], key)
                    for i in range(ib, min(ib + 4, Nq)):
                        for j in range(jb, min(jb + 4, Nk)):
                            m[b, h, i, j] = ((w[i % 4] >> (8 * (j % 4))) & 0xFF) < T
    return m


def check_dropout(orc):
    seed, offset = 0x1234567890ABCDEF, 3
    for (causal, window), (Hq, Hkv), T in itertools.product(
            [(False, (-1, -1)), (True, (-1, -1)), (False, (2, 1))], [(4, 2)], [26, 179]):
        B, Nq, Nk, d = 2, 7, 9, 3
        q, k, v = rand((B, Nq, Hq, d), 151), rand((B, Nk, Hkv, d), 152), rand((B, Nk, Hkv, d), 153)
        o, lse = orc.attention_fwd_dropout(q, k, v, 0.7, T, seed, offset, causal, window)
        # brute force: the plain probabilities (pinned above), the mask decoded
        # here, and O = (256 / T) sum_j P_ij M_ij V_j; LSE is the plain one
        m = dropout_mask_bruteforce(orc, seed, offset, B, Hq, Nq, Nk, T)
        G = Hq // Hkv
        ob = np.zeros_like(o)
        for b in range(B):
            for h in range(Hq):
                P = orc.attention_probs(q, k, b, h, 0.7, causal, window)
                Z = P * m[b, h] * (256.0 / T)
                ob[b, :, h, :] = Z @ v[b, :, h // G, :]
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
        _, lse_plain = orc.attention_fwd(q, k, v, 0.7, causal, window)
        np.testing.assert_array_equal(lse, lse_plain)
    # the keep rate over many elements is T / 256 (binomial, 5 sigma)
    m = dropout_mask_bruteforce(orc, 77, 0, 1, 2, 64, 64, 64)
    n, kept = m.size, m.sum()
    assert abs(kept - n * 0.25) <= 5 * math.sqrt(n * 0.25 * 0.75)
    # the backward is the gradient of the dropout forward (fixed mask): central
    # finite differences of L = sum(dout * O)
    B, Nq, Nk, Hq, Hkv, d, T = 1, 5, 6, 2, 1, 3, 128
    q, k, v = rand((B, Nq, Hq, d), 161), rand((B, Nk, Hkv, d), 162), rand((B, Nk, Hkv, d), 163)
    do = rand((B, Nq, Hq, d), 164)
    dq, dk, dv, _, _ = orc.attention_bwd_dropout(q, k, v, do, 0.6, T, 9, 1, True)

    def loss(qq, kk, vv):
        return float((orc.attention_fwd_dropout(qq, kk, vv, 0.6, T, 9, 1, True)[0] * do).sum())
    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


ALL_CHECKS = [check_bruteforce, check_library_fwd, check_golden, check_closed_forms,
              check_invariants, check_mqa_equivalence, check_walkthrough, check_backward,
              check_empty_rows, check_paged, check_philox_kat, check_dropout]


@pytest.fixture(scope="module")
def orc():
    return oracle._get()


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, check):
    check(orc)


def test_rows_subset_matches_full(orc):
    q, k, v = rand((2, 33, 4, 16), 91), rand((2, 40, 2, 16), 92), rand((2, 40, 2, 16), 93)
    o, lse = orc.attention_fwd(q, k, v, 0.25, True, (5, -1))
    rows = np.array([[0, 0, 0], [1, 3, 32], [0, 2, 17], [1, 1, 1]])
    orow, lrow = orc.attention_fwd_rows(q, k, v, rows, 0.25, True, (5, -1))
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(orow[r], o[b, i, h])
        assert lrow[r] == lse[b, h, i]
    with pytest.raises(RuntimeError):
        orc.attention_fwd_rows(q, k, v, np.array([[0, 0, 33]]), 0.25)


def test_rows_dropout_subset_matches_full(orc):
    # the row-at-a-time dropout forward picks the same rows, keep bits and
    # rescaling as the full dropout forward (pinned by check_dropout)
    q, k, v = rand((2, 45, 4, 16), 95), rand((2, 50, 2, 16), 96), rand((2, 50, 2, 16), 97)
    T, seed, offset = 200, 0x1234ABCD, 3
    o, lse = orc.attention_fwd_dropout(q, k, v, 0.3, T, seed, offset, True, (7, -1))
    rows = np.array([[0, 0, 0], [1, 3, 44], [0, 2, 17], [1, 1, 5]])
    orow, lrow = orc.attention_fwd_rows_dropout(q, k, v, rows, 0.3, T, seed, offset, True, (7, -1))
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(orow[r], o[b, i, h])
        assert lrow[r] == lse[b, h, i]
    with pytest.raises(RuntimeError):
        orc.attention_fwd_rows_dropout(q, k, v, rows, 0.3, 0, seed, offset)  # T out of range


def test_thread_count_does_not_change_bits(orc):
    q, k, v, do = (rand((1, 37, 2, 8), s) for s in (101, 102, 103, 104))
    a = orc.attention_bwd(q, k, v, do, 0.3, True, nthreads=1)
    b = orc.attention_bwd(q, k, v, do, 0.3, True, nthreads=7)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_paged_rejects_bad_page_ids(orc):
    q, k, v = rand((1, 1, 2, 4), 141), rand((1, 9, 2, 4), 142), rand((1, 9, 2, 4), 143)
    kc, vc, bt = scatter_to_pages(k, v, 4, 0, 144)
    bt = bt.copy()
    bt[0, 1] = kc.shape[0]  # past the last page, inside the sequence
    with pytest.raises(RuntimeError):
        orc.attention_fwd_paged(q, kc, vc, bt, [9], 0.5)
    with pytest.raises(RuntimeError):  # longer than the block table allows
        orc.attention_fwd_paged(q, kc, vc, bt, [4 * bt.shape[1] + 1], 0.5)


def test_rejects_bad_shapes(orc):
    with pytest.raises(ValueError):
        orc.attention_fwd(rand((1, 4, 3, 2), 0), rand((1, 4, 2, 2), 0), rand((1, 4, 2, 2), 0), 1.0)


# ---------------------------------------------------------------- mutation test

MUTATIONS = {
    "scale dropped": ("srow[j] = s->tau * dot(", "srow[j] = dot("),
    "causal off by one": ("if (s->causal && j > ip)", "if (s->causal && j >= ip)"),
    "left window exclusive": ("j < ip - s->wl", "j <= ip - s->wl"),
    "right window ignored": ("if (s->wr >= 0 && j > ip + s->wr) return 0;", ""),
    "top-left causal alignment": ("long ip = i + (long)s->Nk - (long)s->Nq;", "long ip = i;"),
    "GQA heads interleaved": ("int g = h / (s->Hq / s->Hkv);\n    const double* qi",
                              "int g = h % s->Hkv;\n    const double* qi"),
    "max not subtracted back": ("return m + log(sum);", "return log(sum);"),
    "dS sign flipped": ("double dS = prow[j] * (dprow[j] - Di);",
                        "double dS = prow[j] * (Di - dprow[j]);"),
    "D dropped in dK": ("double dSij = Pij * (dPij - c->Dvec[li]);", "double dSij = Pij * dPij;"),
    "dK without scale": ("dkj[cc] += s->tau * dSij * qi[cc];", "dkj[cc] += dSij * qi[cc];"),
    "dV uses dS": ("dvj[cc] += Zij * doi[cc];", "dvj[cc] += dSij * doi[cc];"),
    "dQ uses V": ("const double* kj = kv_row(c->k, s, b, j, g);\n        for",
                  "const double* kj = kv_row(c->v, s, b, j, g);\n        for"),
    "one head per kv group in dK": ("for (int h = g * G; h < (g + 1) * G; ++h)",
                                    "for (int h = g * G; h < g * G + 1; ++h)"),
    "paged row from the page index": ("long row = j % c->P;", "long row = j / c->P;"),
    "paged last key dropped": ("int nk = c->seqlens[b];",
                               "int nk = c->seqlens[b] > 0 ? c->seqlens[b] - 1 : 0;"),
    "paged mask aligned top-left": ("shape_t s = {1, c->Nq, nk,", "shape_t s = {1, c->Nq, c->Nq,"),
    "paged kv head interleaved": ("int kv_head = h / (c->Hq / c->Hkv);", "int kv_head = h % c->Hkv;"),
    "philox key bump skipped": ("k0 += 0x9E3779B9u;", ""),
    "dropout byte from the wrong word": ("uint32_t byte = (w[i % 4] >> (8 * (j % 4))) & 0xFFu;",
                                         "uint32_t byte = (w[j % 4] >> (8 * (i % 4))) & 0xFFu;"),
    "dropout rescale missing": ("? 256.0 / s->drop_T", "? 1.0"),
    "dropout mask left out of dP": (
        "dprow[j] = dot(doi, kv_row(c->v, s, b, j, g), s->d) * drop_mult(s, b, h, i, j);",
        "dprow[j] = dot(doi, kv_row(c->v, s, b, j, g), s->d);"),
    "dV without the dropout mask": ("double Zij = Pij * mult;", "double Zij = Pij;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    before, after = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "fa_oracle.c")).read()
    assert src.count(before) == 1, "mutation anchor not unique: %r" % before
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(before, after))
    lib = oracle.build(force=True, src=str(mutant_src), out=str(tmp_path / "libmutant.so"))
    mutant = oracle.Oracle(lib)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(mutant)
        except (AssertionError, RuntimeError):
            caught.append(check.__name__)
    assert caught, "no pin caught the planted mistake %r" % name
