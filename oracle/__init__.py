"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or runs it, and shares no code with
it.

The arithmetic lives in ``fa_oracle.c`` (plain C, fp64, one row or one key at
a time, the textbook definition written out); this module only marshals numpy
arrays through ``ctypes``.  See that file's header for the passages of the
pages it follows and the readings it takes where they are silent.

Every function here is pinned by ``tests/test_oracle_pins.py`` (brute force
with ``math.fsum``, closed forms, invariants, the MQA equivalence, the
8-token / 2x2-block walkthrough and central finite differences); no function
is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the C oracle into a shared library with gcc (no BLAS)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                               "-ffp-contract=off", "-o", tmp, src, "-lm", "-lpthread"])
        os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [batch, seq, heads, head_dim]")
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if Bk != B or dk != d or v.shape != k.shape:
        raise ValueError("inconsistent q/k/v shapes %s %s %s" % (q.shape, k.shape, v.shape))
    if Hq % Hkv:
        raise ValueError("q heads must be a multiple of kv heads")
    return B, Nq, Nk, Hq, Hkv, d


def _mask_args(causal, window_size):
    wl, wr = window_size
    return int(bool(causal)), int(wl), int(wr)


class Oracle:
    """The C oracle loaded from one shared library (the default build, or a
    deliberately mutated copy in the mutation tests)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        i, dbl = ctypes.c_int, ctypes.c_double
        shape = [i, i, i, i, i, i, dbl, i, i, i]
        lib.oracle_fwd.argtypes = [dp, dp, dp, dp, dp] + shape + [i]
        lib.oracle_fwd.restype = i
        lib.oracle_fwd_rows.argtypes = [dp, dp, dp, ip, ctypes.c_long, dp, dp] + shape + [i]
        lib.oracle_fwd_rows.restype = i
        lib.oracle_probs.argtypes = [dp, dp, i, i, dp] + shape
        lib.oracle_probs.restype = i
        lib.oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp] + shape + [i]
        lib.oracle_bwd.restype = i
        ipt = ctypes.POINTER(ctypes.c_int)
        lib.oracle_fwd_paged.argtypes = [dp, dp, dp, ipt, ipt, dp, dp] + [i] * 8 + [dbl, i, i, i, i]
        lib.oracle_fwd_paged.restype = i
        u32p = ctypes.POINTER(ctypes.c_uint32)
        u64, u32 = ctypes.c_uint64, ctypes.c_uint32
        lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        lib.oracle_philox4x32_10.restype = i
        lib.oracle_dropout_keep.argtypes = [u64, u32, ctypes.c_long, ctypes.c_long,
                                            ctypes.c_long, i]
        lib.oracle_dropout_keep.restype = i
        lib.oracle_fwd_dropout.argtypes = [dp, dp, dp, dp, dp] + shape + [i, u64, u32, i]
        lib.oracle_fwd_dropout.restype = i
        lib.oracle_fwd_rows_dropout.argtypes = ([dp, dp, dp, ip, ctypes.c_long, dp, dp] + shape +
                                                [i, u64, u32, i])
        lib.oracle_fwd_rows_dropout.restype = i
        lib.oracle_bwd_dropout.argtypes = [dp] * 9 + shape + [i, u64, u32, i]
        lib.oracle_bwd_dropout.restype = i
        lib.oracle_default_threads.argtypes = []
        lib.oracle_default_threads.restype = i
        self.lib = lib
        self.path = path

    def default_threads(self) -> int:
        return self.lib.oracle_default_threads()

    def attention_fwd(self, q, k, v, softmax_scale, causal=False, window_size=(-1, -1),
                      nthreads=0):
        """O [B,Nq,Hq,d] and LSE [B,Hq,Nq] (natural log), all fp64."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        o = np.zeros((B, Nq, Hq, d), np.float64)
        lse = np.zeros((B, Hq, Nq), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Nq, Nk, Hq,
                                 Hkv, d, float(softmax_scale), c, wl, wr, int(nthreads))
        if rc:
            raise RuntimeError("oracle_fwd failed")
        return o, lse

    def attention_fwd_rows(self, q, k, v, rows, softmax_scale, causal=False,
                           window_size=(-1, -1), nthreads=0):
        """O [n,d] and LSE [n] for selected rows; ``rows`` is int [n, 3] of (b, h, i)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows.shape[0]
        o = np.zeros((n, d), np.float64)
        lse = np.zeros((n,), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v),
                                      rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
                                      _ptr(o), _ptr(lse), B, Nq, Nk, Hq, Hkv, d,
                                      float(softmax_scale), c, wl, wr, int(nthreads))
        if rc:
            raise RuntimeError("oracle_fwd_rows failed (row index out of range?)")
        return o, lse

    def attention_probs(self, q, k, b, h, softmax_scale, causal=False, window_size=(-1, -1)):
        """The full probability matrix P [Nq, Nk] of batch b, query head h."""
        q, k = _f64(q), _f64(k)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, k)
        p = np.zeros((Nq, Nk), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_probs(_ptr(q), _ptr(k), int(b), int(h), _ptr(p), B, Nq, Nk, Hq,
                                   Hkv, d, float(softmax_scale), c, wl, wr)
        if rc:
            raise RuntimeError("oracle_probs failed")
        return p

    def attention_fwd_paged(self, q, k_cache, v_cache, block_table, cache_seqlens, softmax_scale,
                            causal=False, window_size=(-1, -1), nthreads=0):
        """O [B,Nq,Hq,d] and LSE [B,Hq,Nq] of q against a paged KV cache.

        ``k_cache``/``v_cache`` are [num_pages, page_size, Hkv, d];
        ``block_table`` is int [B, max_pages_per_seq]; sequence b holds
        ``cache_seqlens[b]`` keys."""
        q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
        if q.ndim != 4 or kc.ndim != 4 or vc.shape != kc.shape:
            raise ValueError("q must be [B,Nq,Hq,d] and the caches [pages,page_size,Hkv,d]")
        B, Nq, Hq, d = q.shape
        num_pages, P, Hkv, dk = kc.shape
        if dk != d or Hq % Hkv:
            raise ValueError("inconsistent q / cache shapes")
        bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
        sl = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
        if bt.ndim != 2 or bt.shape[0] != B or sl.shape != (B,):
            raise ValueError("block_table must be [B, max_pages] and cache_seqlens [B]")
        o = np.zeros((B, Nq, Hq, d), np.float64)
        lse = np.zeros((B, Hq, Nq), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        ipt = ctypes.POINTER(ctypes.c_int)
        rc = self.lib.oracle_fwd_paged(_ptr(q), _ptr(kc), _ptr(vc), bt.ctypes.data_as(ipt),
                                       sl.ctypes.data_as(ipt), _ptr(o), _ptr(lse), B, Nq, Hq,
                                       Hkv, d, P, num_pages, bt.shape[1], float(softmax_scale),
                                       c, wl, wr, int(nthreads))
        if rc:
            raise RuntimeError("oracle_fwd_paged failed (bad seqlen or page id?)")
        return o, lse

    def philox4x32_10(self, counter, key):
        """Philox4x32-10 of a 4-word counter and 2-word key: four uint32 words."""
        ctr = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in counter])
        k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        out = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(ctr, k, out)
        return [int(x) for x in out]

    def dropout_keep(self, seed, offset, bh, i, j, T):
        return bool(self.lib.oracle_dropout_keep(int(seed), int(offset), int(bh), int(i), int(j),
                                                 int(T)))

    def attention_fwd_dropout(self, q, k, v, softmax_scale, keep_T, seed, offset, causal=False,
                              window_size=(-1, -1), nthreads=0):
        """O and LSE with dropout at keep threshold keep_T (1..255)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        o = np.zeros((B, Nq, Hq, d), np.float64)
        lse = np.zeros((B, Hq, Nq), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Nq, Nk,
                                         Hq, Hkv, d, float(softmax_scale), c, wl, wr, int(keep_T),
                                         int(seed), int(offset), int(nthreads))
        if rc:
            raise RuntimeError("oracle_fwd_dropout failed")
        return o, lse

    def attention_fwd_rows_dropout(self, q, k, v, rows, softmax_scale, keep_T, seed, offset,
                                   causal=False, window_size=(-1, -1), nthreads=0):
        """O [n,d] and LSE [n] with dropout for selected rows (b, h, i)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        n = rows.shape[0]
        o = np.zeros((n, d), np.float64)
        lse = np.zeros((n,), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_fwd_rows_dropout(
            _ptr(q), _ptr(k), _ptr(v), rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n,
            _ptr(o), _ptr(lse), B, Nq, Nk, Hq, Hkv, d, float(softmax_scale), c, wl, wr,
            int(keep_T), int(seed), int(offset), int(nthreads))
        if rc:
            raise RuntimeError("oracle_fwd_rows_dropout failed")
        return o, lse

    def attention_bwd_dropout(self, q, k, v, dout, softmax_scale, keep_T, seed, offset,
                              causal=False, window_size=(-1, -1), nthreads=0):
        """dQ, dK, dV, LSE and D with dropout at keep threshold keep_T."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        lse = np.zeros((B, Hq, Nq), np.float64)
        D = np.zeros((B, Hq, Nq), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                         _ptr(dk), _ptr(dv), _ptr(lse), _ptr(D), B, Nq, Nk, Hq,
                                         Hkv, d, float(softmax_scale), c, wl, wr, int(keep_T),
                                         int(seed), int(offset), int(nthreads))
        if rc:
            raise RuntimeError("oracle_bwd_dropout failed")
        return dq, dk, dv, lse, D

    def attention_bwd(self, q, k, v, dout, softmax_scale, causal=False, window_size=(-1, -1),
                      nthreads=0):
        """dQ, dK, dV of L = sum(dout * O), plus the oracle's own LSE and D (fp64)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, Nq, Nk, Hq, Hkv, d = _dims(q, k, v)
        if dout.shape != q.shape:
            raise ValueError("dout must have the shape of q")
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        lse = np.zeros((B, Hq, Nq), np.float64)
        D = np.zeros((B, Hq, Nq), np.float64)
        c, wl, wr = _mask_args(causal, window_size)
        rc = self.lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                 _ptr(dv), _ptr(lse), _ptr(D), B, Nq, Nk, Hq, Hkv, d,
                                 float(softmax_scale), c, wl, wr, int(nthreads))
        if rc:
            raise RuntimeError("oracle_bwd failed")
        return dq, dk, dv, lse, D


_default = None


def _get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def default_threads() -> int:
    return _get().default_threads()


def attention_fwd(*a, **kw):
    return _get().attention_fwd(*a, **kw)


def attention_fwd_rows(*a, **kw):
    return _get().attention_fwd_rows(*a, **kw)


def attention_probs(*a, **kw):
    return _get().attention_probs(*a, **kw)


def attention_bwd(*a, **kw):
    return _get().attention_bwd(*a, **kw)


def attention_fwd_paged(*a, **kw):
    return _get().attention_fwd_paged(*a, **kw)


def attention_fwd_dropout(*a, **kw):
    return _get().attention_fwd_dropout(*a, **kw)


def attention_fwd_rows_dropout(*a, **kw):
    return _get().attention_fwd_rows_dropout(*a, **kw)


def attention_bwd_dropout(*a, **kw):
    return _get().attention_bwd_dropout(*a, **kw)


def dropout_keep_threshold(p: float) -> int:
    """T = round(256 (1 - p)): an element is kept iff its random byte is below T."""
    return int(round(256.0 * (1.0 - float(p))))
