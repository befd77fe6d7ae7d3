"""Python binding of libfa143.so, the B200 (sm_100a) exact-attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/fa143.h.  PyTorch provides the
device memory and the current stream.  There is no fallback: if the shared
library is missing or a tensor is not on a CUDA device the call raises.

    o, lse = fa_fwd(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1))
    dq, dk, dv = fa_bwd(do, q, k, v, o, lse, softmax_scale=None, causal=False,
                        window_size=(-1, -1))

Tensors use the [batch, seqlen, heads, head_dim] layout and fp16/bf16 of
flash_attn_func ("optimizing-attention-flash", Workflow 2 Steps 2-3);
softmax_scale=None means 1/sqrt(head_dim); k and v may have fewer heads than
q (MQA/GQA); window_size=(left, right) with -1 for unbounded.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa143.so")

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_ALIGNMENT = 3
FA_ERR_WORKSPACE = 4
FA_ERR_CUDA = 5
FA_ERR_DEVICE_TIMEOUT = 6

# names exported by libfa143.so (the declarations of include/fa143.h)
EXPORTED = ("fa_status_string", "fa_fwd", "fa_bwd_workspace_size", "fa_bwd",
            "fa_get_device_error", "fa_set_wait_limit_ns", "fa_set_bwd_main_events",
            "fa_bwd_noalloc", "fa_bwd_noalloc_scratch_bytes", "fa_selftest_wait_timeout", "fa_selftest_exp2", "fa_fwd_varlen", "fa_bwd_varlen",
            "fa_fwd_paged_workspace_size", "fa_fwd_paged", "fa_fwd_fp8", "fa_fwd_dropout",
            "fa_bwd_dropout", "fa_fwd_varlen_dropout", "fa_bwd_varlen_dropout")

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, status_string(status), status))


def load_library(path: str = LIB_PATH):
    """Load libfa143.so and declare its C signatures (no GPU needed)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libfa143.so is not built (%s); run exact_attention_143_b200.build"
                           ".build() or __graft_entry__.build()" % path)
    lib = ctypes.CDLL(path)
    vp, i, f, i64p = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.POINTER(ctypes.c_int64)
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i64p, i64p, i64p, i64p, i, f, i,
                           i, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = ctypes.c_size_t
    lib.fa_bwd.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [i] * 6 + [i64p] * 8 +
                           [i, f, i, i, i, vp])
    lib.fa_bwd.restype = i
    lib.fa_get_device_error.argtypes = [vp]
    lib.fa_get_device_error.restype = i
    lib.fa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.fa_set_wait_limit_ns.restype = ctypes.c_uint64
    lib.fa_set_bwd_main_events.argtypes = [vp, vp]
    lib.fa_set_bwd_main_events.restype = i
    lib.fa_bwd_noalloc.argtypes = [vp] * 9 + [i] * 6 + [i64p] * 8 + [i, f, i, i, i, vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_selftest_exp2.argtypes = [vp, vp, i, i, vp]
    lib.fa_selftest_exp2.restype = i
    lib.fa_bwd_noalloc_scratch_bytes.argtypes = []
    lib.fa_bwd_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_varlen.argtypes = [vp] * 7 + [i] * 8 + [i64p] * 4 + [i, f, i, i, i, vp]
    lib.fa_fwd_varlen.restype = i
    lib.fa_bwd_varlen.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [vp, vp] + [i] * 8 +
                                  [i64p] * 8 + [i, f, i, i, i, vp])
    lib.fa_bwd_varlen.restype = i
    lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.fa_selftest_wait_timeout.restype = i
    lib.fa_fwd_paged_workspace_size.argtypes = [i] * 8
    lib.fa_fwd_paged_workspace_size.restype = ctypes.c_size_t
    lib.fa_fwd_paged.argtypes = ([vp] * 7 + [i] * 8 + [ctypes.c_int64] + [i64p] * 4 +
                                 [i, f, i, i, i, i, vp, ctypes.c_size_t, vp])
    lib.fa_fwd_paged.restype = i
    lib.fa_fwd_fp8.argtypes = [vp] * 5 + [i] * 6 + [i64p] * 4 + [f] * 4 + [i, i, i, vp]
    lib.fa_fwd_fp8.restype = i
    u64, u32 = ctypes.c_uint64, ctypes.c_uint32
    lib.fa_fwd_dropout.argtypes = ([vp, vp, vp, vp, vp, i, i, i, i, i, i, i64p, i64p, i64p, i64p,
                                    i, f, i, i, i, f, u64, u32, vp])
    lib.fa_fwd_dropout.restype = i
    lib.fa_bwd_dropout.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [i] * 6 + [i64p] * 8 +
                                   [i, f, i, i, i, f, u64, u32, vp])
    lib.fa_bwd_dropout.restype = i
    lib.fa_fwd_varlen_dropout.argtypes = ([vp] * 7 + [i] * 8 + [i64p] * 4 +
                                          [i, f, i, i, i, f, u64, u32, vp])
    lib.fa_fwd_varlen_dropout.restype = i
    lib.fa_bwd_varlen_dropout.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [vp, vp] + [i] * 8 +
                                          [i64p] * 8 + [i, f, i, i, i, f, u64, u32, vp])
    lib.fa_bwd_varlen_dropout.restype = i
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return 0
    if t.dtype == torch.bfloat16:
        return 1
    raise TypeError("fp16 or bf16 tensors only (got %s)" % t.dtype)


def _strides(t: torch.Tensor):
    if t.dim() != 4:
        raise ValueError("expected a [batch, seqlen, heads, head_dim] tensor, got shape %s"
                         % (tuple(t.shape),))
    if t.stride(3) != 1 and t.shape[3] > 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def _check_cuda(*ts):
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda:
            raise RuntimeError("tensors must be on a CUDA device (no CPU path exists)")
        if t.device != dev:
            raise RuntimeError("all tensors must be on the same device")
    return dev


def _scale(softmax_scale, d):
    return 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def fa_fwd(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1), out=None, lse=None,
           dropout_p=0.0, seed=0, offset=0):
    """Exact attention forward; returns (o [B,Nq,Hq,d], lse [B,Hq,Nq] fp32).

    With dropout_p > 0 the probabilities are dropped before P V (keep bits
    from Philox4x32-10 keyed by `seed`, counter offset `offset`; the kept ones
    are rescaled by 256 / round(256 (1 - dropout_p))); pass the same seed and
    offset to fa_bwd."""
    lib = load_library()
    dev = _check_cuda(q, k, v)
    code = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    _check_cuda(q, out, lse)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Nq] tensor")
    wl, wr = window_size
    with torch.cuda.device(dev):
        if dropout_p:
            rc = lib.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, Nq, Nk, Hq, Hkv, d, _strides(q),
                                    _strides(k), _strides(v), _strides(out), code,
                                    _scale(softmax_scale, d), int(bool(causal)), int(wl), int(wr),
                                    float(dropout_p), int(seed), int(offset), _stream(dev))
        else:
            rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), B, Nq, Nk, Hq, Hkv, d, _strides(q), _strides(k),
                            _strides(v), _strides(out), code, _scale(softmax_scale, d),
                            int(bool(causal)), int(wl), int(wr), _stream(dev))
    if rc:
        raise FAError(rc, "fa_fwd")
    return out, lse


def _strides2(t: torch.Tensor):
    if t.dim() != 3:
        raise ValueError("expected a packed [tokens, heads, head_dim] tensor, got shape %s"
                         % (tuple(t.shape),))
    if t.stride(2) != 1 and t.shape[2] > 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    return (ctypes.c_int64 * 2)(t.stride(0), t.stride(1))


def _check_cu(cu, n):
    if cu.dtype != torch.int32 or not cu.is_cuda or cu.dim() != 1 or cu.numel() != n + 1 \
            or not cu.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 CUDA tensor of B + 1 offsets")


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                  softmax_scale=None, causal=False, window_size=(-1, -1), out=None, lse=None,
                  dropout_p=0.0, seed=0, offset=0):
    """Forward over a packed variable-length batch (no padding).

    q [total_q, Hq, d], k/v [total_k, Hkv, d]; cu_seqlens_q/k int32 [B+1] on the
    device.  Returns (o [total_q, Hq, d], lse [Hq, total_q] fp32).  With
    dropout_p > 0 the keep bits of sequence b are those a dense batch draws for
    batch index b, at positions counted from the start of the sequence."""
    lib = load_library()
    dev = _check_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k)
    code = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    _check_cu(cu_seqlens_q, B)
    _check_cu(cu_seqlens_k, B)
    if out is None:
        out = torch.empty((total_q, Hq, d), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=dev)
    wl, wr = window_size
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
            cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
            int(max_seqlen_k), total_q, total_k, Hq, Hkv, d, _strides2(q), _strides2(k),
            _strides2(v), _strides2(out), code, _scale(softmax_scale, d), int(bool(causal)),
            int(wl), int(wr))
    with torch.cuda.device(dev):
        if dropout_p:
            name = "fa_fwd_varlen_dropout"
            rc = lib.fa_fwd_varlen_dropout(*args, float(dropout_p), int(seed), int(offset),
                                           _stream(dev))
        else:
            name = "fa_fwd_varlen"
            rc = lib.fa_fwd_varlen(*args, _stream(dev))
    if rc:
        raise FAError(rc, name)
    return out, lse


def fa_bwd_varlen(dout, q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q,
                  max_seqlen_k, softmax_scale=None, causal=False, window_size=(-1, -1),
                  dq=None, dk=None, dv=None, workspace=None, dropout_p=0.0, seed=0, offset=0):
    """Backward over a packed variable-length batch; returns (dq, dk, dv).  dropout_p,
    seed and offset must be those given to the forward."""
    lib = load_library()
    dev = _check_cuda(dout, q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k)
    code = _dtype_code(q)
    for t in (k, v, o, dout):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, o, dout must share one dtype")
    total_q, Hq, d = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    _check_cu(cu_seqlens_q, B)
    _check_cu(cu_seqlens_k, B)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (Hq, total_q):
        raise ValueError("lse must be the contiguous fp32 [Hq, total_q] tensor from fa_fwd_varlen")
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, int(max_seqlen_q), Hq, d), dtype=torch.uint8,
                                device=dev)
    _check_cuda(q, dq, dk, dv, workspace)
    wl, wr = window_size
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), cu_seqlens_q.data_ptr(),
            cu_seqlens_k.data_ptr(), B, int(max_seqlen_q), int(max_seqlen_k), total_q, total_k,
            Hq, Hkv, d, _strides2(q), _strides2(k), _strides2(v), _strides2(o), _strides2(dout),
            _strides2(dq), _strides2(dk), _strides2(dv), code, _scale(softmax_scale, d),
            int(bool(causal)), int(wl), int(wr))
    with torch.cuda.device(dev):
        if dropout_p:
            name = "fa_bwd_varlen_dropout"
            rc = lib.fa_bwd_varlen_dropout(*args, float(dropout_p), int(seed), int(offset),
                                           _stream(dev))
        else:
            name = "fa_bwd_varlen"
            rc = lib.fa_bwd_varlen(*args, _stream(dev))
    if rc:
        raise FAError(rc, name)
    return dq, dk, dv


def bwd_workspace_size(B, Nq, Hq, d) -> int:
    return int(load_library().fa_bwd_workspace_size(B, Nq, Hq, d))


def fa_bwd(dout, q, k, v, o, lse, softmax_scale=None, causal=False, window_size=(-1, -1),
           dq=None, dk=None, dv=None, workspace=None, dropout_p=0.0, seed=0, offset=0):
    """Exact attention backward from the forward's O and LSE; returns (dq, dk, dv)."""
    lib = load_library()
    dev = _check_cuda(dout, q, k, v, o, lse)
    code = _dtype_code(q)
    for t in (k, v, o, dout):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, o, dout must share one dtype")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be the contiguous fp32 [B, Hq, Nq] tensor from fa_fwd")
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    ws_bytes = bwd_workspace_size(B, Nq, Hq, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    _check_cuda(q, dq, dk, dv, workspace)
    wl, wr = window_size
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), B, Nq, Nk, Hq, Hkv, d, _strides(q),
            _strides(k), _strides(v), _strides(o), _strides(dout), _strides(dq), _strides(dk),
            _strides(dv), code, _scale(softmax_scale, d), int(bool(causal)), int(wl), int(wr))
    with torch.cuda.device(dev):
        if dropout_p:
            rc = lib.fa_bwd_dropout(*args, float(dropout_p), int(seed), int(offset), _stream(dev))
        else:
            rc = lib.fa_bwd(*args, _stream(dev))
    if rc:
        raise FAError(rc, "fa_bwd")
    return dq, dk, dv


def get_device_error(device=None) -> int:
    """Synchronise the current stream and return/clear the device error word."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(lib.fa_get_device_error(_stream(dev)))


def set_bwd_main_events(start=None, stop=None) -> None:
    """Have later fa_bwd calls record torch.cuda.Event `start`/`stop` around
    their main kernel (None, None switches it off).  The events must already
    exist on the device (record them once before passing them)."""
    lib = load_library()
    h0 = ctypes.c_void_p(start.cuda_event) if start is not None else None
    h1 = ctypes.c_void_p(stop.cuda_event) if stop is not None else None
    lib.fa_set_bwd_main_events(h0, h1)


def selftest_wait_timeout(limit_ns: int, device=None) -> int:
    """Launch the bounded-wait self-test kernel (see include/fa143.h) and
    return fa_get_device_error()'s status afterwards."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        rc = lib.fa_selftest_wait_timeout(int(limit_ns), _stream(dev))
    if rc:
        raise FAError(rc, "fa_selftest_wait_timeout")
    return get_device_error(dev)


def selftest_exp2(x, bf16=False):
    """2^x by the kernels' FMA-pipe polynomial, for x an fp32 CUDA tensor."""
    lib = load_library()
    dev = _check_cuda(x)
    if x.dtype != torch.float32:
        raise TypeError("x must be fp32")
    x = x.contiguous()
    y = torch.empty_like(x)
    with torch.cuda.device(dev):
        rc = lib.fa_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), int(bool(bf16)),
                                  _stream(dev))
    if rc:
        raise FAError(rc, "fa_selftest_exp2")
    return y


def set_wait_limit_ns(limit_ns: int) -> int:
    return int(load_library().fa_set_wait_limit_ns(int(limit_ns)))


def fa_fwd_paged_workspace_size(B, Nq, Hq, Hkv, d, page_size, max_pages_per_seq, num_splits=0):
    """Bytes of workspace fa_fwd_paged needs (0 when the keys are not split)."""
    return int(load_library().fa_fwd_paged_workspace_size(int(B), int(Nq), int(Hq), int(Hkv),
                                                          int(d), int(page_size),
                                                          int(max_pages_per_seq),
                                                          int(num_splits)))


def _cache_strides(t: torch.Tensor):
    if t.dim() != 4:
        raise ValueError("expected a [num_pages, page_size, kv_heads, head_dim] cache, got shape "
                         "%s" % (tuple(t.shape),))
    if t.stride(3) != 1 and t.shape[3] > 1:
        raise ValueError("head_dim must be contiguous (stride 1)")
    return (ctypes.c_int64 * 3)(t.stride(0), t.stride(1), t.stride(2))


def fa_fwd_paged(q, k_cache, v_cache, block_table, cache_seqlens, softmax_scale=None,
                 causal=False, window_size=(-1, -1), num_splits=0, out=None, lse=None,
                 workspace=None):
    """Decode: q [B, Nq, Hq, d] against a paged KV cache.

    k_cache / v_cache are [num_pages, page_size, Hkv, d]; block_table is int32
    [B, max_pages_per_seq] (row stride free, entries contiguous) and
    cache_seqlens int32 [B], both on the device.  The queries are the last Nq
    positions of each sequence.  Returns (o [B, Nq, Hq, d], lse [B, Hq, Nq])."""
    lib = load_library()
    dev = _check_cuda(q, k_cache, v_cache, block_table, cache_seqlens)
    code = _dtype_code(q)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q and the caches must share one dtype")
    if tuple(k_cache.shape) != tuple(v_cache.shape):
        raise ValueError("k_cache and v_cache must have one shape")
    B, Nq, Hq, d = q.shape
    num_pages, page_size, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B \
            or block_table.stride(1) != 1:
        raise ValueError("block_table must be an int32 [B, max_pages] tensor with contiguous rows")
    if cache_seqlens.dtype != torch.int32 or tuple(cache_seqlens.shape) != (B,) \
            or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 [B] tensor")
    max_pages = block_table.shape[1]
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=q.dtype, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Nq] tensor")
    need = fa_fwd_paged_workspace_size(B, Nq, Hq, Hkv, d, page_size, max_pages, num_splits)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    wl, wr = window_size
    with torch.cuda.device(dev):
        rc = lib.fa_fwd_paged(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                              block_table.data_ptr(), cache_seqlens.data_ptr(), out.data_ptr(),
                              lse.data_ptr(), B, Nq, Hq, Hkv, d, page_size, num_pages, max_pages,
                              block_table.stride(0), _strides(q), _cache_strides(k_cache),
                              _cache_strides(v_cache), _strides(out), code,
                              _scale(softmax_scale, d), int(bool(causal)), int(wl), int(wr),
                              int(num_splits), ws_ptr, ws_bytes, _stream(dev))
    if rc:
        raise FAError(rc, "fa_fwd_paged")
    return out, lse


def fa_fwd_fp8(q, k, v, softmax_scale=None, causal=False, window_size=(-1, -1), descale_q=1.0,
               descale_k=1.0, descale_v=1.0, out=None, lse=None):
    """Forward on float8_e4m3fn q, k, v [B, N, H, d]; returns (o bf16 [B,Nq,Hq,d],
    lse fp32 [B,Hq,Nq]) for attention of (descale_q q, descale_k k, descale_v v)."""
    lib = load_library()
    dev = _check_cuda(q, k, v)
    for t in (q, k, v):
        if t.dtype != torch.float8_e4m3fn:
            raise TypeError("q, k, v must be float8_e4m3fn (got %s)" % t.dtype)
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=dev)
    if out.dtype != torch.bfloat16:
        raise TypeError("the FP8 forward writes a bf16 output")
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be a contiguous fp32 [B, Hq, Nq] tensor")
    wl, wr = window_size
    with torch.cuda.device(dev):
        rc = lib.fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), B, Nq, Nk, Hq, Hkv, d, _strides(q), _strides(k),
                            _strides(v), _strides(out), float(descale_q), float(descale_k),
                            float(descale_v), _scale(softmax_scale, d), int(bool(causal)),
                            int(wl), int(wr), _stream(dev))
    if rc:
        raise FAError(rc, "fa_fwd_fp8")
    return out, lse
