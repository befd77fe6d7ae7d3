"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds the workload shapes and the random draws only -- none of
the attention arithmetic -- so that the CUDA path and the fp64 oracle are fed
bit-identical fp16/bf16 values without sharing any code.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws
``torch.randn`` in fp32, in the order Q, K, V, then dO, each in the
``[batch, seq, heads, head_dim]`` layout of ``flash_attn_func``
("optimizing-attention-flash", Workflow 2, Step 2); the fp32 draws are then
rounded once to the workload dtype.  Values are i.i.d. N(0, 1), as in the
pages' own benchmark and accuracy snippets (``torch.randn``, Workflow 1
Steps 3-4).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen_q: int
    seqlen_k: int
    q_heads: int
    kv_heads: int
    head_dim: int
    dtype: torch.dtype
    causal: bool
    window: tuple = (-1, -1)
    seed: int = 0
    backward: bool = False
    note: str = field(default="", compare=False)

    @property
    def softmax_scale(self) -> float:
        # the pages' default: 1 / sqrt(head_dim)
        return float(self.head_dim) ** -0.5

    def describe(self) -> dict:
        return {
            "workload": self.name, "batch": self.batch, "seqlen_q": self.seqlen_q,
            "seqlen_k": self.seqlen_k, "q_heads": self.q_heads, "kv_heads": self.kv_heads,
            "head_dim": self.head_dim, "dtype": str(self.dtype).replace("torch.", ""),
            "causal": self.causal, "window_size": list(self.window), "seed": self.seed,
            "backward": self.backward,
        }


F16, BF16 = torch.float16, torch.bfloat16

# The five workloads of the pages' benchmark plan; shapes of 2 and 3 restate the
# pages' own benchmark snippets ("optimizing-attention-flash", Workflow 1 Step 3
# at 2x8x2048x64 and Workflow 2 Step 4 at 4x32x4096x64).
WORKLOADS = {
    "tiny_128_d64_fp16": Workload("tiny_128_d64_fp16", 1, 128, 128, 2, 2, 64, F16, False, seed=0),
    "fwd_2x2048_h8_d64_fp16": Workload("fwd_2x2048_h8_d64_fp16", 2, 2048, 2048, 8, 8, 64, F16,
                                       False, seed=1),
    "fwd_2x2048_h8_d64_fp16_causal": Workload("fwd_2x2048_h8_d64_fp16_causal", 2, 2048, 2048, 8,
                                              8, 64, F16, True, seed=1),
    "fwd_4x4096_h32_d64_fp16_causal": Workload("fwd_4x4096_h32_d64_fp16_causal", 4, 4096, 4096,
                                               32, 32, 64, F16, True, seed=2),
    "fwd_2x4096_h32kv8_d128_bf16_causal_win256": Workload(
        "fwd_2x4096_h32kv8_d128_bf16_causal_win256", 2, 4096, 4096, 32, 8, 128, BF16, True,
        window=(256, 0), seed=3),
    "fwdbwd_1x16384_h16_d128_bf16_causal": Workload("fwdbwd_1x16384_h16_d128_bf16_causal", 1,
                                                    16384, 16384, 16, 16, 128, BF16, True,
                                                    seed=4, backward=True),
    # head_dim 256, the largest the pages list, on a causal 2 x 4096 batch
    "fwd_2x4096_h16_d256_bf16_causal": Workload("fwd_2x4096_h16_d256_bf16_causal", 2, 4096, 4096,
                                                16, 16, 256, BF16, True, seed=9),
}


def make_qkv(batch, seqlen_q, seqlen_k, q_heads, kv_heads, head_dim, dtype, seed,
             with_dout=False):
    """Q, K, V (and dO) as CPU tensors of ``dtype``, drawn in the order Q, K, V, dO."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((batch, seqlen_q, q_heads, head_dim), generator=g, dtype=torch.float32)
    k = torch.randn((batch, seqlen_k, kv_heads, head_dim), generator=g, dtype=torch.float32)
    v = torch.randn((batch, seqlen_k, kv_heads, head_dim), generator=g, dtype=torch.float32)
    out = [q.to(dtype), k.to(dtype), v.to(dtype)]
    if with_dout:
        do = torch.randn((batch, seqlen_q, q_heads, head_dim), generator=g, dtype=torch.float32)
        out.append(do.to(dtype))
    return tuple(out)


def make_workload_inputs(w: Workload, with_dout=None):
    if with_dout is None:
        with_dout = w.backward
    return make_qkv(w.batch, w.seqlen_q, w.seqlen_k, w.q_heads, w.kv_heads, w.head_dim, w.dtype,
                    w.seed, with_dout=with_dout)


@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of independent sequences of mixed length (no padding)."""
    name: str
    n_seqs: int
    min_len: int
    max_len: int
    q_heads: int
    kv_heads: int
    head_dim: int
    dtype: torch.dtype
    causal: bool
    seed: int

    @property
    def softmax_scale(self) -> float:
        return float(self.head_dim) ** -0.5

    def lengths(self):
        g = torch.Generator(device="cpu")
        g.manual_seed(int(self.seed))
        return [int(x) for x in torch.randint(self.min_len, self.max_len + 1, (self.n_seqs,),
                                              generator=g)]

    def describe(self) -> dict:
        return {"workload": self.name, "sequences": self.n_seqs,
                "lengths": "uniform in [%d, %d]" % (self.min_len, self.max_len),
                "q_heads": self.q_heads, "kv_heads": self.kv_heads, "head_dim": self.head_dim,
                "dtype": str(self.dtype).replace("torch.", ""), "causal": self.causal,
                "seed": self.seed}


VARLEN_WORKLOADS = {
    "varlen_8seq_512to4096_h16_d128_bf16_causal": VarlenWorkload(
        "varlen_8seq_512to4096_h16_d128_bf16_causal", 8, 512, 4096, 16, 16, 128, BF16, True,
        seed=5),
}


def make_varlen_inputs(w: VarlenWorkload):
    """Packed Q [total, Hq, d], K, V [total, Hkv, d], dO and int32 offsets [B+1]
    (CPU tensors); drawn in the order Q, K, V, dO after the lengths."""
    lens = w.lengths()
    total = sum(lens)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) + 1)
    q = torch.randn((total, w.q_heads, w.head_dim), generator=g).to(w.dtype)
    k = torch.randn((total, w.kv_heads, w.head_dim), generator=g).to(w.dtype)
    v = torch.randn((total, w.kv_heads, w.head_dim), generator=g).to(w.dtype)
    do = torch.randn((total, w.q_heads, w.head_dim), generator=g).to(w.dtype)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    return q, k, v, do, cu, lens


def sample_rows(batch, q_heads, seqlen_q, n, seed):
    """n distinct (b, h, i) triples, always including the first and last row of
    the sequence so the ragged tail and the causal corner are covered."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 7919)
    b = torch.randint(0, batch, (n,), generator=g)
    h = torch.randint(0, q_heads, (n,), generator=g)
    i = torch.randint(0, seqlen_q, (n,), generator=g)
    i[0] = 0
    if n > 1:
        i[1] = seqlen_q - 1
    rows = torch.stack([b, h, i], dim=1)
    return torch.unique(rows, dim=0).numpy()


@dataclass(frozen=True)
class PagedWorkload:
    """Decode: Nq new queries per sequence against a paged KV cache."""
    name: str
    n_seqs: int
    min_len: int
    max_len: int
    Nq: int
    q_heads: int
    kv_heads: int
    head_dim: int
    dtype: torch.dtype
    page_size: int
    causal: bool
    seed: int

    @property
    def softmax_scale(self) -> float:
        return float(self.head_dim) ** -0.5

    def lengths(self):
        g = torch.Generator(device="cpu")
        g.manual_seed(int(self.seed))
        return [int(x) for x in torch.randint(self.min_len, self.max_len + 1, (self.n_seqs,),
                                              generator=g)]

    def describe(self) -> dict:
        return {"workload": self.name, "sequences": self.n_seqs,
                "cache_lengths": "uniform in [%d, %d]" % (self.min_len, self.max_len),
                "new_queries": self.Nq, "q_heads": self.q_heads, "kv_heads": self.kv_heads,
                "head_dim": self.head_dim, "dtype": str(self.dtype).replace("torch.", ""),
                "page_size": self.page_size, "causal": self.causal, "seed": self.seed}


# Decode shape: 128 running sequences and 16-token pages, as in the vLLM launch
# example of the FlashAttention V3 page (section 四: max_num_seqs=128,
# block_size=16); 32 query heads over 8 kv heads of dimension 128 (the
# geometry of the Llama-3-8B model that example serves).
PAGED_WORKLOADS = {
    "decode_128seq_512to8192_h32kv8_d128_bf16_page16": PagedWorkload(
        "decode_128seq_512to8192_h32kv8_d128_bf16_page16", 128, 512, 8192, 1, 32, 8, 128, BF16,
        16, True, seed=6),
}


def make_paged_inputs(B, Nq, Hq, Hkv, d, dtype, page_size, lens, seed, spare_pages=3,
                      fill=float("nan")):
    """q [B, Nq, Hq, d] and a paged cache holding len_b keys per sequence.

    Returns q, k_cache, v_cache ([num_pages, page_size, Hkv, d]), block_table
    (int32 [B, max_pages]) and cache_seqlens (int32 [B]), all on the CPU.
    Pages are handed out in a seeded random order; cache rows a sequence does
    not own (past its length, and `spare_pages` unused pages) hold `fill`.
    Draw order: q, then per sequence its K rows and V rows."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    n_pages_of = [(n + page_size - 1) // page_size for n in lens]
    max_pages = max(1, max(n_pages_of))
    num_pages = sum(n_pages_of) + spare_pages
    q = torch.randn((B, Nq, Hq, d), generator=g, dtype=torch.float32).to(dtype)
    perm = torch.randperm(max(num_pages, 1), generator=g)
    k_cache = torch.full((max(num_pages, 1), page_size, Hkv, d), fill, dtype=dtype)
    v_cache = torch.full((max(num_pages, 1), page_size, Hkv, d), fill, dtype=dtype)
    block_table = torch.zeros((B, max_pages), dtype=torch.int32)
    k_rows = k_cache.view(-1, Hkv, d)  # row p * page_size + t of page p
    v_rows = v_cache.view(-1, Hkv, d)
    first = 0
    for b, n in enumerate(lens):
        pages = perm[first:first + n_pages_of[b]]
        first += n_pages_of[b]
        block_table[b, :len(pages)] = pages.to(torch.int32)
        kk = torch.randn((n, Hkv, d), generator=g, dtype=torch.float32).to(dtype)
        vv = torch.randn((n, Hkv, d), generator=g, dtype=torch.float32).to(dtype)
        j = torch.arange(n)
        rows = pages[j // page_size] * page_size + j % page_size
        k_rows[rows] = kk
        v_rows[rows] = vv
    cache_seqlens = torch.tensor(lens, dtype=torch.int32)
    return q, k_cache, v_cache, block_table, cache_seqlens


@dataclass(frozen=True)
class Fp8Workload:
    """Forward on float8_e4m3fn inputs (optionally quantised with per-tensor
    factors: the stored value is x / descale)."""
    name: str
    batch: int
    seqlen: int
    q_heads: int
    kv_heads: int
    head_dim: int
    causal: bool
    descales: tuple
    seed: int

    @property
    def softmax_scale(self) -> float:
        return float(self.head_dim) ** -0.5

    def describe(self) -> dict:
        return {"workload": self.name, "batch": self.batch, "seqlen_q": self.seqlen,
                "seqlen_k": self.seqlen, "q_heads": self.q_heads, "kv_heads": self.kv_heads,
                "head_dim": self.head_dim, "dtype": "float8_e4m3fn in, bfloat16 out",
                "causal": self.causal, "descales": list(self.descales), "seed": self.seed}


# The pages' FP8 example shape ("optimizing-attention-flash", Workflow 3,
# Step 3: 2 x 4096 tokens, 32 heads of 64, cast straight to float8_e4m3fn),
# and the 16384-token causal d = 128 shape of the 16-bit benchmark.
FP8_WORKLOADS = {
    "fwd_fp8_2x4096_h32_d64_e4m3": Fp8Workload("fwd_fp8_2x4096_h32_d64_e4m3", 2, 4096, 32, 32, 64,
                                               False, (1.0, 1.0, 1.0), seed=7),
    "fwd_fp8_1x16384_h16_d128_e4m3_causal": Fp8Workload(
        "fwd_fp8_1x16384_h16_d128_e4m3_causal", 1, 16384, 16, 16, 128, True, (1.0, 1.0, 1.0),
        seed=8),
}


def make_fp8_inputs(B, Nq, Nk, Hq, Hkv, d, descales, seed):
    """float8_e4m3fn q [B,Nq,Hq,d], k, v [B,Nk,Hkv,d] on the CPU: seeded N(0,1)
    fp32 draws in the order Q, K, V, each divided by its descale factor and
    cast (round to nearest, as torch's cast does)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Nq, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Nk, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Nk, Hkv, d), generator=g, dtype=torch.float32)
    return tuple((x / float(s)).to(torch.float8_e4m3fn) for x, s in zip((q, k, v), descales))
