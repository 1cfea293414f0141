"""Seeded synthetic workloads (shapes, arguments and random inputs).

This module only draws inputs and states shapes and call arguments; it holds
none of the attention arithmetic, so both the CUDA path and the fp64 oracle
can take their inputs from it without sharing any of the method.

Input recipe (every workload): a CPU ``torch.Generator`` seeded with the
workload's seed draws, in this order, the varlen lengths (TND workloads
only), then q, k and v as float32 N(0, 1) which are rounded to bfloat16.
The scale is 1/sqrt(D). Paged workloads draw the lengths and the block
order on the CPU generator and q and the caches on the device the inputs
are made for (see ``paged_inputs``).

The named workloads follow the shapes of the Ascend "sparseMode参数说明"
page's scenarios (band, leftUpCausal, right-down band, varlen
rightDownCausal, prefix, and the causal case given as an explicit allMask)
at sizes of long-context inference.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

LAYOUTS = ("BNSD", "BSND", "TND")


@dataclasses.dataclass
class Workload:
    name: str
    layout: str
    B: int
    N: int
    Sq: int
    Skv: int
    D: int
    sparse_mode: int
    pre_tokens: int = 0
    next_tokens: int = 0
    seed: int = 0
    mask_kind: Optional[str] = None      # "SS", "B1SS", "BNSS" or None
    prefix: Optional[list] = None        # modes 5/6, one entry per batch
    actual_seq_qlen: Optional[list] = None   # TND cumulative ends (no leading 0)
    actual_seq_kvlen: Optional[list] = None
    scale: Optional[float] = None
    block_size: Optional[int] = None     # paged K/V caches of this block size (TND queries)
    alibi: Optional[str] = None          # ALiBi variant ("right", "sqrt", "left") or None

    def __post_init__(self):
        if self.scale is None:
            self.scale = 1.0 / math.sqrt(self.D)

    def q_shape(self):
        if self.layout == "BNSD":
            return (self.B, self.N, self.Sq, self.D)
        if self.layout == "BSND":
            return (self.B, self.Sq, self.N, self.D)
        return (self.Sq, self.N, self.D)

    def kv_shape(self):
        if self.layout == "BNSD":
            return (self.B, self.N, self.Skv, self.D)
        if self.layout == "BSND":
            return (self.B, self.Skv, self.N, self.D)
        return (self.Skv, self.N, self.D)

    def lse_shape(self):
        if self.layout == "TND":
            return (self.N, self.Sq)
        return (self.B, self.N, self.Sq)

    def mask_shape(self):
        if self.mask_kind == "SS":
            return (self.Sq, self.Skv)
        if self.mask_kind == "B1SS":
            return (self.B, 1, self.Sq, self.Skv)
        if self.mask_kind == "BNSS":
            return (self.B, self.N, self.Sq, self.Skv)
        return None

    def seq_lens(self):
        """[(Sq_b, Skv_b)] per sequence."""
        if self.layout != "TND":
            return [(self.Sq, self.Skv)] * self.B
        out, pq, pk = [], 0, 0
        for cq, ck in zip(self.actual_seq_qlen, self.actual_seq_kvlen):
            out.append((cq - pq, ck - pk))
            pq, pk = cq, ck
        return out


def varlen_lengths(gen: torch.Generator, nseq: int, q_lo: int, q_hi: int, extra_hi: int):
    """Draw varlen lengths: Sq_b uniform in [q_lo, q_hi], Skv_b = Sq_b + uniform[0, extra_hi].

    Returns the cumulative end-offset arrays (no leading 0).
    """
    sq = torch.randint(q_lo, q_hi + 1, (nseq,), generator=gen)
    extra = torch.randint(0, extra_hi + 1, (nseq,), generator=gen)
    skv = sq + extra
    return torch.cumsum(sq, 0).tolist(), torch.cumsum(skv, 0).tolist()


def alibi_slopes(N: int):
    """Per-head ALiBi coefficients for N heads, the geometric sequence
    2^(-8 (h + 1) / N), h = 0..N-1, as synthetic inputs (the compressed-mask
    page passes slopes in but does not say how they are chosen)."""
    return [2.0 ** (-8.0 * (h + 1) / N) for h in range(N)]


def lower_triangular_mask(S: int) -> torch.Tensor:
    """The S x S lower-triangular attenMask the band page asks for in the causal
    case (1 = masked, i.e. the strictly upper triangle)."""
    return torch.triu(torch.ones(S, S, dtype=torch.uint8), diagonal=1)


# Patterns of block_mask, one per 128 x 128 block (1 = masked).
BLOCK_PATTERNS = ("hidden", "visible", "random", "one_visible", "one_hidden", "lower")


def block_mask(shape, seed: int, block: int = 128, weights=None) -> torch.Tensor:
    """A uint8 mask of `shape` (..., Sq, Skv) made of blocks of `block` rows x
    `block` keys, each drawn from BLOCK_PATTERNS with the given weights (by
    default: hidden 0.35, visible 0.3, random 0.15, one visible / one hidden
    pair 0.05 each, lower triangle 0.1): whole hidden and whole visible blocks
    as in the page's causal and band masks, and mixed ones. Leading dims are
    independent planes."""
    g = torch.Generator("cpu").manual_seed(seed)
    w = torch.tensor(weights or [0.35, 0.3, 0.15, 0.05, 0.05, 0.1], dtype=torch.float64)
    *lead, Sq, Skv = shape
    nq, nk = (Sq + block - 1) // block, (Skv + block - 1) // block
    planes = 1
    for d in lead:
        planes *= d
    out = torch.ones((planes, nq * block, nk * block), dtype=torch.uint8)
    pat = torch.multinomial(w, planes * nq * nk, replacement=True, generator=g)
    rnd = (torch.rand((planes, nq * block, nk * block), generator=g) < 0.3).to(torch.uint8)
    pos = torch.randint(0, block * block, (planes * nq * nk,), generator=g)
    tri = torch.triu(torch.ones(block, block, dtype=torch.uint8), diagonal=1)
    n = 0
    for p in range(planes):
        for a in range(nq):
            for b in range(nk):
                blk = out[p, a * block:(a + 1) * block, b * block:(b + 1) * block]
                kind = BLOCK_PATTERNS[int(pat[n])]
                r, c = divmod(int(pos[n]), block)
                if kind == "visible":
                    blk.zero_()
                elif kind == "random":
                    blk.copy_(rnd[p, a * block:(a + 1) * block, b * block:(b + 1) * block])
                elif kind == "one_visible":
                    blk[r, c] = 0
                elif kind == "one_hidden":
                    blk.zero_()
                    blk[r, c] = 1
                elif kind == "lower":
                    blk.copy_(tri)
                n += 1
    return out[:, :Sq, :Skv].reshape(*lead, Sq, Skv).contiguous()


def decode_lengths(gen: torch.Generator, nseq: int, kv_lo: int, kv_hi: int):
    """One query token per sequence and Skv_b uniform in [kv_lo, kv_hi]:
    cumulative end offsets (no leading 0)."""
    skv = torch.randint(kv_lo, kv_hi + 1, (nseq,), generator=gen)
    return list(range(1, nseq + 1)), torch.cumsum(skv, 0).tolist()


def paged_inputs(w: "Workload", gen: torch.Generator, device="cpu"):
    """q [T_q, N, D] and paged caches [num_blocks, block_size, N, D] for a
    TND workload: each sequence's keys fill ceil(Skv_b / block_size) blocks
    taken in a random order (randperm of the CPU generator `gen`), the rest
    of a last block is zero; block_table [B, max_blocks] int32 (-1 past a
    sequence's blocks). q and the cache values (N(0, 1), bf16) are drawn on
    `device` by a generator of that device seeded with the workload's seed,
    so a GPU run does not wait for the host to draw gigabytes."""
    bs = w.block_size
    lens = w.seq_lens()
    nblk = [-(-skv // bs) for _, skv in lens]
    total = sum(nblk)
    order = torch.randperm(total, generator=gen).to(torch.int32)
    table = torch.full((len(lens), max(max(nblk), 1)), -1, dtype=torch.int32)
    nxt = 0
    for b in range(len(lens)):
        table[b, :nblk[b]] = order[nxt:nxt + nblk[b]]
        nxt += nblk[b]
    dg = torch.Generator(device=device).manual_seed(w.seed)
    q = torch.randn(w.q_shape(), generator=dg, device=device, dtype=torch.float32).to(torch.bfloat16)
    k_cache = torch.randn((total, bs, w.N, w.D), generator=dg, device=device, dtype=torch.bfloat16)
    v_cache = torch.randn((total, bs, w.N, w.D), generator=dg, device=device, dtype=torch.bfloat16)
    for b, (_, skv) in enumerate(lens):
        tail = skv - (nblk[b] - 1) * bs
        if nblk[b] and tail < bs:  # slots past the sequence's last key
            last = int(table[b, nblk[b] - 1])
            k_cache[last, tail:] = 0
            v_cache[last, tail:] = 0
    return q, k_cache, v_cache, table.to(device)


def named_workloads() -> dict:
    """The long-context scenarios, by name."""
    g4 = torch.Generator("cpu").manual_seed(4)
    cu_q, cu_kv = varlen_lengths(g4, 16, 512, 4096, 1024)
    g6 = torch.Generator("cpu").manual_seed(6)
    dq, dkv = decode_lengths(g6, 16, 4096, 16384)
    return {
        # band from the top-left via preTokens/nextTokens, with the
        # lower-triangular attenMask the page asks for (causal via band)
        "band_causal_256": Workload("band_causal_256", "BNSD", 1, 2, 256, 256, 64, 0,
                                    pre_tokens=256, next_tokens=0, seed=1, mask_kind="SS"),
        "leftup_causal_4k": Workload("leftup_causal_4k", "BNSD", 2, 16, 4096, 4096, 128, 2,
                                     seed=2),
        "rightdown_band_2k_8k": Workload("rightdown_band_2k_8k", "BSND", 1, 32, 2048, 8192, 128,
                                         4, pre_tokens=1024, next_tokens=0, seed=3),
        "varlen_rightdown_16seq": Workload("varlen_rightdown_16seq", "TND", 16, 32, cu_q[-1],
                                           cu_kv[-1], 128, 3, seed=4, actual_seq_qlen=cu_q,
                                           actual_seq_kvlen=cu_kv),
        "prefix_8k": Workload("prefix_8k", "BNSD", 4, 16, 8192, 8192, 128, 5, seed=5,
                              prefix=[512, 1024, 2048, 4096]),
        # leftUpCausal with the right-aligned ALiBi bias of the compressed-mask
        # page (slopes: alibi_slopes(16)); same shape and q, k, v as above
        "alibi_causal_4k": Workload("alibi_causal_4k", "BNSD", 2, 16, 4096, 4096, 128, 2, seed=2,
                                    alibi="right"),
        # the leftUpCausal problem (same shape and seed, so the same q, k, v)
        # given as an explicit lower-triangular allMask (sparseMode 1)
        "allmask_causal_4k": Workload("allmask_causal_4k", "BNSD", 2, 16, 4096, 4096, 128, 1,
                                      seed=2, mask_kind="SS"),
        # one long rightDownCausal sequence, the job the sparseMode=7/8
        # sections cut across cards by query rows (bench.py --split)
        "split_rightdown_32k": Workload("split_rightdown_32k", "TND", 1, 32, 32768, 32768, 128,
                                        3, seed=7, actual_seq_qlen=[32768],
                                        actual_seq_kvlen=[32768]),
        # decode: one query token per sequence against a long context held
        # in paged caches (blocks of 128 tokens in random order), mode 3
        "paged_decode_16k": Workload("paged_decode_16k", "TND", 16, 32, dq[-1], dkv[-1], 128, 3,
                                     seed=6, actual_seq_qlen=dq, actual_seq_kvlen=dkv,
                                     block_size=128),
    }


def make_inputs(w: Workload, device="cpu"):
    """Draw q, k, v (bf16) and the mask for workload w with its seed.

    Returns a dict with q, k, v (on `device`) and mask (uint8 on `device`, or
    None). TND lengths are part of the workload itself.
    """
    g = torch.Generator("cpu").manual_seed(w.seed)
    if w.layout == "TND" and w.name == "varlen_rightdown_16seq":
        # the lengths were drawn first from the same seed; redraw to advance
        varlen_lengths(g, 16, 512, 4096, 1024)
    if w.block_size is not None:
        decode_lengths(g, w.B, 4096, 16384)  # drawn first from the same seed
        q, k_cache, v_cache, table = paged_inputs(w, g, device)
        return {"q": q, "k_cache": k_cache, "v_cache": v_cache, "block_table": table,
                "mask": None}
    q = torch.randn(w.q_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(w.kv_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(w.kv_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    mask = None
    if w.mask_kind is not None:
        if w.name in ("band_causal_256", "allmask_causal_4k"):
            mask = lower_triangular_mask(w.Sq)
        else:
            mask = (torch.rand(w.mask_shape(), generator=g) < 0.3).to(torch.uint8)
    out = {"q": q.to(device), "k": k.to(device), "v": v.to(device),
           "mask": None if mask is None else mask.to(device)}
    return out


def random_inputs(layout, B, N, Sq, Skv, D, seed, mask_kind=None, mask_density=0.3,
                  device="cpu"):
    """q, k, v (bf16 N(0,1)) and an optional Bernoulli(mask_density) mask."""
    w = Workload("random", layout, B, N, Sq, Skv, D, 0, seed=seed, mask_kind=mask_kind)
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(w.q_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(w.kv_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(w.kv_shape(), generator=g, dtype=torch.float32).to(torch.bfloat16)
    mask = None
    if mask_kind is not None:
        mask = (torch.rand(w.mask_shape(), generator=g) < mask_density).to(torch.uint8)
    return {"q": q.to(device), "k": k.to(device), "v": v.to(device),
            "mask": None if mask is None else mask.to(device)}
