"""Parity at the full sizes of the named long-context workloads, in the
launch configuration the bench times (one handle, one fa_fwd over the whole
workload): sampled rows (tile edges, sequence ends and random rows of a few
heads) against the fp64 oracle computed row by row, plus properties that
hold for every row."""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from oracle import Problem
from masked_attention_fa_b200.workloads import alibi_slopes, make_inputs, named_workloads
from gpu_helpers import TOL_LSE, TOL_MAX_O, TOL_MEAN_O

pytestmark = pytest.mark.gpu


def _arrays(w):
    a = {}
    if w.prefix is not None:
        a["prefix"] = w.prefix
    if w.layout == "TND":
        a["actual_seq_qlen"] = w.actual_seq_qlen
        a["actual_seq_kvlen"] = w.actual_seq_kvlen
    return a


def _rows_of(sq, rng):
    base = [0, 1, 127, 128, 129, 255, 256, sq - 129, sq - 128, sq - 1]
    rnd = rng.integers(0, sq, size=12).tolist()
    return sorted({r for r in base + rnd if 0 <= r < sq})


def _bias(w, slopes, h):
    """The oracle's ALiBi arguments for head h of workload w (one head per
    oracle problem)."""
    return {} if w.alibi is None else {"alibi": w.alibi, "slopes": slopes[h:h + 1]}


@pytest.mark.parametrize("name", ["leftup_causal_4k", "rightdown_band_2k_8k",
                                  "varlen_rightdown_16seq", "prefix_8k", "alibi_causal_4k"])
def test_named_workload_sampled_rows(name):
    w = named_workloads()[name]
    inp = make_inputs(w)
    attn = fa.MaskedAttention(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode,
                              w.pre_tokens, w.next_tokens, w.scale, w.mask_kind, w.alibi)
    slopes = alibi_slopes(w.N) if w.alibi else None
    o, lse = attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), **_arrays(w),
                  slopes=None if slopes is None else torch.tensor(slopes, device="cuda"))
    torch.cuda.synchronize()
    attn.sync_status()
    attn.close()
    of = o.float()
    assert torch.isfinite(of).all()
    o = of.cpu().numpy()
    lse = lse.cpu().numpy()
    rng = np.random.default_rng(5)
    heads = sorted({0, w.N - 1, int(rng.integers(0, w.N))})
    seqs = range(w.B) if w.layout != "TND" else sorted({0, w.B - 1, int(rng.integers(0, w.B))})
    seq_lens = w.seq_lens()
    q0s = np.concatenate([[0], np.cumsum([s for s, _ in seq_lens])]) if w.layout == "TND" else None
    errs, lerrs = [], []
    for h in heads:
        if w.layout == "TND":
            qh, kh, vh = (inp[x][:, h:h + 1] for x in ("q", "k", "v"))
            pb = Problem("TND", w.B, 1, w.Sq, w.Skv, w.D, sparse_mode=w.sparse_mode,
                         pre_tokens=w.pre_tokens, next_tokens=w.next_tokens, scale=w.scale,
                         actual_seq_qlen=w.actual_seq_qlen, actual_seq_kvlen=w.actual_seq_kvlen)
        for b in seqs:
            sq = seq_lens[b][0]
            rows = _rows_of(sq, rng)
            if w.layout == "TND":
                o_ref, l_ref = oracle.attention_rows(pb, qh, kh, vh, [(b, 0, i) for i in rows],
                                                     **_bias(w, slopes, h))
                got = o[[q0s[b] + i for i in rows], h]
                gl = lse[h, [q0s[b] + i for i in rows]]
            else:
                sl = (slice(b, b + 1), slice(h, h + 1)) if w.layout == "BNSD" else \
                     (slice(b, b + 1), slice(None), slice(h, h + 1))
                qs, ks, vs = (inp[x][sl] for x in ("q", "k", "v"))
                pb1 = Problem(w.layout, 1, 1, w.Sq, w.Skv, w.D, sparse_mode=w.sparse_mode,
                              pre_tokens=w.pre_tokens, next_tokens=w.next_tokens,
                              scale=w.scale,
                              prefix=None if w.prefix is None else [w.prefix[b]])
                o_ref, l_ref = oracle.attention_rows(pb1, qs, ks, vs, [(0, 0, i) for i in rows],
                                                     **_bias(w, slopes, h))
                got = o[b, h, rows] if w.layout == "BNSD" else o[b, rows, h]
                gl = lse[b, h, rows]
            errs.append(np.abs(got - o_ref))
            live = np.isfinite(l_ref)
            assert np.array_equal(np.isfinite(gl), live)
            lerrs.append(np.abs(gl[live] - l_ref[live]))
    e = np.concatenate([x.ravel() for x in errs])
    le = np.concatenate(lerrs)
    assert e.max() <= TOL_MAX_O and e.mean() <= TOL_MEAN_O, (name, e.max(), e.mean())
    assert le.max() <= TOL_LSE, (name, le.max())


def test_one_sequence_of_a_million_tokens():
    """BSND, one sequence of 2^20 query rows and keys, causal (mode 2), D=64:
    every index that could overflow 32 bits at this length (token offsets
    times strides, tile and item counts) is exercised. Sampled rows, the
    last one seeing all 2^20 keys, against the fp64 oracle."""
    S, D = 1 << 20, 64
    g = torch.Generator(device="cuda").manual_seed(77)
    q = torch.randn(1, S, 1, D, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(1, S, 1, D, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(1, S, 1, D, generator=g, device="cuda").to(torch.bfloat16)
    attn = fa.MaskedAttention("BSND", 1, 1, S, S, D, 2)
    o, lse = attn(q, k, v)
    torch.cuda.synchronize()
    attn.sync_status()
    attn.close()
    assert torch.isfinite(o.float()).all()
    rows = [0, 1, 255, 256, 65535, 65536, S // 2 + 3, S - 129, S - 1]
    pb = Problem("BSND", 1, 1, S, S, D, sparse_mode=2)
    o_ref, l_ref = oracle.attention_rows(pb, q.cpu(), k.cpu(), v.cpu(), [(0, 0, i) for i in rows])
    got = o[0, rows, 0].float().cpu().double().numpy()
    gl = lse[0, 0, rows].cpu().double().numpy()
    assert np.abs(got - o_ref).max() <= TOL_MAX_O
    assert np.abs(gl - l_ref).max() <= TOL_LSE


def test_thousands_of_tiny_varlen_sequences():
    """TND with 3000 sequences of 0-9 query rows and 0-12 keys (rightDownCausal:
    many rows see no key, many sequences have none), compared in full."""
    rng = np.random.default_rng(78)
    lq = rng.integers(0, 10, size=3000)
    lk = rng.integers(0, 13, size=3000)
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    N, D = 2, 128
    g = torch.Generator().manual_seed(78)
    q = torch.randn(cu_q[-1], N, D, generator=g).to(torch.bfloat16)
    k = torch.randn(cu_k[-1], N, D, generator=g).to(torch.bfloat16)
    v = torch.randn(cu_k[-1], N, D, generator=g).to(torch.bfloat16)
    attn = fa.MaskedAttention("TND", 3000, N, cu_q[-1], cu_k[-1], D, 3)
    o, lse = attn(q.cuda(), k.cuda(), v.cuda(), actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
    torch.cuda.synchronize()
    attn.sync_status()
    attn.close()
    pb = Problem("TND", 3000, N, cu_q[-1], cu_k[-1], D, sparse_mode=3, actual_seq_qlen=cu_q,
                 actual_seq_kvlen=cu_k)
    o_ref, l_ref = oracle.attention(pb, q, k, v)
    o = o.float().cpu().double().numpy()
    lse = lse.cpu().double().numpy()
    dead = np.isneginf(l_ref)
    assert np.array_equal(np.isneginf(lse), dead)
    assert np.abs(o - o_ref).max() <= TOL_MAX_O
    assert np.abs(o - o_ref).mean() <= TOL_MEAN_O
    assert np.abs(lse[~dead] - l_ref[~dead]).max() <= TOL_LSE
