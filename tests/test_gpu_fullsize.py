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
from masked_attention_fa_b200.workloads import make_inputs, named_workloads
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


@pytest.mark.parametrize("name", ["leftup_causal_4k", "rightdown_band_2k_8k",
                                  "varlen_rightdown_16seq", "prefix_8k"])
def test_named_workload_sampled_rows(name):
    w = named_workloads()[name]
    inp = make_inputs(w)
    attn = fa.MaskedAttention(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode,
                              w.pre_tokens, w.next_tokens, w.scale, w.mask_kind)
    o, lse = attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), **_arrays(w))
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
                o_ref, l_ref = oracle.attention_rows(pb, qh, kh, vh, [(b, 0, i) for i in rows])
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
                o_ref, l_ref = oracle.attention_rows(pb1, qs, ks, vs, [(0, 0, i) for i in rows])
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
