"""Pins of the fp64 oracle to things other than itself.

Each test ties one part of the oracle to a library routine, a closed form,
an equivalence stated on the Ascend "sparseMode参数说明" page, one of that
page's worked split examples, or the "FlashAttention tiling & online
softmax" exercise page. A plausible slip in the oracle (a wrong anchor
corner, an exclusive band bound, a transposed operand, a dropped scale, a
wrong lse) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import Problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "split_examples.json")


def _rand(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


def _sdpa(q, k, v, scale, attn_mask=None, is_causal=False):
    # q, k, v: [B, N, S, D] float64 (torch's reference math kernel on CPU)
    return F.scaled_dot_product_attention(q, k, v, attn_mask=attn_mask, is_causal=is_causal,
                                          scale=scale)


# --------------------------------------------------------------------------
# Library routines: the softmax/PV arithmetic and the lse.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("Sq,Skv,D", [(7, 7, 8), (5, 11, 16), (13, 6, 4)])
def test_mode0_without_mask_is_plain_attention(Sq, Skv, D):
    """sparseMode=0 with no attenMask masks nothing (pre/next ignored)."""
    B, N = 2, 3
    q, k, v = _rand((B, N, Sq, D), 1), _rand((B, N, Skv, D), 2), _rand((B, N, Skv, D), 3)
    pb = Problem("BNSD", B, N, Sq, Skv, D, sparse_mode=0, pre_tokens=1, next_tokens=0)
    o, lse = oracle.attention(pb, q, k, v)
    ref = _sdpa(q, k, v, pb.scale).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    ref_lse = torch.logsumexp(pb.scale * q @ k.transpose(-1, -2), dim=-1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Sq,Skv", [(9, 9), (6, 10), (10, 6)])
def test_mode2_is_torch_causal(Sq, Skv):
    """leftUpCausal = the lower triangle split at the top-left vertex, which
    is what torch's is_causal computes."""
    B, N, D = 1, 2, 8
    q, k, v = _rand((B, N, Sq, D), 4), _rand((B, N, Skv, D), 5), _rand((B, N, Skv, D), 6)
    pb = Problem("BNSD", B, N, Sq, Skv, D, sparse_mode=2)
    o, lse = oracle.attention(pb, q, k, v)
    ref = _sdpa(q, k, v, pb.scale, is_causal=True).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["SS", "B1SS", "BNSS"])
def test_mode1_is_boolean_mask_attention(kind):
    """allMask: a True entry hides that QK^T position (attenMask rule)."""
    B, N, Sq, Skv, D = 2, 3, 9, 12, 8
    q, k, v = _rand((B, N, Sq, D), 7), _rand((B, N, Skv, D), 8), _rand((B, N, Skv, D), 9)
    g = torch.Generator("cpu").manual_seed(10)
    shape = {"SS": (Sq, Skv), "B1SS": (B, 1, Sq, Skv), "BNSS": (B, N, Sq, Skv)}[kind]
    m = (torch.rand(shape, generator=g) < 0.4).to(torch.uint8)
    m[..., 0] = 0  # keep one visible key per row (torch returns NaN otherwise)
    pb = Problem("BNSD", B, N, Sq, Skv, D, sparse_mode=1, mask=m.numpy(), mask_kind=kind)
    o, lse = oracle.attention(pb, q, k, v)
    allowed = (m == 0)
    while allowed.dim() < 4:
        allowed = allowed.unsqueeze(0)
    ref = _sdpa(q, k, v, pb.scale, attn_mask=allowed.expand(B, N, Sq, Skv)).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    s = pb.scale * q @ k.transpose(-1, -2)
    s = s.masked_fill(~allowed.expand(B, N, Sq, Skv), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_bsnd_and_tnd_layouts_match_bnsd():
    """The same problem in BSND, and each TND sequence alone in BNSD."""
    B, N, S, D = 2, 3, 10, 8
    q, k, v = _rand((B, N, S, D), 11), _rand((B, N, S, D), 12), _rand((B, N, S, D), 13)
    pb = Problem("BNSD", B, N, S, S, D, sparse_mode=3)
    o, lse = oracle.attention(pb, q, k, v)
    pt = Problem("BSND", B, N, S, S, D, sparse_mode=3)
    o2, lse2 = oracle.attention(pt, q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2))
    np.testing.assert_array_equal(o2, o.transpose(0, 2, 1, 3))
    np.testing.assert_array_equal(lse2, lse)
    # TND with three sequences, one of them empty
    lq, lk = [4, 0, 7], [6, 3, 9]
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    qt, kt, vt = _rand((sum(lq), N, D), 14), _rand((sum(lk), N, D), 15), _rand((sum(lk), N, D), 16)
    ptnd = Problem("TND", 3, N, sum(lq), sum(lk), D, sparse_mode=3,
                   actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
    ot, lset = oracle.attention(ptnd, qt, kt, vt)
    q0 = k0 = 0
    for b in range(3):
        if lq[b]:
            one = Problem("BNSD", 1, N, lq[b], lk[b], D, sparse_mode=3)
            ob, lb = oracle.attention(one, qt[q0:q0 + lq[b]].permute(1, 0, 2)[None],
                                      kt[k0:k0 + lk[b]].permute(1, 0, 2)[None],
                                      vt[k0:k0 + lk[b]].permute(1, 0, 2)[None])
            np.testing.assert_array_equal(ot[q0:q0 + lq[b]], ob[0].transpose(1, 0, 2))
            np.testing.assert_array_equal(lset[:, q0:q0 + lq[b]], lb[0])
        q0 += lq[b]
        k0 += lk[b]


# --------------------------------------------------------------------------
# Equivalences stated on the sparseMode page, and ones derived from it.
# --------------------------------------------------------------------------

def _masks_equal(pa, pb_, b=0, h=0):
    return np.array_equal(oracle.mask_matrix(pa, b, h), oracle.mask_matrix(pb_, b, h))


@pytest.mark.parametrize("S,pre", [(8, 8), (8, 20), (13, 13)])
def test_mode0_causal_via_band_equals_leftup_causal(S, pre):
    """Stated: nextTokens=0 and preTokens >= Sq with the lower-triangular
    attenMask is the causal case."""
    tri = np.triu(np.ones((S, S), np.uint8), 1)
    a = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=0, pre_tokens=pre, next_tokens=0,
                mask=tri, mask_kind="SS")
    c = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=2)
    assert _masks_equal(a, c)


@pytest.mark.parametrize("S", [1, 5, 16])
def test_rightdown_equals_leftup_when_square(S):
    """Both triangles are split on the same diagonal when Sq = Skv."""
    assert _masks_equal(Problem("BNSD", 1, 1, S, S, 4, sparse_mode=3),
                        Problem("BNSD", 1, 1, S, S, 4, sparse_mode=2))


def test_rightdown_differs_from_leftup_when_not_square():
    a = oracle.mask_matrix(Problem("BNSD", 1, 1, 4, 6, 4, sparse_mode=3), 0)
    b = oracle.mask_matrix(Problem("BNSD", 1, 1, 4, 6, 4, sparse_mode=2), 0)
    assert not np.array_equal(a, b)
    # the last query row sees every key when anchored at the bottom-right
    assert a[-1].all() and a[0].sum() == 3


def test_band_edges_are_inclusive():
    """nextTokens < 0 is allowed with preTokens = |nextTokens|; that band is
    one diagonal under inclusive bounds and empty under exclusive ones."""
    S = 10
    pb = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=0, pre_tokens=3, next_tokens=-3,
                 mask=np.zeros((S, S), np.uint8), mask_kind="SS")
    m = oracle.mask_matrix(pb, 0)
    assert m.sum() == S - 3
    assert all(m[i, i - 3] for i in range(3, S))
    pb2 = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=0, pre_tokens=-3, next_tokens=3,
                  mask=np.zeros((S, S), np.uint8), mask_kind="SS")
    m2 = oracle.mask_matrix(pb2, 0)
    assert m2.sum() == S - 3 and all(m2[i, i + 3] for i in range(S - 3))


@pytest.mark.parametrize("pre,nxt", [(9, -3), (-3, 7), (2, 2), (20, 0), (0, 20)])
def test_band_top_left_equals_band_bottom_right_when_square(pre, nxt):
    """(ours) mode 0 with an all-False mask and mode 4 share their anchor when
    Sq = Skv."""
    S = 12
    a = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=0, pre_tokens=pre, next_tokens=nxt,
                mask=np.zeros((S, S), np.uint8), mask_kind="SS")
    b = Problem("BNSD", 1, 1, S, S, 4, sparse_mode=4, pre_tokens=pre, next_tokens=nxt)
    assert _masks_equal(a, b)


@pytest.mark.parametrize("Sq,Skv", [(5, 9), (8, 8), (3, 12)])
def test_derived_equivalences(Sq, Skv):
    """(ours) mode 4 with pre >= Skv, next = 0 is mode 3; mode 5 with prefix 0
    is mode 3; mode 5 with prefix Skv sees everything; mode 6 is mode 5;
    mode 1 with the complement of mode k's visibility is mode k."""
    m3 = Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=3)
    assert _masks_equal(Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=4, pre_tokens=Skv,
                                next_tokens=0), m3)
    assert _masks_equal(Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=5, prefix=[0]), m3)
    full = oracle.mask_matrix(Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=5, prefix=[Skv]), 0)
    assert full.all()
    assert _masks_equal(Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=5, prefix=[2]),
                        Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=6, prefix=[2]))
    for mode, kw in [(2, {}), (3, {}), (4, dict(pre_tokens=2, next_tokens=1)),
                     (5, dict(prefix=[2]))]:
        p = Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=mode, **kw)
        vis = oracle.mask_matrix(p, 0)
        m1 = Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=1, mask=(1 - vis), mask_kind="SS")
        assert np.array_equal(oracle.mask_matrix(m1, 0), vis)


# --------------------------------------------------------------------------
# The page's worked varlen split examples (sparseMode=7 and sparseMode=8).
# --------------------------------------------------------------------------

def _split_case(example, unsplit_qlen, unsplit_kvlen, card1_q, card1_kv, card2_q_off,
                card2_kv_off):
    with open(GOLDEN) as f:
        g = json.load(f)[example]
    N, D = 2, 8
    Tq, Tk = unsplit_qlen[-1], unsplit_kvlen[-1]
    q, k, v = _rand((Tq, N, D), 21), _rand((Tk, N, D), 22), _rand((Tk, N, D), 23)
    full = Problem("TND", len(unsplit_qlen), N, Tq, Tk, D, sparse_mode=g["unsplit_mode"],
                   actual_seq_qlen=unsplit_qlen, actual_seq_kvlen=unsplit_kvlen)
    o, lse = oracle.attention(full, q, k, v)
    outs = []
    for card, (q0, q1, k0, k1) in (("card1", (0, card1_q, 0, card1_kv)),
                                   ("card2", (card2_q_off, Tq, card2_kv_off, Tk))):
        c = g[card]
        pc = Problem("TND", len(c["actual_seq_qlen"]), N, q1 - q0, k1 - k0, D,
                     sparse_mode=c["sparse_mode"], pre_tokens=c.get("pre_tokens", 0),
                     next_tokens=c.get("next_tokens", 0),
                     actual_seq_qlen=c["actual_seq_qlen"], actual_seq_kvlen=c["actual_seq_kvlen"])
        assert c["actual_seq_qlen"][-1] == q1 - q0 and c["actual_seq_kvlen"][-1] == k1 - k0
        oc, lc = oracle.attention(pc, q[q0:q1], k[k0:k1], v[k0:k1])
        outs.append((oc, lc))
    o_cat = np.concatenate([outs[0][0], outs[1][0]], axis=0)
    lse_cat = np.concatenate([outs[0][1], outs[1][1]], axis=1)
    np.testing.assert_array_equal(o_cat, o)
    np.testing.assert_array_equal(lse_cat, lse)


def test_mode7_worked_split_reproduces_unsplit_rightdown():
    """Unsplit: sequences (3,3), (4,6), (5,5), (4,4) in mode 3. Card 1 holds
    query rows [0,5) with keys [0,9); card 2 holds query rows [5,16) with
    keys [3,18) (the second sequence's keys are on both cards)."""
    _split_case("mode7", [3, 7, 12, 16], [3, 9, 14, 18], 5, 9, 5, 3)


def test_mode8_worked_split_reproduces_unsplit_leftup():
    """Unsplit: sequences (3,3), (5,4), (5,5), (4,4) in mode 2. Card 1 holds
    query rows [0,5) with keys [0,7); card 2 holds query rows [5,17) with
    keys [3,16)."""
    _split_case("mode8", [3, 8, 13, 17], [3, 7, 12, 16], 5, 7, 5, 3)


@pytest.mark.parametrize("Sq,Skv,c", [(4, 6, 2), (9, 9, 4), (7, 12, 1), (6, 6, 5)])
def test_split_after_c_rows_property(Sq, Skv, c):
    """(ours) Cutting a rightDownCausal sequence after c rows leaves a band
    piece with next = c - Sq, pre = Skv (mode 7, last sequence); cutting a
    leftUpCausal one leaves a band piece with next = Sq - Skv, pre = Skv
    (mode 8, first sequence)."""
    N, D = 1, 4
    m3 = oracle.mask_matrix(Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=3), 0)
    top = Problem("TND", 1, N, c, Skv, D, sparse_mode=7, pre_tokens=Skv, next_tokens=c - Sq,
                  actual_seq_qlen=[c], actual_seq_kvlen=[Skv])
    assert np.array_equal(oracle.mask_matrix(top, 0), m3[:c])
    bot = Problem("TND", 1, N, Sq - c, Skv, D, sparse_mode=3, actual_seq_qlen=[Sq - c],
                  actual_seq_kvlen=[Skv])
    assert np.array_equal(oracle.mask_matrix(bot, 0), m3[c:])
    m2 = oracle.mask_matrix(Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=2), 0)
    top2 = Problem("TND", 1, N, c, Skv, D, sparse_mode=2, actual_seq_qlen=[c],
                   actual_seq_kvlen=[Skv])
    assert np.array_equal(oracle.mask_matrix(top2, 0), m2[:c])
    bot2 = Problem("TND", 1, N, Sq - c, Skv, D, sparse_mode=8, pre_tokens=Skv,
                   next_tokens=Sq - Skv, actual_seq_qlen=[Sq - c], actual_seq_kvlen=[Skv])
    assert np.array_equal(oracle.mask_matrix(bot2, 0), m2[c:])


def test_mode7_only_last_nonempty_sequence_is_band():
    """A trailing empty sequence does not take the band role."""
    pb = Problem("TND", 3, 1, 5, 12, 4, sparse_mode=7, pre_tokens=5, next_tokens=-1,
                 actual_seq_qlen=[2, 5, 5], actual_seq_kvlen=[4, 9, 12])
    m1 = oracle.mask_matrix(pb, 1)  # the band sequence (3 x 5)
    ref = oracle.mask_matrix(Problem("BNSD", 1, 1, 3, 5, 4, sparse_mode=4, pre_tokens=5,
                                     next_tokens=-1), 0)
    assert np.array_equal(m1, ref)
    m0 = oracle.mask_matrix(pb, 0)  # rightDownCausal sequence (2 x 4)
    assert np.array_equal(m0, oracle.mask_matrix(Problem("BNSD", 1, 1, 2, 4, 4, sparse_mode=3), 0))


def test_mode8_only_first_nonempty_sequence_is_band():
    pb = Problem("TND", 3, 1, 5, 12, 4, sparse_mode=8, pre_tokens=5, next_tokens=0,
                 actual_seq_qlen=[0, 3, 5], actual_seq_kvlen=[3, 8, 12])
    m1 = oracle.mask_matrix(pb, 1)
    ref = oracle.mask_matrix(Problem("BNSD", 1, 1, 3, 5, 4, sparse_mode=4, pre_tokens=5,
                                     next_tokens=0), 0)
    assert np.array_equal(m1, ref)
    m2 = oracle.mask_matrix(pb, 2)
    assert np.array_equal(m2, oracle.mask_matrix(Problem("BNSD", 1, 1, 2, 4, 4, sparse_mode=2), 0))


# --------------------------------------------------------------------------
# Closed-form counts, brute force over tiny shapes.
# --------------------------------------------------------------------------

def test_visible_counts_closed_forms():
    S = 37
    assert oracle.visible_count(Problem("BNSD", 2, 3, S, S, 4, sparse_mode=2)) == 6 * S * (S + 1) // 2
    Sq, Skv = 20, 31
    d = Skv - Sq
    assert oracle.visible_count(Problem("BNSD", 1, 1, Sq, Skv, 4, sparse_mode=3)) == \
        sum(min(i + d + 1, Skv) for i in range(Sq))
    # right-down band of the long-context band workload, scaled down 16x:
    # every row sees pre + 1 keys
    Sq, Skv, pre = 128, 512, 64
    assert oracle.visible_count(Problem("BSND", 1, 2, Sq, Skv, 4, sparse_mode=4,
                                        pre_tokens=pre, next_tokens=0)) == 2 * Sq * (pre + 1)
    # prefix: P^2 + S(S+1)/2 - P(P+1)/2 when Sq = Skv = S
    S = 40
    pref = [0, 7, 25, 40]
    expect = sum(P * P + S * (S + 1) // 2 - P * (P + 1) // 2 for P in pref)
    assert oracle.visible_count(Problem("BNSD", 4, 1, S, S, 4, sparse_mode=5,
                                        prefix=pref)) == expect


def test_bruteforce_tiny_shapes_rows_are_intervals():
    """Over all tiny shapes and pre/next, every row of modes 0 (all-False
    mask), 2, 3, 4 is one contiguous run of keys, and the runs move right
    (never left) from row to row."""
    for Sq in range(1, 7):
        for Skv in range(1, 7):
            cases = [(2, 0, 0), (3, 0, 0)]
            cases += [(m, p, n) for m in (0, 4) for p in range(-7, 8) for n in range(-7, 8)]
            for mode, pre, nxt in cases:
                kw = {}
                if mode == 0:
                    kw = dict(mask=np.zeros((Sq, Skv), np.uint8), mask_kind="SS")
                m = oracle.mask_matrix(Problem("BNSD", 1, 1, Sq, Skv, 2, sparse_mode=mode,
                                               pre_tokens=pre, next_tokens=nxt, **kw), 0)
                last_lo = last_hi = -1
                for i in range(Sq):
                    idx = np.nonzero(m[i])[0]
                    if len(idx) == 0:
                        continue
                    assert idx[-1] - idx[0] + 1 == len(idx)
                    assert idx[0] >= last_lo and idx[-1] >= last_hi
                    last_lo, last_hi = idx[0], idx[-1]


# --------------------------------------------------------------------------
# Closed forms of the attention values.
# --------------------------------------------------------------------------

def test_zero_qk_gives_mean_of_visible_values():
    B, N, Sq, Skv, D = 1, 2, 9, 14, 8
    q = torch.zeros(B, N, Sq, D, dtype=torch.float64)
    k = torch.zeros(B, N, Skv, D, dtype=torch.float64)
    v = _rand((B, N, Skv, D), 31)
    pb = Problem("BNSD", B, N, Sq, Skv, D, sparse_mode=4, pre_tokens=3, next_tokens=1)
    o, lse = oracle.attention(pb, q, k, v)
    vis = oracle.mask_matrix(pb, 0)
    for h in range(N):
        for i in range(Sq):
            n = vis[i].sum()
            if n == 0:
                assert np.all(o[0, h, i] == 0) and lse[0, h, i] == -np.inf
            else:
                np.testing.assert_allclose(o[0, h, i], v[0, h][vis[i] == 1].mean(0).numpy(),
                                           atol=1e-14)
                assert abs(lse[0, h, i] - math.log(n)) < 1e-14


def test_single_visible_key_and_constant_values():
    B, N, S, D = 1, 1, 6, 4
    q, k = _rand((B, N, S, D), 32), _rand((B, N, S, D), 33)
    v = _rand((B, N, S, D), 34)
    one = np.ones((S, S), np.uint8)
    perm = [3, 0, 5, 1, 4, 2]
    for i, j in enumerate(perm):
        one[i, j] = 0
    pb = Problem("BNSD", B, N, S, S, D, sparse_mode=1, mask=one, mask_kind="SS")
    o, lse = oracle.attention(pb, q, k, v)
    for i, j in enumerate(perm):
        np.testing.assert_array_equal(o[0, 0, i], v[0, 0, j].numpy())
        assert abs(lse[0, 0, i] - pb.scale * float(q[0, 0, i] @ k[0, 0, j])) < 1e-14
    vc = torch.full((B, N, S, D), 2.5, dtype=torch.float64)
    o2, _ = oracle.attention(Problem("BNSD", B, N, S, S, D, sparse_mode=2), q, k, vc)
    np.testing.assert_allclose(o2, 2.5, atol=1e-14)


def test_key_shift_invariance():
    """K <- K + 1 u^T leaves O unchanged and moves lse_i by scale * q_i . u."""
    B, N, S, D = 1, 2, 11, 8
    q, k, v = _rand((B, N, S, D), 35), _rand((B, N, S, D), 36), _rand((B, N, S, D), 37)
    u = _rand((D,), 38)
    pb = Problem("BNSD", B, N, S, S, D, sparse_mode=5, prefix=[4])
    o, lse = oracle.attention(pb, q, k, v)
    o2, lse2 = oracle.attention(pb, q, k + u, v)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(lse2 - lse, (pb.scale * q @ u).numpy(), atol=1e-12)


def test_fully_masked_rows_give_zero_and_minus_inf():
    # right-down band with Sq > Skv: the first rows see nothing
    pb = Problem("BNSD", 1, 1, 8, 3, 4, sparse_mode=3)
    q, k, v = _rand((1, 1, 8, 4), 39), _rand((1, 1, 3, 4), 40), _rand((1, 1, 3, 4), 41)
    o, lse = oracle.attention(pb, q, k, v)
    assert np.all(o[0, 0, :5] == 0) and np.all(lse[0, 0, :5] == -np.inf)
    assert np.all(np.isfinite(lse[0, 0, 5:]))


def test_rows_entry_matches_full_forward():
    pb = Problem("BSND", 2, 3, 10, 13, 8, sparse_mode=4, pre_tokens=4, next_tokens=2)
    q, k, v = _rand((2, 10, 3, 8), 42), _rand((2, 13, 3, 8), 43), _rand((2, 13, 3, 8), 44)
    o, lse = oracle.attention(pb, q, k, v)
    rows = [(0, 0, 0), (1, 2, 9), (0, 1, 5), (1, 0, 3)]
    orow, lrow = oracle.attention_rows(pb, q, k, v, rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(orow[r], o[b, i, h])
        assert lrow[r] == lse[b, h, i]


# --------------------------------------------------------------------------
# The exercise page's online-softmax recurrence.
# --------------------------------------------------------------------------

def test_tiled_recurrence_page_example_1():
    """Example 1: seed 42, (B, N, D) = (2, 12, 16), float64, block 4, scale 1/sqrt(D)."""
    torch.manual_seed(42)
    B, N, D = 2, 12, 16
    q = torch.randn(B, N, D, dtype=torch.float64)
    k = torch.randn(B, N, D, dtype=torch.float64)
    v = torch.randn(B, N, D, dtype=torch.float64)
    scores = torch.matmul(q, k.transpose(-2, -1)) / math.sqrt(D)
    ref = torch.matmul(F.softmax(scores, dim=-1), v).numpy()
    out = oracle.flash_tiled(q, k, v, block_size=4)
    assert out.shape == (2, 12, 16) and out.dtype == np.float64
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_tiled_recurrence_every_block_size_with_ragged_tail():
    """Example 2's shape (1, 7, 8) with block 3 leaves a one-key tail block;
    every block size 1..S must give the unfused result."""
    for shape in [(1, 7, 8), (2, 12, 16)]:
        B, S, D = shape
        q, k, v = _rand(shape, 50), _rand(shape, 51), _rand(shape, 52)
        ref = _sdpa(q[:, None], k[:, None], v[:, None], 1 / math.sqrt(D))[:, 0].numpy()
        for blk in range(1, S + 1):
            out = oracle.flash_tiled(q, k, v, block_size=blk)
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_tiled_recurrence_with_masks_matches_masked_softmax():
    """Fully masked blocks leave (m, l, O) unchanged: the tiled form with a
    sparseMode mask equals the plain masked softmax for every block size."""
    B, S, D = 1, 11, 8
    q, k, v = _rand((B, S, D), 53), _rand((B, S, D), 54), _rand((B, S, D), 55)
    for mode, kw in [(4, dict(pre_tokens=2, next_tokens=-1)), (5, dict(prefix=[3])),
                     (2, {})]:
        pb = Problem("BNSD", 1, 1, S, S, D, sparse_mode=mode, **kw)
        o, _ = oracle.attention(pb, q[:, None], k[:, None], v[:, None])
        vis = oracle.mask_matrix(pb, 0)[None]
        for blk in (1, 2, 3, 5, 11):
            out = oracle.flash_tiled(q, k, v, block_size=blk, vis=vis)
            np.testing.assert_allclose(out, o[:, 0], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Block occupancy of the visibility matrix (what the attention may skip or
# compute without the element mask) and the key-block range per query block.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("nb", [1, 4])
def test_tile_classes_of_causal_are_the_triangle(nb):
    """leftUpCausal on a square of nb x nb whole blocks: blocks below the
    diagonal are all visible, diagonal blocks mixed, blocks above it empty."""
    S = 128 * nb
    pb = Problem("BNSD", 1, 1, S, S, 8, sparse_mode=2)
    qt, kt = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    want = np.where(kt < qt, 2, np.where(kt == qt, 1, 0)).astype(np.uint8)
    assert np.array_equal(oracle.tile_classes(pb, 0), want)
    r = oracle.tile_ranges(want)
    for q in range(nb):
        assert r[q].tolist() == [0, q + 1, 0, q]


@pytest.mark.parametrize("pre", [300, 10 ** 6])
def test_tile_classes_of_band_mask_zero_equal_causal(pre):
    """sparseMode 0 with an all-zero mask, nextTokens 0 and preTokens >= Sq is
    causal (the page's "causal via band"), block by block."""
    S = 256
    zero = np.zeros((S, S), dtype=np.uint8)
    pb0 = Problem("BNSD", 1, 1, S, S, 8, sparse_mode=0, pre_tokens=pre, next_tokens=0,
                  mask=zero, mask_kind="SS")
    pb2 = Problem("BNSD", 1, 1, S, S, 8, sparse_mode=2)
    assert np.array_equal(oracle.tile_classes(pb0, 0), oracle.tile_classes(pb2, 0))


def test_tile_classes_of_open_and_closed_masks():
    """allMask with nothing masked: whole key blocks are full, the ragged last
    key block (keys past Skv) is mixed; everything masked: all empty."""
    Sq, Skv = 300, 333
    open_ = Problem("BNSD", 1, 1, Sq, Skv, 8, sparse_mode=1,
                    mask=np.zeros((Sq, Skv), np.uint8), mask_kind="SS")
    want = np.array([[2, 2, 1]] * 3, dtype=np.uint8)
    assert np.array_equal(oracle.tile_classes(open_, 0), want)
    assert oracle.tile_ranges(want).tolist() == [[0, 3, 0, 2]] * 3
    shut = Problem("BNSD", 1, 1, Sq, Skv, 8, sparse_mode=1,
                   mask=np.ones((Sq, Skv), np.uint8), mask_kind="SS")
    assert not oracle.tile_classes(shut, 0).any()
    assert not oracle.tile_ranges(np.zeros((3, 3), np.uint8)).any()


def test_tile_classes_of_a_constructed_block_mask():
    """Blocks of 4 on a 10 x 13 allMask, each block set up to have a known
    class: whole-visible (2), one visible pair (1), one hidden pair (1),
    visible rows that end at Sq (2: rows past Sq do not exist), visible keys
    that end at Skv (1: the block's keys past Skv do not exist), hidden (0).
    Per batch and head (BNSS) the classes follow that plane's mask."""
    Sq, Skv, t = 10, 13, 4
    m = np.ones((2, 1, Sq, Skv), dtype=np.uint8)
    m[0, 0, 0:4, 0:4] = 0          # (0, 0) full
    m[0, 0, 1, 6] = 0              # (0, 1) one visible pair
    m[0, 0, 4:8, 8:12] = 0         # (1, 2) full ...
    m[0, 0, 5, 9] = 1              # ... but one hidden pair: mixed
    m[0, 0, 8:10, 0:4] = 0         # (2, 0) rows 8, 9 only: full
    m[0, 0, 8:10, 12] = 0          # (2, 3) key 12 only: mixed
    m[1, 0, 4:8, 4:8] = 0          # batch 1: (1, 1) full
    pb = Problem("BNSD", 2, 1, Sq, Skv, 8, sparse_mode=1, mask=m, mask_kind="B1SS")
    want0 = np.zeros((3, 4), np.uint8)
    want0[0, 0], want0[0, 1], want0[1, 2], want0[2, 0], want0[2, 3] = 2, 1, 1, 2, 1
    assert np.array_equal(oracle.tile_classes(pb, 0, tile=t), want0)
    want1 = np.zeros((3, 4), np.uint8)
    want1[1, 1] = 2
    assert np.array_equal(oracle.tile_classes(pb, 1, tile=t), want1)
    assert oracle.tile_ranges(want0).tolist() == [[0, 2, 0, 1], [2, 3, 2, 2], [0, 4, 0, 1]]
    assert oracle.tile_ranges(want1).tolist() == [[0, 0, 0, 0], [1, 2, 1, 2], [0, 0, 0, 0]]


@pytest.mark.parametrize("row,want", [
    ([0, 1, 2, 2, 0, 2, 2, 2, 1, 0], [1, 9, 5, 8]),   # longest full run wins
    ([2, 2, 0, 2, 2], [0, 5, 0, 2]),                  # equal runs: the first
    ([1, 0, 1], [0, 3, 0, 0]),                        # no full block: lo, lo
    ([0, 0, 2], [2, 3, 2, 3]),
    ([0, 0, 0], [0, 0, 0, 0]),                        # nothing visible
])
def test_tile_ranges_hand_cases(row, want):
    assert oracle.tile_ranges(np.array([row], np.uint8)).tolist() == [want]


def test_tile_classes_match_bruteforce_blocks():
    """Against the visibility matrix cut into blocks by numpy, over every
    sparseMode on a small ragged shape with tile 5."""
    rng = np.random.default_rng(3)
    Sq, Skv, t = 17, 23, 5
    for mode, extra in [(0, dict(pre_tokens=6, next_tokens=2)), (1, {}), (2, {}), (3, {}),
                        (4, dict(pre_tokens=7, next_tokens=1))]:
        mask = None
        if mode <= 1:
            mask = (rng.random((Sq, Skv)) < 0.2).astype(np.uint8)
            mask[:, 15:] = 0                       # some whole-visible blocks
            mask[10:15, :] = 1                     # a hidden block row
        pb = Problem("BNSD", 1, 1, Sq, Skv, 8, sparse_mode=mode, mask=mask,
                     mask_kind="SS" if mask is not None else None, **extra)
        vis = oracle.mask_matrix(pb, 0).astype(bool)
        pad = np.zeros((-(-Sq // t) * t, -(-Skv // t) * t), dtype=bool)
        pad[:Sq, :Skv] = vis
        got = oracle.tile_classes(pb, 0, tile=t)
        for qt in range(got.shape[0]):
            for kt in range(got.shape[1]):
                blk = pad[qt * t:min((qt + 1) * t, Sq), kt * t:(kt + 1) * t]
                cls = 2 if blk.all() else (1 if blk.any() else 0)
                assert got[qt, kt] == cls, (mode, qt, kt)


# --------------------------------------------------------------------------
# Paged K/V caches ("Norm" layout of the aclnnScatterPaKvCache page): key j
# of sequence b sits at block block_table[b][j // bs], offset j % bs.
# --------------------------------------------------------------------------

def _paged_from_packed(k, v, cu_kv, bs, rng, spare=3, shuffle=True):
    """Scatter packed TND K/V [T_kv, N, D] into caches of bs-token blocks in a
    random block order; unused slots hold NaN so that reading one shows."""
    T, N, D = k.shape
    lens = np.diff(np.concatenate([[0], cu_kv]))
    nblk = [(-(-int(n) // bs)) for n in lens]
    total = sum(nblk) + spare
    order = rng.permutation(total) if shuffle else np.arange(total)
    kc = np.full((total, bs, N, D), np.nan)
    vc = np.full((total, bs, N, D), np.nan)
    table = np.full((len(lens), max(max(nblk), 1)), -1, dtype=np.int32)
    nxt, start = 0, 0
    for b, n in enumerate(lens):
        for c in range(nblk[b]):
            blk = int(order[nxt]); nxt += 1
            table[b, c] = blk
            rows = np.arange(c * bs, min((c + 1) * bs, n))
            kc[blk, :len(rows)] = k[start + rows]
            vc[blk, :len(rows)] = v[start + rows]
        start += n
    return kc, vc, table


@pytest.mark.parametrize("mode,extra", [(3, {}), (2, {}), (0, {}), (4, dict(pre_tokens=5, next_tokens=1))])
@pytest.mark.parametrize("bs", [4, 16])
def test_paged_equals_packed_forward(mode, extra, bs):
    """The paged forward with any block order equals the packed TND forward
    (already pinned to SDPA and the page's examples), and never reads a slot
    outside the sequences' keys (those hold NaN)."""
    rng = np.random.default_rng(11)
    lq, lkv = [1, 3, 0, 2], [7, 19, 5, 33]
    cu_q, cu_kv = np.cumsum(lq).tolist(), np.cumsum(lkv).tolist()
    N, D = 2, 8
    q = rng.standard_normal((cu_q[-1], N, D))
    k = rng.standard_normal((cu_kv[-1], N, D))
    v = rng.standard_normal((cu_kv[-1], N, D))
    pb = Problem("TND", len(lq), N, cu_q[-1], cu_kv[-1], D, sparse_mode=mode,
                 actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv, **extra)
    o_ref, l_ref = oracle.attention(pb, q, k, v)
    for shuffle in (False, True):
        kc, vc, table = _paged_from_packed(k, v, np.array(cu_kv), bs, rng, shuffle=shuffle)
        o, l = oracle.attention_paged(pb, q, kc, vc, table, bs)
        assert np.all(np.isfinite(o))
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
        np.testing.assert_array_equal(np.isneginf(l), np.isneginf(l_ref))
        live = ~np.isneginf(l_ref)
        np.testing.assert_allclose(l[live], l_ref[live], rtol=0, atol=1e-13)


def test_paged_decode_row_is_sdpa_over_the_gathered_keys():
    """One decode row per sequence (rightDownCausal sees every key): torch
    SDPA over the keys gathered by hand from the block table."""
    rng = np.random.default_rng(12)
    lkv = [9, 1, 40]
    cu_q, cu_kv = [1, 2, 3], np.cumsum(lkv).tolist()
    N, D, bs = 3, 16, 8
    q = rng.standard_normal((3, N, D))
    k = rng.standard_normal((cu_kv[-1], N, D))
    v = rng.standard_normal((cu_kv[-1], N, D))
    kc, vc, table = _paged_from_packed(k, v, np.array(cu_kv), bs, rng)
    pb = Problem("TND", 3, N, 3, cu_kv[-1], D, sparse_mode=3, actual_seq_qlen=cu_q,
                 actual_seq_kvlen=cu_kv)
    o, l = oracle.attention_paged(pb, q, kc, vc, table, bs)
    for b, n in enumerate(lkv):
        idx = np.arange(n)
        kb = kc[table[b, idx // bs], idx % bs]          # [n, N, D]
        vb = vc[table[b, idx // bs], idx % bs]
        qt = torch.from_numpy(q[b]).unsqueeze(1)           # [N, 1, D]
        ref = _sdpa(qt, torch.from_numpy(kb).transpose(0, 1), torch.from_numpy(vb).transpose(0, 1),
                    pb.scale).squeeze(1).numpy()
        np.testing.assert_allclose(o[b], ref, rtol=0, atol=1e-12)
        s = pb.scale * np.einsum("hd,nhd->hn", q[b], kb)
        np.testing.assert_allclose(l[:, b], np.log(np.exp(s).sum(1)), rtol=0, atol=1e-12)


def _runs_of_full(row):
    """Every maximal run of class-2 blocks as (start, end)."""
    runs, k = [], 0
    while k < len(row):
        if row[k] == 2:
            e = k
            while e < len(row) and row[e] == 2:
                e += 1
            runs.append((k, e))
            k = e
        else:
            k += 1
    return runs


@pytest.mark.parametrize("seed", range(6))
def test_tile_ranges_properties_on_random_class_rows(seed):
    """Properties any correct block range must have, on random class rows:
    [lo, hi) holds every non-empty block and starts and ends on one; nothing
    outside it is non-empty; [full_lo, full_hi) holds only full blocks and is
    a maximal run that no other run of full blocks is longer than (on ties no
    earlier run is as long); with no full block it is the empty run at lo.
    These do not depend on the loop the oracle uses to find them."""
    rng = np.random.default_rng(seed)
    n_qt, n_kt = 40, int(rng.integers(1, 30))
    p = rng.dirichlet([1.0, 1.0, 1.0])
    cls = rng.choice(3, size=(n_qt, n_kt), p=p).astype(np.uint8)
    cls[0] = 0                        # a query block without a visible pair
    cls[1] = 2                        # one that is full end to end
    got = oracle.tile_ranges(cls)
    for qt in range(n_qt):
        row = cls[qt]
        lo, hi, flo, fhi = (int(x) for x in got[qt])
        nz = np.flatnonzero(row)
        if nz.size == 0:
            assert (lo, hi, flo, fhi) == (0, 0, 0, 0)
            continue
        assert lo == nz[0] and hi == nz[-1] + 1          # tight cover of the non-empty blocks
        assert not row[:lo].any() and not row[hi:].any()
        runs = _runs_of_full(row)
        if not runs:
            assert (flo, fhi) == (lo, lo)
            continue
        assert lo <= flo < fhi <= hi
        assert np.all(row[flo:fhi] == 2)
        assert (flo, fhi) in runs                         # a maximal run, not part of one
        longest = max(e - s for s, e in runs)
        assert fhi - flo == longest
        assert all(s >= flo for s, e in runs if e - s == longest)


# --------------------------------------------------------------------------
# ALiBi bias ("压缩mask" page, alibi section): per-head coefficient (slope)
# times a bias, plus the triangular mask. Readings: right-aligned bias =
# signed distance of key j from the row's bottom-right-anchored diagonal;
# sqrt variant = the square root of that distance's size, sign kept;
# left-aligned bias = j.
# --------------------------------------------------------------------------

ALIBI_SLOPES = [0.5, 0.125]


def _zero_qk_identity_v(Sq, Skv, N):
    """Q = K = 0 (every visible score is the bias alone) and V[j] = e_j, so
    O[i, j] is the softmax weight of key j in row i."""
    D = Skv
    q = np.zeros((1, N, Sq, D))
    k = np.zeros((1, N, Skv, D))
    v = np.zeros((1, N, Skv, D))
    for h in range(N):
        v[0, h, np.arange(Skv), np.arange(Skv)] = 1.0
    return q, k, v


@pytest.mark.parametrize("Sq,Skv", [(5, 9), (7, 7)])
def test_alibi_right_aligned_is_a_geometric_series(Sq, Skv):
    """rightDownCausal with zero scores: row i sees n = i + delta + 1 keys with
    weights exp(-a m), m = i + delta - j = 0..n-1, so lse = ln((1 - e^{-an}) /
    (1 - e^{-a})) and O[i, j] = e^{-a m} (1 - e^{-a}) / (1 - e^{-an})."""
    N = len(ALIBI_SLOPES)
    q, k, v = _zero_qk_identity_v(Sq, Skv, N)
    pb = Problem("BNSD", 1, N, Sq, Skv, Skv, sparse_mode=3)
    o, lse = oracle.attention(pb, q, k, v, alibi="right", slopes=ALIBI_SLOPES)
    delta = Skv - Sq
    for h, a in enumerate(ALIBI_SLOPES):
        for i in range(Sq):
            n = i + delta + 1
            assert lse[0, h, i] == pytest.approx(np.log((1 - np.exp(-a * n)) / (1 - np.exp(-a))),
                                                 abs=1e-13)
            want = np.zeros(Skv)
            m = i + delta - np.arange(n)
            want[:n] = np.exp(-a * m) * (1 - np.exp(-a)) / (1 - np.exp(-a * n))
            np.testing.assert_allclose(o[0, h, i], want, rtol=0, atol=1e-14)


def test_alibi_sqrt_equals_right_aligned_at_unit_distances():
    """A band one key wide on each side of the diagonal (pre = 1, next = 1)
    holds distances -1, 0, 1 only, whose square roots are themselves: the two
    variants agree there; at larger distances they do not."""
    Sq, Skv, D, N = 9, 12, 8, 2
    q, k, v = _rand((1, N, Sq, D), 61), _rand((1, N, Skv, D), 62), _rand((1, N, Skv, D), 63)
    pb = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=4, pre_tokens=1, next_tokens=1)
    o_r, l_r = oracle.attention(pb, q, k, v, alibi="right", slopes=ALIBI_SLOPES)
    o_s, l_s = oracle.attention(pb, q, k, v, alibi="sqrt", slopes=ALIBI_SLOPES)
    np.testing.assert_allclose(o_s, o_r, rtol=0, atol=1e-14)
    np.testing.assert_allclose(l_s, l_r, rtol=0, atol=1e-14)
    wide = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=3)
    assert not np.allclose(oracle.attention(wide, q, k, v, alibi="sqrt", slopes=ALIBI_SLOPES)[1],
                           oracle.attention(wide, q, k, v, alibi="right", slopes=ALIBI_SLOPES)[1])


def test_alibi_sqrt_on_zero_scores():
    """rightDownCausal with zero scores and the square-root bias: weights
    exp(-a sqrt(m)) over m = 0..n-1."""
    Sq, Skv = 6, 8
    N = len(ALIBI_SLOPES)
    q, k, v = _zero_qk_identity_v(Sq, Skv, N)
    pb = Problem("BNSD", 1, N, Sq, Skv, Skv, sparse_mode=3)
    o, lse = oracle.attention(pb, q, k, v, alibi="sqrt", slopes=ALIBI_SLOPES)
    for h, a in enumerate(ALIBI_SLOPES):
        for i in range(Sq):
            n = i + (Skv - Sq) + 1
            w = np.exp(-a * np.sqrt(np.arange(n)[::-1].astype(float)))
            assert lse[0, h, i] == pytest.approx(np.log(w.sum()), abs=1e-13)
            np.testing.assert_allclose(o[0, h, i, :n], w / w.sum(), rtol=0, atol=1e-14)


@pytest.mark.parametrize("mode,extra", [(3, {}), (2, {}), (4, dict(pre_tokens=4, next_tokens=2)),
                                        (0, {})])
def test_alibi_left_aligned_moves_only_lse(mode, extra):
    """Left- and right-aligned biases differ by slope * (i + delta) in each
    row, a constant the softmax removes: O is the same, lse moves by it."""
    Sq, Skv, D, N = 7, 10, 8, 2
    q, k, v = _rand((1, N, Sq, D), 71), _rand((1, N, Skv, D), 72), _rand((1, N, Skv, D), 73)
    pb = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=mode, **extra)
    o_r, l_r = oracle.attention(pb, q, k, v, alibi="right", slopes=ALIBI_SLOPES)
    o_l, l_l = oracle.attention(pb, q, k, v, alibi="left", slopes=ALIBI_SLOPES)
    np.testing.assert_allclose(o_l, o_r, rtol=0, atol=1e-13)
    for h, a in enumerate(ALIBI_SLOPES):
        np.testing.assert_allclose(l_l[0, h] - l_r[0, h], a * (np.arange(Sq) + Skv - Sq),
                                   rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode,extra", [(3, {}), (0, {}), (5, dict(prefix=[4]))])
def test_alibi_matches_sdpa_with_an_additive_mask(mode, extra):
    """torch SDPA (fp64) with a float attn_mask: slope * bias on visible pairs
    and -inf elsewhere, added to the scaled scores (the bias is not scaled);
    keys right of the diagonal (mode 0, the prefix) get a positive bias."""
    Sq, Skv, D, N = 6, 11, 8, 2
    q, k, v = _rand((1, N, Sq, D), 81), _rand((1, N, Skv, D), 82), _rand((1, N, Skv, D), 83)
    pb = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=mode, **extra)
    vis = oracle.mask_matrix(pb, 0).astype(bool)
    dist = np.arange(Skv)[None, :] - (np.arange(Sq)[:, None] + Skv - Sq)
    add = np.stack([np.where(vis, a * dist, -np.inf) for a in ALIBI_SLOPES])[None]
    want = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=torch.from_numpy(add), scale=pb.scale).numpy()
    o, lse = oracle.attention(pb, q, k, v, alibi="right", slopes=ALIBI_SLOPES)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    s = np.einsum("bhid,bhjd->bhij", q.numpy(), k.numpy()) * pb.scale + add
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(s), -1).numpy(), atol=1e-12)


def test_alibi_with_zero_slopes_is_the_plain_forward():
    Sq, Skv, D, N = 9, 9, 8, 2
    q, k, v = _rand((1, N, Sq, D), 91), _rand((1, N, Skv, D), 92), _rand((1, N, Skv, D), 93)
    pb = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=2)
    o0, l0 = oracle.attention(pb, q, k, v)
    for kind in ("right", "sqrt", "left"):
        o, lse = oracle.attention(pb, q, k, v, alibi=kind, slopes=[0.0, 0.0])
        assert np.array_equal(o, o0) and np.array_equal(lse, l0)


def test_alibi_rows_entry_matches_full_forward():
    """The sampled-rows entry with a bias gives the full forward's rows."""
    Sq, Skv, D, N = 9, 13, 8, 2
    q, k, v = _rand((1, N, Sq, D), 95), _rand((1, N, Skv, D), 96), _rand((1, N, Skv, D), 97)
    pb = Problem("BNSD", 1, N, Sq, Skv, D, sparse_mode=4, pre_tokens=5, next_tokens=2)
    rows = [(0, h, i) for h in range(N) for i in range(Sq)]
    for kind in ("right", "sqrt", "left"):
        o, lse = oracle.attention(pb, q, k, v, alibi=kind, slopes=ALIBI_SLOPES)
        orow, lrow = oracle.attention_rows(pb, q, k, v, rows, alibi=kind, slopes=ALIBI_SLOPES)
        for r, (_, h, i) in enumerate(rows):
            assert np.array_equal(orow[r], o[0, h, i]) and lrow[r] == lse[0, h, i]
