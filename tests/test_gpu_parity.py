"""GPU parity: the CUDA path against the fp64 oracle, element by element.

Sizes span several 128x128 tiles with ragged tails; every sparseMode,
layout and head dim is covered, plus the exact visibility probe, empty and
fully masked rows, determinism and the pages' worked split examples.
"""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from masked_attention_fa_b200.workloads import random_inputs, varlen_lengths
from gpu_helpers import TOL_LSE, assert_close, check_against_oracle, problem_of, run_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()
    assert torch.cuda.is_available()
    fa.load_library()


def _kw(layout, B, N, Sq, Skv, D, mode, **extra):
    kw = dict(layout=layout, B=B, N=N, Sq=Sq, Skv=Skv, D=D, sparse_mode=mode)
    kw.update(extra)
    return kw


CASES = [
    # (mode, extra kwargs, Sq, Skv)
    (0, {}, 300, 333),
    (0, dict(pre_tokens=70, next_tokens=20, mask_kind="SS"), 300, 333),
    (0, dict(pre_tokens=150, next_tokens=-40, mask_kind="B1SS"), 260, 300),
    (0, dict(pre_tokens=-30, next_tokens=200, mask_kind="BNSS"), 300, 260),
    (1, dict(mask_kind="SS"), 300, 333),
    (1, dict(mask_kind="BNSS"), 129, 385),
    (2, {}, 300, 333),
    (2, {}, 333, 300),
    (3, {}, 300, 333),
    (3, {}, 333, 200),           # Sq > Skv: the first rows see no key
    (4, dict(pre_tokens=100, next_tokens=0), 300, 700),
    (4, dict(pre_tokens=200, next_tokens=-50), 384, 512),
    (4, dict(pre_tokens=-20, next_tokens=90), 256, 256),
    (5, dict(prefix=[40, 333]), 300, 333),
    (6, dict(prefix=[0, 129]), 300, 300),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", ["BNSD", "BSND"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_modes_match_oracle(case, layout, D):
    mode, extra, Sq, Skv = CASES[case]
    extra = dict(extra)
    prefix = extra.pop("prefix", None)
    B, N = 2, 2
    kw = _kw(layout, B, N, Sq, Skv, D, mode, **extra)
    inp = random_inputs(layout, B, N, Sq, Skv, D, seed=1000 + case, mask_kind=kw.get("mask_kind"))
    check_against_oracle(kw, inp, prefix=prefix)


def _tnd_inputs(lens_q, lens_kv, N, D, seed):
    cu_q = np.cumsum(lens_q).tolist()
    cu_k = np.cumsum(lens_kv).tolist()
    inp = random_inputs("TND", len(lens_q), N, cu_q[-1], cu_k[-1], D, seed)
    return cu_q, cu_k, inp


TND_CASES = [
    # mode, extra, lens_q, lens_kv
    (2, {}, [130, 0, 257, 5], [140, 3, 300, 5]),
    (3, {}, [130, 0, 257, 5], [140, 3, 300, 5]),
    (3, {}, [300, 20, 64], [200, 0, 64]),          # Sq > Skv and an empty key set
    (4, dict(pre_tokens=60, next_tokens=10), [200, 129], [260, 400]),
    (5, dict(prefix=[17, 0, 300]), [150, 1, 257], [150, 2, 300]),
    (7, dict(pre_tokens=300, next_tokens=-40), [100, 200, 0], [120, 260, 7]),
    (8, dict(pre_tokens=200, next_tokens=10), [0, 150, 300], [3, 190, 350]),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(TND_CASES)))
def test_varlen_tnd_matches_oracle(case, D):
    mode, extra, lq, lk = TND_CASES[case]
    extra = dict(extra)
    prefix = extra.pop("prefix", None)
    N = 3
    cu_q, cu_k, inp = _tnd_inputs(lq, lk, N, D, seed=2000 + case)
    kw = _kw("TND", len(lq), N, cu_q[-1], cu_k[-1], D, mode, **extra)
    check_against_oracle(kw, inp, prefix=prefix, cu_q=cu_q, cu_kv=cu_k)


def _probe_mask(kind, B, N, Sq, Skv, seed, dead_rows=()):
    """A Bernoulli(0.25) uint8 mask of the given kind, with rows in
    `dead_rows` hidden entirely (rows that see no key)."""
    shape = {"SS": (Sq, Skv), "B1SS": (B, 1, Sq, Skv), "BNSS": (B, N, Sq, Skv)}[kind]
    g = torch.Generator().manual_seed(seed)
    m = (torch.rand(shape, generator=g) < 0.25).to(torch.uint8)
    for r in dead_rows:
        m[..., r, :] = 1
    return m


# (layout, mode, extra kwargs, B, N, Sq or lens_q, Skv or lens_kv, prefix, mask spec)
PROBE_CASES = [
    ("BNSD", 2, {}, 1, 1, 200, 300, None, None),
    ("BNSD", 3, {}, 1, 1, 300, 200, None, None),
    ("BSND", 4, dict(pre_tokens=50, next_tokens=-10), 1, 1, 300, 330, None, None),
    # the right-down band across many key tiles (each sub-tile has two
    # boundary tiles and several full ones)
    ("BSND", 4, dict(pre_tokens=300, next_tokens=0), 1, 2, 256, 1024, None, None),
    ("BNSD", 5, {}, 1, 1, 260, 260, [70], None),
    ("BNSD", 5, {}, 2, 1, 200, 333, [0, 333], None),
    ("BNSD", 6, {}, 1, 1, 300, 520, [130], None),
    ("BNSD", 0, dict(pre_tokens=40, next_tokens=3, mask_kind="SS"), 1, 1, 200, 260, None,
     ("SS", ())),
    ("BSND", 0, dict(pre_tokens=150, next_tokens=-40, mask_kind="B1SS"), 2, 2, 260, 300, None,
     ("B1SS", (5, 131))),
    ("BNSD", 1, dict(mask_kind="SS"), 1, 1, 200, 300, None, ("SS", (0, 77, 199))),
    ("BNSD", 1, dict(mask_kind="BNSS"), 2, 2, 150, 260, None, ("BNSS", (3, 128, 149))),
    ("BSND", 1, dict(mask_kind="B1SS"), 2, 2, 129, 385, None, ("B1SS", (128,))),
    # varlen: the two worked split examples, unsplit and per card
    ("TND", 3, {}, 4, 2, [3, 4, 5, 4], [3, 6, 5, 4], None, None),
    ("TND", 7, dict(pre_tokens=6, next_tokens=-2), 2, 2, [3, 2], [3, 6], None, None),
    ("TND", 3, {}, 3, 2, [2, 5, 4], [6, 5, 4], None, None),
    ("TND", 2, {}, 4, 2, [3, 5, 5, 4], [3, 4, 5, 4], None, None),
    ("TND", 2, {}, 2, 2, [3, 2], [3, 4], None, None),
    ("TND", 8, dict(pre_tokens=4, next_tokens=1), 3, 2, [3, 5, 4], [4, 5, 4], None, None),
    # varlen with empty sequences (a trailing one, one in the middle)
    ("TND", 3, {}, 4, 2, [130, 0, 257, 0], [140, 3, 300, 0], None, None),
    # modes 7 and 8 with a band sequence spanning several key tiles
    ("TND", 7, dict(pre_tokens=1000, next_tokens=-100), 3, 2, [100, 0, 700], [150, 3, 1000],
     None, None),
    ("TND", 8, dict(pre_tokens=950, next_tokens=-50), 3, 2, [0, 600, 300], [3, 900, 350], None,
     None),
    ("TND", 4, dict(pre_tokens=60, next_tokens=10), 2, 1, [200, 129], [260, 400], None, None),
    ("TND", 5, {}, 3, 1, [150, 1, 257], [150, 2, 300], [17, 0, 300], None),
]


def _probe_case(case):
    layout, mode, extra, B, N, sq, skv, prefix, mspec = PROBE_CASES[case]
    cu_q = cu_kv = None
    if layout == "TND":
        cu_q, cu_kv = np.cumsum(sq).tolist(), np.cumsum(skv).tolist()
        sq, skv = cu_q[-1], cu_kv[-1]
    mask = None
    if mspec is not None:
        mask = _probe_mask(mspec[0], B, N, sq, skv, seed=7 + case, dead_rows=mspec[1])
    return _kw(layout, B, N, sq, skv, None, mode, **extra), mask, prefix, cu_q, cu_kv


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(PROBE_CASES)))
def test_visibility_probe_is_exact(case, D):
    """Q = K = 0 and, for key block c of every sequence, V = the identity on
    that block (V[j, j - cD] = 1): then O[i, j - cD] != 0 exactly when key j
    is visible to row i (every visible key gets the same weight 1/|vis(i)|,
    a power-of-two fraction or a bf16 value well above 0, every hidden key
    exactly 0), for every sequence and head; and lse_i = ln |vis(i)|, -inf
    for a row that sees no key. Compared with the oracle's visibility matrix
    with no tolerance."""
    kw, mask, prefix, cu_q, cu_kv = _probe_case(case)
    kw["D"] = D
    layout, B, N, Sq, Skv = kw["layout"], kw["B"], kw["N"], kw["Sq"], kw["Skv"]
    pb = problem_of(kw, mask, prefix, cu_q, cu_kv)
    seqs = [pb.seq(b) for b in range(B)]
    shape_q = pb.q_shape()
    shape_kv = pb.kv_shape()
    q = torch.zeros(shape_q, dtype=torch.bfloat16)
    k = torch.zeros(shape_kv, dtype=torch.bfloat16)
    seen = {(b, h): np.zeros((s[2], s[3]), dtype=bool) for b, s in enumerate(seqs)
            for h in range(N)}
    lse_all = None
    n_blocks = max((s[3] + D - 1) // D for s in seqs) if seqs else 0
    for c in range(max(n_blocks, 1)):
        v = torch.zeros(shape_kv, dtype=torch.bfloat16)
        for b, (_, k0, _, skv_b) in enumerate(seqs):
            if skv_b <= c * D:
                continue
            jj = torch.arange(c * D, min(skv_b, (c + 1) * D))
            for h in range(N):
                if layout == "BNSD":
                    v[b, h, jj, jj - c * D] = 1
                elif layout == "BSND":
                    v[b, jj, h, jj - c * D] = 1
                else:
                    v[k0 + jj, h, jj - c * D] = 1
        o, lse = run_cuda(kw, q, k, v, mask, prefix, cu_q, cu_kv)
        lse_all = lse
        for b, (q0, _, sq_b, skv_b) in enumerate(seqs):
            w = min(skv_b, (c + 1) * D) - c * D
            if w <= 0 or sq_b == 0:
                continue
            for h in range(N):
                if layout == "BNSD":
                    ob = o[b, h]
                elif layout == "BSND":
                    ob = o[b, :, h]
                else:
                    ob = o[q0:q0 + sq_b, h]
                seen[(b, h)][:, c * D:c * D + w] = ob[:, :w] != 0
    for b, (q0, _, sq_b, skv_b) in enumerate(seqs):
        for h in range(N):
            vis = oracle.mask_matrix(pb, b, h).astype(bool)
            assert np.array_equal(seen[(b, h)], vis), (b, h)
            cnt = vis.sum(1)
            lrow = lse_all[h, q0:q0 + sq_b] if layout == "TND" else lse_all[b, h]
            assert np.all(np.isneginf(lrow[cnt == 0])), (b, h)
            np.testing.assert_allclose(lrow[cnt > 0], np.log(cnt[cnt > 0]), rtol=0,
                                       atol=TOL_LSE)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("growth", ["rising", "falling"])
def test_running_max_rescale_paths(growth, D):
    """Keys whose norm rises (falls) along the sequence, with large logits
    (up to ~60 at scale 1/sqrt(D)): the running maximum of a row moves up
    tile after tile, so the lazy rescale of O is taken on many tiles (or only
    on the first); both must match the oracle."""
    layout, B, N, Sq, Skv = "BNSD", 1, 2, 256, 1200
    inp = random_inputs(layout, B, N, Sq, Skv, D, seed=77)
    j = torch.arange(Skv, dtype=torch.float32)
    f = 1 + 5 * j / Skv if growth == "rising" else 6 - 5 * j / Skv
    k = (inp["k"].float() * f.view(1, 1, Skv, 1)).to(torch.bfloat16)
    q = (inp["q"].float() * 3).to(torch.bfloat16)
    kw = _kw(layout, B, N, Sq, Skv, D, 0)  # mode 0 without a mask: every key visible
    check_against_oracle(kw, {"q": q, "k": k, "v": inp["v"]})


@pytest.mark.parametrize("scale", [0.05, 0.3])
def test_explicit_scale(scale):
    """A scale other than 1/sqrt(D) is applied to q.k before the softmax."""
    kw = _kw("BSND", 2, 2, 300, 420, 128, 3, scale=scale)
    inp = random_inputs("BSND", 2, 2, 300, 420, 128, seed=91)
    check_against_oracle(kw, inp)


def test_deterministic_bitwise():
    kw = _kw("BNSD", 2, 4, 700, 900, 128, 3)
    inp = random_inputs("BNSD", 2, 4, 700, 900, 128, seed=11)
    a = run_cuda(kw, inp["q"], inp["k"], inp["v"])
    b = run_cuda(kw, inp["q"], inp["k"], inp["v"])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1], equal_nan=True)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", ["BNSD", "TND"])
def test_o_only_16_byte_aligned(layout, D):
    """O rows leave the SM in 32-byte stores when O is 32-byte aligned and in
    16-byte stores otherwise: an O that starts 16 bytes past a 32-byte
    boundary gets the same bits, and the guard elements on both sides of it
    stay untouched."""
    if layout == "TND":
        cu = [300, 700]
        kw = _kw("TND", 2, 2, 700, 700, D, 3)
        inp = random_inputs("TND", 2, 2, 700, 700, D, seed=93)
        shape = (700, 2, D)
        extra = dict(actual_seq_qlen=cu, actual_seq_kvlen=cu)
    else:
        kw = _kw("BNSD", 2, 2, 300, 333, D, 2)
        inp = random_inputs("BNSD", 2, 2, 300, 333, D, seed=93)
        shape = (2, 2, 300, D)
        extra = {}
    attn = fa.MaskedAttention(**kw)
    q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
    o_ref, l_ref = attn(q, k, v, **extra)
    n = int(np.prod(shape))
    raw = torch.full((n + 32,), -7.0, dtype=torch.bfloat16, device="cuda")
    assert raw.data_ptr() % 256 == 0
    o16 = raw[8:8 + n].view(shape)  # 16 bytes past a 256-byte boundary
    l16 = torch.empty_like(l_ref)
    attn(q, k, v, out=o16, lse=l16, **extra)
    torch.cuda.synchronize()
    attn.sync_status()
    attn.close()
    assert torch.equal(o16.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(l16.nan_to_num(0.0), l_ref.nan_to_num(0.0))
    assert bool((raw[:8] == -7.0).all()) and bool((raw[8 + n:] == -7.0).all())


def test_worked_split_examples_on_gpu():
    """Both cards of the sparseMode=7 and sparseMode=8 worked examples, each
    against the oracle, and their concatenation against the unsplit call."""
    N, D = 2, 64
    for unsplit, cards in (
        (dict(mode=3, cu_q=[3, 7, 12, 16], cu_k=[3, 9, 14, 18]),
         [dict(mode=7, pre=6, nxt=-2, cu_q=[3, 5], cu_k=[3, 9], q0=0, k0=0),
          dict(mode=3, pre=0, nxt=0, cu_q=[2, 7, 11], cu_k=[6, 11, 15], q0=5, k0=3)]),
        (dict(mode=2, cu_q=[3, 8, 13, 17], cu_k=[3, 7, 12, 16]),
         [dict(mode=2, pre=0, nxt=0, cu_q=[3, 5], cu_k=[3, 7], q0=0, k0=0),
          dict(mode=8, pre=4, nxt=1, cu_q=[3, 8, 12], cu_k=[4, 9, 13], q0=5, k0=3)]),
    ):
        Tq, Tk = unsplit["cu_q"][-1], unsplit["cu_k"][-1]
        inp = random_inputs("TND", 4, N, Tq, Tk, D, seed=31)
        kw = _kw("TND", 4, N, Tq, Tk, D, unsplit["mode"])
        o_full, lse_full = check_against_oracle(kw, inp, cu_q=unsplit["cu_q"],
                                                cu_kv=unsplit["cu_k"])
        parts_o, parts_l = [], []
        for c in cards:
            tq, tk = c["cu_q"][-1], c["cu_k"][-1]
            sub = {"q": inp["q"][c["q0"]:c["q0"] + tq], "k": inp["k"][c["k0"]:c["k0"] + tk],
                   "v": inp["v"][c["k0"]:c["k0"] + tk]}
            kwc = _kw("TND", len(c["cu_q"]), N, tq, tk, D, c["mode"], pre_tokens=c["pre"],
                      next_tokens=c["nxt"])
            o, l = check_against_oracle(kwc, sub, cu_q=c["cu_q"], cu_kv=c["cu_k"])
            parts_o.append(o)
            parts_l.append(l)
        np.testing.assert_allclose(np.concatenate(parts_o, 0), o_full, atol=2e-2)
        np.testing.assert_allclose(np.concatenate(parts_l, 1), lse_full, atol=1e-3)


def test_bad_pointer_alignment_and_nulls_are_rejected():
    attn = fa.MaskedAttention("BNSD", 1, 1, 64, 64, 64, 2)
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    raw = torch.zeros(64 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    mis = raw[1:1 + 64 * 64].view(1, 1, 64, 64)
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 64, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(attn.handle, mis, q, q, o, lse)
    assert e.value.name == "FA_ERR_PARAM_INVALID"
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(attn.handle, q, q, None, o, lse)
    assert e.value.name == "FA_ERR_NULLPTR"
    attn.close()
