"""GPU parity of the ALiBi bias ("压缩mask" page, alibi section: a per-head
coefficient times an alibi bias, on top of the mask geometry) against the
fp64 oracle: the right-aligned, square-root and left-aligned variants on
modes 0 (no mask: keys right of the diagonal get a positive bias), 2, 3, 4,
5, 7 and 8, in BNSD, BSND and TND, both head dims; the claimed-work
instance; and repeated calls giving the same bits."""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from masked_attention_fa_b200.workloads import alibi_slopes, random_inputs
from gpu_helpers import assert_close, problem_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()
    fa.load_library()


# (layout, mode, extra, B, N, Sq or lens_q, Skv or lens_kv, prefix)
CASES = [
    ("BNSD", 3, {}, 2, 3, 300, 333, None),
    ("BNSD", 2, {}, 1, 4, 333, 300, None),
    ("BSND", 4, dict(pre_tokens=100, next_tokens=20), 1, 3, 300, 700, None),
    ("BNSD", 5, {}, 2, 2, 300, 333, [40, 333]),
    ("BNSD", 0, {}, 1, 2, 200, 260, None),
    ("TND", 3, {}, 4, 3, [130, 0, 257, 5], [140, 3, 300, 5], None),
    ("TND", 7, dict(pre_tokens=300, next_tokens=-40), 3, 2, [100, 200, 0], [120, 260, 7], None),
    ("TND", 8, dict(pre_tokens=200, next_tokens=10), 3, 2, [0, 150, 300], [3, 190, 350], None),
]


def _run(kw, inp, slopes, prefix=None, cu_q=None, cu_kv=None):
    attn = fa.MaskedAttention(**kw)
    try:
        o, lse = attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), prefix=prefix,
                      actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv,
                      slopes=torch.tensor(slopes, dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    return o.float().cpu().double().numpy(), lse.cpu().double().numpy()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("kind", ["right", "sqrt", "left"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_alibi_matches_oracle(case, kind, D):
    layout, mode, extra, B, N, sq, skv, prefix = CASES[case]
    cu_q = cu_kv = None
    if layout == "TND":
        cu_q, cu_kv = np.cumsum(sq).tolist(), np.cumsum(skv).tolist()
        sq, skv = cu_q[-1], cu_kv[-1]
    kw = dict(layout=layout, B=B, N=N, Sq=sq, Skv=skv, D=D, sparse_mode=mode, alibi=kind,
              **extra)
    inp = random_inputs(layout, B, N, sq, skv, D, seed=3000 + case)
    slopes = alibi_slopes(N)
    o, lse = _run(kw, inp, slopes, prefix, cu_q, cu_kv)
    pkw = {k: v for k, v in kw.items() if k != "alibi"}
    o_ref, lse_ref = oracle.attention(problem_of(pkw, None, prefix, cu_q, cu_kv), inp["q"],
                                      inp["k"], inp["v"], alibi=kind, slopes=slopes)
    assert_close(o, lse, o_ref, lse_ref, f"{kind} {kw}")


def test_alibi_on_claimed_work_is_deterministic():
    """1,200 varlen sequences x 2 heads (2,400 items, enough to claim them at
    run time): against the oracle, and the same bits on a second call."""
    g = torch.Generator().manual_seed(3100)
    nseq = 1200
    sq = torch.randint(1, 200, (nseq,), generator=g)
    skv = sq + torch.randint(0, 60, (nseq,), generator=g)
    cu_q, cu_kv = torch.cumsum(sq, 0).tolist(), torch.cumsum(skv, 0).tolist()
    N, D = 2, 128
    kw = dict(layout="TND", B=nseq, N=N, Sq=cu_q[-1], Skv=cu_kv[-1], D=D, sparse_mode=3,
              alibi="right")
    items = fa.fa_plan_stats(fa.make_desc(**kw), actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)[0]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert items >= fa.CLAIM_MIN_ITEMS_PER_CTA * sms
    inp = random_inputs("TND", nseq, N, cu_q[-1], cu_kv[-1], D, seed=3101)
    slopes = [0.7, 0.03]
    a = _run(kw, inp, slopes, None, cu_q, cu_kv)
    b = _run(kw, inp, slopes, None, cu_q, cu_kv)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    pkw = {k: v for k, v in kw.items() if k != "alibi"}
    o_ref, lse_ref = oracle.attention(problem_of(pkw, None, None, cu_q, cu_kv), inp["q"],
                                      inp["k"], inp["v"], alibi="right", slopes=slopes)
    assert_close(a[0], a[1], o_ref, lse_ref, "claimed ALiBi")


@pytest.mark.parametrize("kind", ["right", "left", "sqrt"])
def test_alibi_claimed_long_items_sampled_rows(kind):
    """Claimed ALiBi work whose items span up to 9 key tiles, so that the
    claim, the Q releases and the last V of the descending walk fall in the
    middle of long items: 260 varlen sequences of 500-1100 query rows x 4
    heads (about 3,700 items), slopes from steep to flat; 600 sampled rows
    against the oracle row by row, and the same bits on a second call."""
    g = torch.Generator().manual_seed(3200)
    nseq = 260
    sq = torch.randint(500, 1101, (nseq,), generator=g)
    skv = sq + torch.randint(0, 100, (nseq,), generator=g)
    cu_q, cu_kv = torch.cumsum(sq, 0).tolist(), torch.cumsum(skv, 0).tolist()
    N, D = 4, 128
    kw = dict(layout="TND", B=nseq, N=N, Sq=cu_q[-1], Skv=cu_kv[-1], D=D, sparse_mode=3,
              alibi=kind)
    items = fa.fa_plan_stats(fa.make_desc(**kw), actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)[0]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert items >= fa.CLAIM_MIN_ITEMS_PER_CTA * sms
    inp = random_inputs("TND", nseq, N, cu_q[-1], cu_kv[-1], D, seed=3201)
    slopes = [0.71, 0.125, 0.02, 0.0039]
    a = _run(kw, inp, slopes, None, cu_q, cu_kv)
    b = _run(kw, inp, slopes, None, cu_q, cu_kv)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    pkw = {k_: v_ for k_, v_ in kw.items() if k_ != "alibi"}
    pb = problem_of(pkw, None, None, cu_q, cu_kv)
    gr = np.random.default_rng(3202)
    q_off = [0] + cu_q[:-1]
    rows = []  # (sequence, head, row inside the sequence)
    for b, h in zip(gr.integers(0, nseq, 600), gr.integers(0, N, 600)):
        rows.append((int(b), int(h), int(gr.integers(0, int(sq[b])))))
    o_ref, l_ref = oracle.attention_rows(pb, inp["q"], inp["k"], inp["v"], rows, alibi=kind,
                                         slopes=slopes)
    o_got = np.stack([a[0][q_off[b] + i, h] for b, h, i in rows])
    l_got = np.array([a[1][h, q_off[b] + i] for b, h, i in rows])
    assert_close(o_got, l_got, o_ref, l_ref, f"claimed ALiBi ({kind}), long items")


def test_alibi_left_equals_right_in_o():
    """Left- and right-aligned biases give the same weights: equal O bits up
    to the last rounding (the kernel computes both through the same
    right-aligned scores), lse apart by slope * (i + Skv - Sq)."""
    kw = dict(layout="BNSD", B=1, N=2, Sq=256, Skv=384, D=128, sparse_mode=3)
    inp = random_inputs("BNSD", 1, 2, 256, 384, 128, seed=3200)
    slopes = [0.25, 0.0625]
    o_r, l_r = _run(dict(kw, alibi="right"), inp, slopes)
    o_l, l_l = _run(dict(kw, alibi="left"), inp, slopes)
    assert np.array_equal(o_r, o_l)
    for h, s in enumerate(slopes):
        np.testing.assert_allclose(l_l[0, h] - l_r[0, h], s * (np.arange(256) + 128), atol=1e-3)
