"""fa_fwd_noalloc, the forward for callers that cannot allocate, against fa_fwd.

Some callers cannot let a library call cudaMalloc: code running under a
framework that owns every device allocation through its own pool, real-time
loops that must not allocate once started, or plugins invoked from another
library's memory callbacks. fa_fwd_noalloc serves them by keeping its work
list in a fixed device array inside the library instead of a workspace it
allocates. These tests call it through the C ABI twice in a row, on two
different problems, and compare each result with the handle-based fa_fwd on
the same inputs, within the tolerances of the other parity tests. The file
is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
from masked_attention_fa_b200.workloads import random_inputs
from gpu_helpers import TOL_LSE, TOL_MAX_O, TOL_MEAN_O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()
    fa.load_library()


def _desc_kw(c):
    return {k: c[k] for k in ("layout", "B", "N", "Sq", "Skv", "D", "sparse_mode",
                              "pre_tokens", "next_tokens") if k in c}


def _arrays(c):
    return {k: c[k] for k in ("prefix", "actual_seq_qlen", "actual_seq_kvlen") if k in c}


def _with_handle(c, q, k, v):
    attn = fa.MaskedAttention(**_desc_kw(c))
    try:
        o, lse = attn(q, k, v, **_arrays(c))
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    return o, lse


def _without_alloc(c, q, k, v):
    attn_shapes = fa.MaskedAttention(**_desc_kw(c))
    oshape, lshape = attn_shapes.out_shapes()
    attn_shapes.close()
    o = torch.full(oshape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(lshape, float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_fwd_noalloc(fa.make_desc(**_desc_kw(c)), q, k, v, o, lse, **_arrays(c))
    torch.cuda.synchronize()
    return o, lse


def _compare(a, b, what):
    oa, la = a[0].float().cpu().double().numpy(), a[1].cpu().double().numpy()
    ob, lb = b[0].float().cpu().double().numpy(), b[1].cpu().double().numpy()
    assert np.all(np.isfinite(ob)), what
    d = np.abs(oa - ob)
    assert d.max() <= TOL_MAX_O and d.mean() <= TOL_MEAN_O, (what, d.max(), d.mean())
    assert np.array_equal(np.isneginf(la), np.isneginf(lb)), what
    live = ~np.isneginf(la)
    assert np.abs(la[live] - lb[live]).max() <= TOL_LSE, what


CASES = [
    dict(layout="BNSD", B=2, N=3, Sq=600, Skv=700, D=128, sparse_mode=3),
    dict(layout="TND", B=3, N=2, Sq=420, Skv=550, D=64, sparse_mode=7, pre_tokens=400,
         next_tokens=-20, actual_seq_qlen=[100, 100, 420], actual_seq_kvlen=[150, 170, 550]),
]


def test_noalloc_matches_fa_fwd_on_two_calls_in_a_row():
    tensors = []
    for i, c in enumerate(CASES):
        inp = random_inputs(c["layout"], c["B"], c["N"], c["Sq"], c["Skv"], c["D"], seed=90 + i,
                            device="cuda")
        tensors.append((inp["q"], inp["k"], inp["v"]))
    refs = [_with_handle(c, *t) for c, t in zip(CASES, tensors)]
    # two calls in a row on different problems, then the first one again:
    # each call must not depend on what the previous call left in the array
    for idx in (0, 1, 0):
        got = _without_alloc(CASES[idx], *tensors[idx])
        _compare(refs[idx], got, f"case {idx}")


def test_noalloc_rejects_a_work_list_beyond_its_array():
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(16, dtype=torch.float32, device="cuda")
    desc = fa.make_desc("BNSD", 1, 4096, 65536, 65536, 128, 2)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_noalloc(desc, t, t, t, t, lse)
    assert e.value.name == "FA_ERR_UNSUPPORTED" and "fixed device array" in str(e.value)


def _oracle_compare(c, q, k, v, got, mask=None):
    import oracle
    from gpu_helpers import assert_close, problem_of
    pb_kw = {x: c[x] for x in ("layout", "B", "N", "Sq", "Skv", "D", "sparse_mode",
                               "pre_tokens", "next_tokens") if x in c}
    a = _arrays(c)
    pb = problem_of(pb_kw, mask, a.get("prefix"), a.get("actual_seq_qlen"),
                    a.get("actual_seq_kvlen"))
    o_ref, lse_ref = oracle.attention(pb, q.cpu(), k.cpu(), v.cpu())
    assert_close(got[0].float().cpu().double().numpy(), got[1].cpu().double().numpy(),
                 o_ref, lse_ref, "noalloc vs oracle")


def test_noalloc_matches_the_oracle():
    """The allocation-free result against the fp64 oracle directly, on both
    problems of the two-call test."""
    for i, c in enumerate(CASES):
        inp = random_inputs(c["layout"], c["B"], c["N"], c["Sq"], c["Skv"], c["D"], seed=90 + i,
                            device="cuda")
        got = _without_alloc(c, inp["q"], inp["k"], inp["v"])
        fa.fa_noalloc_sync_status()
        _oracle_compare(c, inp["q"], inp["k"], inp["v"], got)


def test_noalloc_without_room_for_item_ranges():
    """3,000 short varlen sequences x 8 heads: the 24,000-item work list fits
    the fixed array but the per-item key-tile ranges do not, so the kernel
    derives each item's ranges from its sequence record (the instance only
    this situation reaches). Bit for bit equal to fa_fwd, which reads the
    ranges from its workspace, and within the parity bar of the oracle."""
    g = torch.Generator().manual_seed(404)
    nseq = 3000
    sq = torch.randint(1, 41, (nseq,), generator=g)
    skv = sq + torch.randint(0, 21, (nseq,), generator=g)
    cu_q, cu_kv = torch.cumsum(sq, 0).tolist(), torch.cumsum(skv, 0).tolist()
    c = dict(layout="TND", B=nseq, N=8, Sq=cu_q[-1], Skv=cu_kv[-1], D=64, sparse_mode=3,
             actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)
    n_items = nseq * 8
    need = 256 + (32 * nseq + 255) // 256 * 256 + 16 * n_items
    assert need <= (1 << 20) < (need + 255) // 256 * 256 + 32 * n_items
    inp = random_inputs("TND", nseq, 8, cu_q[-1], cu_kv[-1], 64, seed=405, device="cuda")
    ref = _with_handle(c, inp["q"], inp["k"], inp["v"])
    for _ in range(2):
        got = _without_alloc(c, inp["q"], inp["k"], inp["v"])
        fa.fa_noalloc_sync_status()
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1].nan_to_num(), ref[1].nan_to_num())
    _oracle_compare(c, inp["q"], inp["k"], inp["v"], got)


def test_noalloc_dense_mask_without_room_for_the_prepass():
    """A BNSS allMask over 64 x 256 planes of 128 x 128: the work list fits,
    the occupancy pre-pass's scratch does not, so the call runs without the
    pre-pass (every tile of the band with the element mask, the kernel
    deriving its ranges from the sequence record). Against fa_fwd (which
    runs the pre-pass) and, on sampled planes, against the oracle."""
    B, N, S, D = 64, 256, 128, 64
    planes = B * N
    need = 256 + (32 * B + 255) // 256 * 256 + 16 * planes
    occ = (need + 255) // 256 * 256 + 32 * planes + 16 * planes + planes
    assert need <= (1 << 20) < occ
    dg = torch.Generator(device="cuda").manual_seed(406)
    q, k, v = (torch.randn((B, N, S, D), generator=dg, device="cuda").to(torch.bfloat16)
               for _ in range(3))
    mask = (torch.rand((B, N, S, S), generator=dg, device="cuda") < 0.4).to(torch.uint8)
    mask[:, :, 5, :] = 1                                   # a row with no visible key
    mask[:7, :, :, 64:] = 1                                # half-hidden tiles
    c = dict(layout="BNSD", B=B, N=N, Sq=S, Skv=S, D=D, sparse_mode=1)
    attn = fa.MaskedAttention(**c, mask_kind="BNSS")
    try:
        ref = attn(q, k, v, atten_mask=mask)
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, N, S), float("nan"), device="cuda")
    fa.fa_fwd_noalloc(fa.make_desc(**c, mask_kind="BNSS"), q, k, v, o, lse, atten_mask=mask)
    fa.fa_noalloc_sync_status()
    _compare((ref[0], ref[1]), (o, lse), "dense fallback vs fa_fwd")
    import oracle
    from gpu_helpers import assert_close, problem_of
    sel = torch.randperm(planes, generator=torch.Generator().manual_seed(407))[:24].tolist()
    for pl in sel + [0, planes - 1]:
        b, h = divmod(pl, N)
        kw = dict(layout="BNSD", B=1, N=1, Sq=S, Skv=S, D=D, sparse_mode=1, mask_kind="SS")
        pb = problem_of(kw, mask[b, h].cpu())
        o_ref, l_ref = oracle.attention(pb, q[b:b + 1, h:h + 1].cpu(), k[b:b + 1, h:h + 1].cpu(),
                                        v[b:b + 1, h:h + 1].cpu())
        assert_close(o[b:b + 1, h:h + 1].float().cpu().double().numpy(),
                     lse[b:b + 1, h:h + 1].cpu().double().numpy(), o_ref, l_ref, f"plane {pl}")


def test_noalloc_refuses_stream_capture():
    """A replayed capture would re-read the one static host image after later
    calls rewrote it, so a call on a capturing stream is refused (nothing is
    enqueued and the capture stays valid); outside capture it runs."""
    c = CASES[0]
    inp = random_inputs(c["layout"], c["B"], c["N"], c["Sq"], c["Skv"], c["D"], seed=90,
                        device="cuda")
    o, lse = _without_alloc(c, inp["q"], inp["k"], inp["v"])   # set-up happens outside capture
    desc = fa.make_desc(**_desc_kw(c))
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with pytest.raises(fa.FaError) as e:
        with torch.cuda.graph(g, stream=s, capture_error_mode="relaxed"):
            fa.fa_fwd_noalloc(desc, inp["q"], inp["k"], inp["v"], o, lse, stream=s)
    assert e.value.name == "FA_ERR_UNSUPPORTED" and "captured" in str(e.value)
    del g
    torch.cuda.synchronize()
    again = _without_alloc(c, inp["q"], inp["k"], inp["v"])
    fa.fa_noalloc_sync_status()
    assert torch.equal(again[0], o) and torch.equal(again[1], lse)
