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
