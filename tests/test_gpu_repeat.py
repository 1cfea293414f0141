"""Repeated calls: one handle (and the allocation-free entry point) called
again and again with its outputs poisoned (NaN) before every call. Every call
must write every row, with the same bits as the first call, which is compared
with the oracle: the work list, its per-item tile ranges and the dense-mask
pre-pass's scratch live in device memory that each call reuses, so a stale
entry or an item left out would show as unwritten rows or changed bits. The
lists mix items of many lengths, items whose second sub-tile is empty or
ragged, and items without a key tile (they sort last and are still written:
O = 0, lse = -inf)."""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from gpu_helpers import assert_close, problem_of

pytestmark = pytest.mark.gpu

CALLS = 6


def _poisoned(shape, dtype):
    return torch.full(shape, float("nan"), dtype=dtype, device="cuda")


def _check_repeat(run, o, lse, first):
    for _ in range(CALLS):
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        run()
        torch.cuda.synchronize()
        assert not torch.isnan(o).any() and not torch.isnan(lse).any(), "rows left unwritten"
        if first is None:
            first = (o.clone(), lse.clone())
        else:
            assert torch.equal(o, first[0]) and torch.equal(lse, first[1]), "calls differ"
    return first


def _varlen_case():
    # 400 sequences of 0-299 query rows: 1-2 items per sequence and head,
    # many with an empty or ragged second sub-tile; some without keys.
    rng = np.random.default_rng(91)
    B, N, D = 400, 4, 64
    lq = rng.integers(0, 300, size=B)
    lk = lq + rng.integers(0, 200, size=B)
    lq[[3, 17, 250]] = 0                  # sequences without query rows (no items)
    lk[[5, 22, 31, 123, 399]] = 0         # rows without any key: items without a key tile
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    g = torch.Generator().manual_seed(91)
    q = torch.randn(cu_q[-1], N, D, generator=g).to(torch.bfloat16)
    k = torch.randn(cu_k[-1], N, D, generator=g).to(torch.bfloat16)
    v = torch.randn(cu_k[-1], N, D, generator=g).to(torch.bfloat16)
    kw = dict(layout="TND", B=B, N=N, Sq=cu_q[-1], Skv=cu_k[-1], D=D, sparse_mode=3)
    return kw, q, k, v, cu_q, cu_k


def test_varlen_every_call_writes_every_row():
    kw, q, k, v, cu_q, cu_k = _varlen_case()
    attn = fa.MaskedAttention(**kw)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o = _poisoned((kw["Sq"], kw["N"], kw["D"]), torch.bfloat16)
    lse = _poisoned((kw["N"], kw["Sq"]), torch.float32)
    try:
        def run():
            attn(qc, kc, vc, out=o, lse=lse, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
            torch.cuda.synchronize()
            attn.sync_status()
        first = _check_repeat(run, o, lse, None)
    finally:
        attn.close()
    o_ref, l_ref = oracle.attention(problem_of(kw, cu_q=cu_q, cu_kv=cu_k), q, k, v)
    assert_close(first[0].float().cpu().double().numpy(), first[1].cpu().double().numpy(),
                 o_ref, l_ref, "repeated varlen")
    # The allocation-free entry point rebuilds its list in its own array on
    # every call: the same bits, call after call.
    desc = fa.make_desc(**kw)
    _check_repeat(lambda: fa.fa_fwd_noalloc(desc, qc, kc, vc, o, lse, actual_seq_qlen=cu_q,
                                            actual_seq_kvlen=cu_k), o, lse, first)


def test_dense_mask_every_call_writes_every_row():
    # 320 heads x 4 row blocks over one SS mask that hides whole 128-row
    # sub-tiles (items without a key tile once the pre-pass has reduced it)
    # and leaves others ragged; sampled heads against the oracle.
    B, N, S, D = 1, 320, 1024, 64
    g = torch.Generator().manual_seed(92)
    q = torch.randn(B, N, S, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, N, S, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, N, S, D, generator=g).to(torch.bfloat16)
    mask = torch.triu(torch.ones(S, S, dtype=torch.uint8), diagonal=1)
    mask[256:512, :] = 1                   # rows 256-511 see nothing
    mask[768:, 100:700] = 1                # a hole in the visible band
    attn = fa.MaskedAttention("BNSD", B, N, S, S, D, 1, mask_kind="SS")
    qc, kc, vc, mc = q.cuda(), k.cuda(), v.cuda(), mask.cuda()
    o = _poisoned((B, N, S, D), torch.bfloat16)
    lse = _poisoned((B, N, S), torch.float32)
    try:
        def run():
            attn(qc, kc, vc, atten_mask=mc, out=o, lse=lse)
            torch.cuda.synchronize()
            attn.sync_status()
        first = _check_repeat(run, o, lse, None)
    finally:
        attn.close()
    kw1 = dict(layout="BNSD", B=1, N=1, Sq=S, Skv=S, D=D, sparse_mode=1, mask_kind="SS")
    for h in (0, 161, 319):
        sl = slice(h, h + 1)
        o_ref, l_ref = oracle.attention(problem_of(kw1, mask=mask), q[:, sl].contiguous(),
                                        k[:, sl].contiguous(), v[:, sl].contiguous())
        assert_close(first[0][:, sl].float().cpu().double().numpy(),
                     first[1][:, sl].cpu().double().numpy(), o_ref, l_ref, f"repeated dense head {h}")
