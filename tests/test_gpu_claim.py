"""Claimed work: a closed-form call whose work list holds at least 8 items
per CTA runs the kernel instance in which each CTA starts on one item and
then takes the next unclaimed position of the longest-first list from a
counter in device memory (the handle's workspace, or the allocation-free
array), which the last CTA of every launch sets back to 0.

A counter left non-zero would make the next call skip the first items of the
list, and an item claimed twice or not at all would leave rows unwritten. So
each path is called repeatedly with its outputs poisoned (NaN) before every
call: every call must write every row, with the same bits as the first call,
which is compared with the oracle. Items without a key tile sort last; a CTA
that claims many of them in a row must still finish its last real item
(its last V tile is loaded when the first of them is claimed)."""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from gpu_helpers import assert_close, problem_of

pytestmark = pytest.mark.gpu

CALLS = 6


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


def _run_case(lq, lk, N, D, seed, what):
    B = len(lq)
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    n_items = N * sum((int(x) + 255) // 256 for x in lq)
    assert n_items >= fa.CLAIM_MIN_ITEMS_PER_CTA * \
        torch.cuda.get_device_properties(0).multi_processor_count, "too few items to claim"
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(cu_q[-1], N, D, generator=g).to(torch.bfloat16)
    k = torch.randn(max(cu_k[-1], 1), N, D, generator=g).to(torch.bfloat16)[:cu_k[-1]]
    v = torch.randn(max(cu_k[-1], 1), N, D, generator=g).to(torch.bfloat16)[:cu_k[-1]]
    kw = dict(layout="TND", B=B, N=N, Sq=cu_q[-1], Skv=cu_k[-1], D=D, sparse_mode=3)
    qc, kc, vc = q.cuda(), k.contiguous().cuda(), v.contiguous().cuda()
    o = torch.empty(cu_q[-1], N, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(N, cu_q[-1], dtype=torch.float32, device="cuda")
    attn = fa.MaskedAttention(**kw)
    try:
        def run():
            attn(qc, kc, vc, out=o, lse=lse, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
            torch.cuda.synchronize()
            attn.sync_status()
        first = _check_repeat(run, o, lse, None)
    finally:
        attn.close()
    o_ref, l_ref = oracle.attention(problem_of(kw, cu_q=cu_q, cu_kv=cu_k), q,
                                    k.contiguous(), v.contiguous())
    assert_close(first[0].float().cpu().double().numpy(), first[1].cpu().double().numpy(),
                 o_ref, l_ref, what)
    # The allocation-free entry point claims through the counters in its own
    # array's header: the same bits, call after call.
    desc = fa.make_desc(**kw)
    _check_repeat(lambda: fa.fa_fwd_noalloc(desc, qc, kc, vc, o, lse, actual_seq_qlen=cu_q,
                                            actual_seq_kvlen=cu_k), o, lse, first)


def test_varlen_claims_every_item_once_per_call():
    # 400 sequences of 0-299 query rows: 1-2 items per sequence and head,
    # many with an empty or ragged second sub-tile; a few without keys.
    rng = np.random.default_rng(91)
    lq = rng.integers(0, 300, size=400)
    lk = lq + rng.integers(0, 200, size=400)
    lq[[3, 17, 250]] = 0
    lk[[5, 22, 31, 123, 399]] = 0
    _run_case(lq, lk, N=4, D=64, seed=91, what="claimed varlen")


def test_claims_through_a_long_tail_of_items_without_keys():
    # Half of the sequences have query rows but no key at all: ~1,200 items
    # without a key tile at the end of the list, so CTAs claim long runs of
    # them after their last real item.
    rng = np.random.default_rng(93)
    lq = rng.integers(1, 256, size=600)
    lk = lq + rng.integers(0, 300, size=600)
    lk[1::2] = 0
    _run_case(lq, lk, N=4, D=128, seed=93, what="claimed, long empty tail")
