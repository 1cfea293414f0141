"""GPU parity of the paged K/V forward (decode-shaped calls).

Keys and values sit in paged caches [num_blocks, block_size, N, D] (the
"Norm" cache of the aclnnScatterPaKvCache page) in a shuffled block order;
cache slots that belong to no sequence hold NaN, so any read outside a
sequence's keys shows up in O. Every case is compared with the fp64 paged
oracle element by element at the kernel's tolerances.
"""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from oracle import Problem
from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()
    assert torch.cuda.is_available()
    fa.load_library()


def paged_case(lens_q, lens_kv, N, D, bs, seed, spare=5):
    """Packed q and paged caches (random block order, NaN in unused slots)."""
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    cu_q, cu_kv = np.cumsum(lens_q).tolist(), np.cumsum(lens_kv).tolist()
    q = torch.randn(cu_q[-1], N, D, generator=g).to(torch.bfloat16)
    nblk = [-(-n // bs) for n in lens_kv]
    total = sum(nblk) + spare
    order = rng.permutation(total)
    kc = torch.full((total, bs, N, D), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((total, bs, N, D), float("nan"), dtype=torch.bfloat16)
    table = torch.full((len(lens_kv), max(max(nblk), 1)), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(lens_kv):
        kb = torch.randn(n, N, D, generator=g).to(torch.bfloat16)
        vb = torch.randn(n, N, D, generator=g).to(torch.bfloat16)
        for c in range(nblk[b]):
            blk = int(order[nxt]); nxt += 1
            table[b, c] = blk
            r = slice(c * bs, min((c + 1) * bs, n))
            kc[blk, :r.stop - r.start] = kb[r]
            vc[blk, :r.stop - r.start] = vb[r]
    return cu_q, cu_kv, q, kc, vc, table


def run_paged(mode, extra, cu_q, cu_kv, q, kc, vc, table, N, D, prefix=None):
    B = len(cu_q)
    attn = fa.MaskedAttention("TND", B, N, cu_q[-1], cu_kv[-1], D, mode, **extra)
    try:
        o, lse = attn.paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), cu_q, cu_kv,
                            prefix=prefix)
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    return o.float().cpu().double().numpy(), lse.cpu().double().numpy()


def oracle_paged(mode, extra, cu_q, cu_kv, q, kc, vc, table, N, D, bs, prefix=None):
    pb = Problem("TND", len(cu_q), N, cu_q[-1], cu_kv[-1], D, sparse_mode=mode,
                 actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv, prefix=prefix, **extra)
    return oracle.attention_paged(pb, q, kc, vc, table.numpy(), bs)


CASES = [
    # mode, extra, lens_q, lens_kv, block size
    (3, {}, [1, 1, 1, 1], [300, 1, 777, 128], 16),           # decode
    (3, {}, [1, 3, 5, 9], [64, 200, 129, 1000], 64),          # a few rows, several row groups
    (3, {}, [2, 0, 1], [5, 40, 0], 128),                      # empty query / key sets
    (2, {}, [4, 7], [4, 300], 32),
    (0, {}, [3, 1], [250, 17], 16),                           # no mask: every key
    (4, dict(pre_tokens=100, next_tokens=0), [1, 6], [900, 333], 64),   # sliding window
    (5, {}, [2, 5], [400, 70], 16),                           # prefix
    (7, dict(pre_tokens=600, next_tokens=-1), [1, 2], [500, 600], 128),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_paged_matches_oracle(case, D):
    mode, extra, lq, lkv, bs = CASES[case]
    N = 4
    prefix = [37, 5] if mode == 5 else None
    cu_q, cu_kv, q, kc, vc, table = paged_case(lq, lkv, N, D, bs, seed=300 + case)
    o, lse = run_paged(mode, extra, cu_q, cu_kv, q, kc, vc, table, N, D, prefix)
    o_ref, lse_ref = oracle_paged(mode, extra, cu_q, cu_kv, q, kc, vc, table, N, D, bs, prefix)
    assert_close(o, lse, o_ref, lse_ref, what=f"paged case {case}")


def test_paged_long_context_is_split_and_deterministic():
    """Contexts long enough to be cut into several key chunks per row: the
    merge in chunk order gives the same bits on every run."""
    N, D, bs = 8, 128, 128
    cu_q, cu_kv, q, kc, vc, table = paged_case([1, 2, 1], [20000, 9000, 33000], N, D, bs, 41)
    a = run_paged(3, {}, cu_q, cu_kv, q, kc, vc, table, N, D)
    b = run_paged(3, {}, cu_q, cu_kv, q, kc, vc, table, N, D)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    o_ref, lse_ref = oracle_paged(3, {}, cu_q, cu_kv, q, kc, vc, table, N, D, bs)
    assert_close(a[0], a[1], o_ref, lse_ref, what="long context")


def test_paged_bad_block_id_is_reported_not_read():
    """A block-table entry outside [0, num_blocks) is never dereferenced:
    its keys are left out and fa_sync_status reports FA_ERR_DEVICE; the next
    call on a good table is exact again."""
    N, D, bs = 2, 64, 16
    cu_q, cu_kv, q, kc, vc, table = paged_case([1, 1], [40, 40], N, D, bs, 51)
    bad = table.clone()
    bad[1, 1] = kc.shape[0] + 1000
    attn = fa.MaskedAttention("TND", 2, N, cu_q[-1], cu_kv[-1], D, 3)
    try:
        attn.paged(q.cuda(), kc.cuda(), vc.cuda(), bad.cuda(), cu_q, cu_kv)
        torch.cuda.synchronize()
        with pytest.raises(fa.FaError) as e:
            attn.sync_status()
        assert e.value.status == 8 and "block_table" in str(e.value)
        o, lse = attn.paged(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), cu_q, cu_kv)
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    o_ref, lse_ref = oracle_paged(3, {}, cu_q, cu_kv, q, kc, vc, table, N, D, bs)
    assert_close(o.float().cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, lse_ref)


def test_paged_rejects_bad_arguments_before_device_work():
    N, D = 2, 64
    cu_q, cu_kv, q, kc, vc, table = paged_case([1], [40], N, D, 16, 61)
    bsnd = fa.MaskedAttention("BSND", 1, N, 1, 40, D, 3)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_paged(bsnd.handle, q.cuda(), kc.cuda(), vc.cuda(), table.cuda(),
                        torch.empty(1, N, D, dtype=torch.bfloat16, device="cuda"),
                        torch.empty(N, 1, device="cuda"), cu_q, cu_kv)
    assert e.value.name == "FA_ERR_UNSUPPORTED"
    bsnd.close()
    attn = fa.MaskedAttention("TND", 1, N, 1, 40, D, 3)
    short = table[:, :1].contiguous()  # 40 keys need 3 blocks of 16
    with pytest.raises(fa.FaError) as e:
        attn.paged(q.cuda(), kc.cuda(), vc.cuda(), short.cuda(), cu_q, cu_kv)
    assert e.value.name == "FA_ERR_SHAPE"
    attn.close()


def test_paged_decode_workload_full_size_sampled():
    """The bench's decode workload (16 sequences, 32 heads, 4k-16k cached
    keys in 128-token blocks, caches drawn on the device) through the call
    the bench times: sampled (sequence, head) rows against the paged oracle,
    with the keys of that sequence and head gathered to the host; and two
    runs give the same bits."""
    from masked_attention_fa_b200.workloads import make_inputs, named_workloads
    w = named_workloads()["paged_decode_16k"]
    inp = make_inputs(w, device="cuda")
    q, kc, vc, table = (inp[x] for x in ("q", "k_cache", "v_cache", "block_table"))
    attn = fa.MaskedAttention("TND", w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode)
    try:
        o1, l1 = attn.paged(q, kc, vc, table, w.actual_seq_qlen, w.actual_seq_kvlen)
        o2, l2 = attn.paged(q, kc, vc, table, w.actual_seq_qlen, w.actual_seq_kvlen)
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    lens = w.seq_lens()
    rng = np.random.default_rng(9)
    for b in sorted({0, w.B - 1, int(rng.integers(0, w.B))}):
        sq, skv = lens[b]
        nblk = -(-skv // w.block_size)
        blocks = table[b, :nblk].long()
        for h in sorted({0, w.N - 1, int(rng.integers(0, w.N))}):
            kb = kc[blocks][:, :, h:h + 1].cpu()
            vb = vc[blocks][:, :, h:h + 1].cpu()
            q0 = w.actual_seq_qlen[b - 1] if b else 0
            qb = q[q0:q0 + sq, h:h + 1].cpu()
            pb = Problem("TND", 1, 1, sq, skv, w.D, sparse_mode=w.sparse_mode, scale=w.scale,
                         actual_seq_qlen=[sq], actual_seq_kvlen=[skv])
            o_ref, l_ref = oracle.attention_paged(pb, qb, kb, vb,
                                                  np.arange(nblk, dtype=np.int32)[None],
                                                  w.block_size)
            got = o1[q0:q0 + sq, h:h + 1].float().cpu().double().numpy()
            gl = l1[h:h + 1, q0:q0 + sq].cpu().double().numpy()
            assert_close(got, gl, o_ref, l_ref, what=f"sequence {b} head {h}")
