"""The multi-card query split of the sparseMode page (sparseMode=7 and
sparseMode=8 sections): queries cut across devices, keys/values kept whole,
each part an independent call.

- fa_split_queries reproduces both of the page's worked examples exactly;
- any split, run part by part through the fp64 oracle, reassembles the
  unsplit result bit for bit;
- two gloo ranks (world size 2, CPU) each run their own part and gather.
"""
import json
import os

import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from oracle import Problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "split_examples.json")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()


def _desc(mode, cu_q, cu_k, N=2, D=64):
    return fa.make_desc("TND", len(cu_q), N, cu_q[-1], cu_k[-1], D, mode)


@pytest.mark.parametrize("example,cu_q,cu_k", [
    ("mode7", [3, 7, 12, 16], [3, 9, 14, 18]),
    ("mode8", [3, 8, 13, 17], [3, 7, 12, 16]),
])
def test_split_reproduces_the_worked_examples(example, cu_q, cu_k):
    with open(GOLDEN) as f:
        g = json.load(f)[example]
    d = _desc(g["unsplit_mode"], cu_q, cu_k)
    for part, card in enumerate(("card1", "card2")):
        r = fa.fa_split_queries(d, cu_q, cu_k, 2, part, cuts=[5])
        c = g[card]
        assert r["desc"].sparse_mode == c["sparse_mode"]
        assert r["actual_seq_qlen"] == c["actual_seq_qlen"]
        assert r["actual_seq_kvlen"] == c["actual_seq_kvlen"]
        if "pre_tokens" in c:
            assert r["desc"].pre_tokens == c["pre_tokens"]
            assert r["desc"].next_tokens == c["next_tokens"]
    # the key ranges: card 1 starts at key 0, card 2 at the second sequence's keys
    assert fa.fa_split_queries(d, cu_q, cu_k, 2, 1, cuts=[5])["kv_begin"] == 3


def _run_part_oracle(r, q, k, v):
    pd = r["desc"]
    if pd.Sq == 0:
        return np.zeros((0,) + q.shape[1:]), np.zeros((q.shape[1], 0))
    pb = Problem("TND", pd.B, pd.N, pd.Sq, pd.Skv, q.shape[-1], sparse_mode=pd.sparse_mode,
                 pre_tokens=pd.pre_tokens, next_tokens=pd.next_tokens,
                 actual_seq_qlen=r["actual_seq_qlen"], actual_seq_kvlen=r["actual_seq_kvlen"])
    return oracle.attention(pb, q[r["q_begin"]:r["q_end"]], k[r["kv_begin"]:r["kv_end"]],
                            v[r["kv_begin"]:r["kv_end"]])


@pytest.mark.parametrize("mode", [2, 3])
@pytest.mark.parametrize("n_parts", [2, 3, 5])
def test_any_split_reassembles_the_unsplit_result(mode, n_parts):
    rng = np.random.default_rng(7 * n_parts + mode)
    lq = rng.integers(0, 40, size=5)
    lk = lq + rng.integers(0, 20, size=5)
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    N, D = 2, 8
    g = torch.Generator().manual_seed(3)
    q = torch.randn(cu_q[-1], N, D, generator=g, dtype=torch.float64)
    k = torch.randn(cu_k[-1], N, D, generator=g, dtype=torch.float64)
    v = torch.randn(cu_k[-1], N, D, generator=g, dtype=torch.float64)
    full = Problem("TND", 5, N, cu_q[-1], cu_k[-1], D, sparse_mode=mode,
                   actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
    o_ref, l_ref = oracle.attention(full, q, k, v)
    d = _desc(mode, cu_q, cu_k, N, 64)
    for cuts in (None, sorted(rng.integers(0, cu_q[-1] + 1, size=n_parts - 1).tolist())):
        os_, ls_, cover = [], [], 0
        for part in range(n_parts):
            r = fa.fa_split_queries(d, cu_q, cu_k, n_parts, part, cuts=cuts)
            assert r["q_begin"] == cover
            cover = r["q_end"]
            o, l = _run_part_oracle(r, q, k, v)
            os_.append(o)
            ls_.append(l)
        assert cover == cu_q[-1]
        np.testing.assert_array_equal(np.concatenate(os_, 0), o_ref)
        np.testing.assert_array_equal(np.concatenate(ls_, 1), l_ref)


def test_balanced_split_evens_the_visible_pairs():
    cu_q, cu_k = [4096], [4096]
    d = _desc(3, cu_q, cu_k)
    pairs = []
    for part in range(4):
        r = fa.fa_split_queries(d, cu_q, cu_k, 4, part)
        pairs.append(fa.fa_visible_pairs(r["desc"], actual_seq_qlen=r["actual_seq_qlen"],
                                         actual_seq_kvlen=r["actual_seq_kvlen"]))
    assert sum(pairs) == 2 * 4096 * 4097 // 2
    assert max(pairs) - min(pairs) <= 2 * 4096 * 2


def test_split_rejects_what_the_pages_exclude():
    with pytest.raises(fa.FaError):   # rightDownCausal with Sq > Skv in a sequence
        fa.fa_split_queries(_desc(3, [5, 9], [3, 9]), [5, 9], [3, 9], 2, 0)
    with pytest.raises(fa.FaError):   # not a varlen causal job
        fa.fa_split_queries(_desc(4, [5], [9]), [5], [9], 2, 0)


def _rank_main(rank, world, port, result):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cu_q, cu_k = [30, 75, 90], [40, 90, 130]
        N, D = 2, 8
        g = torch.Generator().manual_seed(11)
        q = torch.randn(cu_q[-1], N, D, generator=g, dtype=torch.float64)
        k = torch.randn(cu_k[-1], N, D, generator=g, dtype=torch.float64)
        v = torch.randn(cu_k[-1], N, D, generator=g, dtype=torch.float64)
        d = _desc(3, cu_q, cu_k, N, 64)
        r = fa.fa_split_queries(d, cu_q, cu_k, world, rank)
        o, l = _run_part_oracle(r, q, k, v)
        # ranks own disjoint rows; gather them only to check the assembly
        sizes = [None] * world
        dist.all_gather_object(sizes, (r["q_begin"], r["q_end"]))
        outs = [None] * world
        dist.all_gather_object(outs, (o, l))
        if rank == 0:
            full = Problem("TND", 3, N, cu_q[-1], cu_k[-1], D, sparse_mode=3,
                           actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
            o_ref, l_ref = oracle.attention(full, q, k, v)
            assert [s for s in sizes] == sorted(sizes) and sizes[-1][1] == cu_q[-1]
            np.testing.assert_array_equal(np.concatenate([x[0] for x in outs], 0), o_ref)
            np.testing.assert_array_equal(np.concatenate([x[1] for x in outs], 1), l_ref)
            result.put("ok")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_their_parts():
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(timeout=240)
    assert all(p_.exitcode == 0 for p_ in procs), [p_.exitcode for p_ in procs]
    assert q.get(timeout=5) == "ok"
