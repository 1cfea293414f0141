"""The bench's query-split path (bench.py --split) on CPU: two gloo ranks each
take their part of the sparseMode page's multi-card split of one varlen job
(sparseMode=7/8 sections: query tokens cut across cards, K/V whole) through
the same planning, slicing and per-rank step the bench uses, with the fp64
oracle standing in for the device call; the parts, gathered, equal the
unsplit job's result bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch

import bench
import oracle
from oracle import Problem
from masked_attention_fa_b200.workloads import Workload, make_inputs


def _job(mode):
    cu_q, cu_k = ([200, 700, 1000], [260, 800, 1150]) if mode == 3 else \
        ([200, 700, 1000], [150, 640, 900])
    return Workload(f"split_test_{mode}", "TND", 3, 2, cu_q[-1], cu_k[-1], 64, mode, seed=17,
                    actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)


def _oracle_forward(desc, q, k, v, cu_q, cu_kv):
    pb = Problem("TND", desc.B, desc.N, desc.Sq, desc.Skv, desc.D,
                 sparse_mode=desc.sparse_mode, pre_tokens=desc.pre_tokens,
                 next_tokens=desc.next_tokens, scale=desc.scale, actual_seq_qlen=cu_q,
                 actual_seq_kvlen=cu_kv)
    return oracle.attention(pb, q, k, v)


def _rank_main(rank, world, port, mode, result):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _job(mode)
        inputs = make_inputs(w)
        part = bench.split_rank_part(w, world, rank)
        got = bench.split_step(part, bench.split_part_inputs(inputs, part), _oracle_forward)
        parts = [None] * world
        dist.all_gather_object(parts, (part["q_begin"], part["q_end"], part["desc"].sparse_mode,
                                       got))
        if rank == 0:
            pb = Problem("TND", w.B, w.N, w.Sq, w.Skv, w.D, sparse_mode=mode,
                         actual_seq_qlen=w.actual_seq_qlen, actual_seq_kvlen=w.actual_seq_kvlen)
            o_ref, l_ref = oracle.attention(pb, inputs["q"], inputs["k"], inputs["v"])
            ranges = [(a, b) for a, b, _, _ in parts]
            assert ranges[0][0] == 0 and ranges[-1][1] == w.Sq
            assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
            # the part that cuts a sequence at its top is the band (7 from a
            # rightDownCausal job, 8 from a leftUpCausal one)
            assert {m for _, _, m, _ in parts} <= ({3, 7} if mode == 3 else {2, 8})
            o = np.concatenate([g[0] for _, _, _, g in parts if g is not None], 0)
            lse = np.concatenate([g[1] for _, _, _, g in parts if g is not None], 1)
            np.testing.assert_array_equal(o, o_ref)
            np.testing.assert_array_equal(lse, l_ref)
            result.put("ok")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [3, 2])
def test_bench_split_path_on_two_gloo_ranks(mode):
    import torch.multiprocessing as mp
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, mode, q)) for r in range(2)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(timeout=240)
    assert all(p_.exitcode == 0 for p_ in procs), [p_.exitcode for p_ in procs]
    assert q.get(timeout=5) == "ok"


def test_split_of_one_part_is_the_whole_job():
    w = _job(3)
    part = bench.split_rank_part(w, 1, 0)
    assert (part["q_begin"], part["q_end"], part["kv_begin"], part["kv_end"]) == \
        (0, w.Sq, 0, w.Skv)
    assert part["actual_seq_qlen"] == w.actual_seq_qlen
