"""The query split on one device: every part runs through fa_fwd on its own
slice of Q/K/V and the parts' rows reassemble the unsplit call (within the
parity tolerances) and match the oracle."""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
from masked_attention_fa_b200.workloads import random_inputs
from gpu_helpers import assert_close, check_against_oracle, run_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", [2, 3])
def test_split_parts_on_one_device_reassemble(mode):
    lq = [700, 1300, 260, 900]
    lk = [900, 1300, 400, 1000]
    cu_q, cu_k = np.cumsum(lq).tolist(), np.cumsum(lk).tolist()
    N, D = 4, 128
    inp = random_inputs("TND", 4, N, cu_q[-1], cu_k[-1], D, seed=77 + mode)
    kw = dict(layout="TND", B=4, N=N, Sq=cu_q[-1], Skv=cu_k[-1], D=D, sparse_mode=mode)
    o_full, l_full = check_against_oracle(kw, inp, cu_q=cu_q, cu_kv=cu_k)
    desc = fa.make_desc("TND", 4, N, cu_q[-1], cu_k[-1], D, mode)
    n_parts = 3
    parts_o, parts_l, modes = [], [], set()
    for part in range(n_parts):
        r = fa.fa_split_queries(desc, cu_q, cu_k, n_parts, part)
        pd = r["desc"]
        modes.add(pd.sparse_mode)
        sub = {"q": inp["q"][r["q_begin"]:r["q_end"]], "k": inp["k"][r["kv_begin"]:r["kv_end"]],
               "v": inp["v"][r["kv_begin"]:r["kv_end"]]}
        pkw = dict(layout="TND", B=pd.B, N=N, Sq=pd.Sq, Skv=pd.Skv, D=D,
                   sparse_mode=pd.sparse_mode, pre_tokens=pd.pre_tokens,
                   next_tokens=pd.next_tokens)
        o, l = check_against_oracle(pkw, sub, cu_q=r["actual_seq_qlen"],
                                    cu_kv=r["actual_seq_kvlen"])
        parts_o.append(o)
        parts_l.append(l)
    assert modes & {7, 8}, "the balanced cut should land inside a sequence"
    assert_close(np.concatenate(parts_o, 0), np.concatenate(parts_l, 1), o_full, l_full,
                 "reassembled parts vs the unsplit call")
