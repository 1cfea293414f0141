"""Shared pieces of the GPU tests: run the CUDA path, compare with the oracle."""
import numpy as np
import torch

import masked_attention_fa_b200 as fa
import oracle
from oracle import Problem

# Tolerances on O (bf16 in, fp32 accumulate, bf16 out) and on the fp32 lse.
TOL_MAX_O = 2e-2
TOL_MEAN_O = 2e-3
TOL_LSE = 1e-3


def run_cuda(kw, q, k, v, mask=None, prefix=None, cu_q=None, cu_kv=None):
    """One call through the C ABI; returns (O, lse) as CPU float64 arrays."""
    desc_kw = {k_: kw[k_] for k_ in ("layout", "B", "N", "Sq", "Skv", "D", "sparse_mode",
                                      "pre_tokens", "next_tokens", "scale", "mask_kind")
               if k_ in kw}
    attn = fa.MaskedAttention(**desc_kw)
    try:
        o, lse = attn(q.cuda(), k.cuda(), v.cuda(),
                      atten_mask=None if mask is None else mask.cuda(), prefix=prefix,
                      actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)
        torch.cuda.synchronize()
        attn.sync_status()
    finally:
        attn.close()
    return o.float().cpu().double().numpy(), lse.cpu().double().numpy()


def problem_of(kw, mask=None, prefix=None, cu_q=None, cu_kv=None):
    pkw = {k_: kw[k_] for k_ in ("layout", "B", "N", "Sq", "Skv", "D", "sparse_mode",
                                  "pre_tokens", "next_tokens", "scale") if k_ in kw}
    return Problem(**pkw, mask=None if mask is None else mask.numpy(),
                   mask_kind=kw.get("mask_kind"), prefix=prefix, actual_seq_qlen=cu_q,
                   actual_seq_kvlen=cu_kv)


def assert_close(o, lse, o_ref, lse_ref, what=""):
    """The parity bar: max|dO| <= 2e-2, mean|dO| <= 2e-3, max|dlse| <= 1e-3,
    and exactly the same rows with no visible key (lse = -inf)."""
    assert o.shape == o_ref.shape, what
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), f"{what}: rows without visible keys differ"
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    d = np.abs(o - o_ref)
    assert d.max() <= TOL_MAX_O, f"{what}: max|dO| = {d.max():.3e}"
    assert d.mean() <= TOL_MEAN_O, f"{what}: mean|dO| = {d.mean():.3e}"
    live = ~dead
    if live.any():
        dl = np.abs(lse[live] - lse_ref[live]).max()
        assert dl <= TOL_LSE, f"{what}: max|dlse| = {dl:.3e}"


def check_against_oracle(kw, inputs, prefix=None, cu_q=None, cu_kv=None, what=""):
    q, k, v, mask = inputs["q"], inputs["k"], inputs["v"], inputs.get("mask")
    o, lse = run_cuda(kw, q, k, v, mask, prefix, cu_q, cu_kv)
    pb = problem_of(kw, mask, prefix, cu_q, cu_kv)
    o_ref, lse_ref = oracle.attention(pb, q, k, v)
    assert_close(o, lse, o_ref, lse_ref, what or str(kw))
    return o, lse
