"""Failure detection without a GPU fault: a test hook makes CTA 0 skip its
first Q load, so a bounded device-side wait runs out; the kernel records the
site, drains its copies and MMAs, frees its tensor memory and returns, the
host reads FA_ERR_TIMEOUT, and the next call in the same process is correct."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CODE = r'''
import os, sys, numpy as np, torch
sys.path.insert(0, os.environ["FA_ROOT"]); sys.path.insert(0, os.path.join(os.environ["FA_ROOT"], "tests"))
import masked_attention_fa_b200 as fa
from masked_attention_fa_b200.workloads import random_inputs
from gpu_helpers import check_against_oracle
inp = random_inputs("BNSD", 1, 4, 512, 512, 128, seed=5)
attn = fa.MaskedAttention("BNSD", 1, 4, 512, 512, 128, 3)
o, l = attn(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda())
torch.cuda.synchronize()
st = fa.fa_sync_status(attn.handle)
print("FIRST", fa.STATUS[st], fa.fa_last_error())
attn.close()
os.environ.pop("FA_TEST_DROP_FIRST_Q")
kw = dict(layout="BNSD", B=1, N=4, Sq=512, Skv=512, D=128, sparse_mode=3)
check_against_oracle(kw, inp)
print("SECOND OK")
'''

# The allocation-free entry point: same hook, its status read through
# fa_noalloc_sync_status, then a call without the hook against the oracle.
CODE_NOALLOC = r'''
import os, sys, numpy as np, torch
sys.path.insert(0, os.environ["FA_ROOT"]); sys.path.insert(0, os.path.join(os.environ["FA_ROOT"], "tests"))
import masked_attention_fa_b200 as fa
import oracle
from masked_attention_fa_b200.workloads import random_inputs
from gpu_helpers import assert_close, problem_of
inp = random_inputs("BNSD", 1, 4, 512, 512, 128, seed=5)
q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
desc = fa.make_desc("BNSD", 1, 4, 512, 512, 128, 3)
o = torch.empty_like(q)
lse = torch.empty(1, 4, 512, device="cuda")
fa.fa_fwd_noalloc(desc, q, k, v, o, lse)
st = fa.fa_noalloc_sync_status(raise_on_error=False)
print("FIRST", fa.STATUS[st], fa.fa_last_error())
print("CLEARED", fa.STATUS[fa.fa_noalloc_sync_status(raise_on_error=False)])
os.environ.pop("FA_TEST_DROP_FIRST_Q")
o.fill_(float("nan"))
fa.fa_fwd_noalloc(desc, q, k, v, o, lse)
fa.fa_noalloc_sync_status()
kw = dict(layout="BNSD", B=1, N=4, Sq=512, Skv=512, D=128, sparse_mode=3)
o_ref, lse_ref = oracle.attention(problem_of(kw), inp["q"], inp["k"], inp["v"])
assert_close(o.float().cpu().double().numpy(), lse.cpu().double().numpy(), o_ref, lse_ref)
print("SECOND OK")
'''


def test_bounded_wait_reports_timeout_and_context_survives():
    env = dict(os.environ, FA_TEST_DROP_FIRST_Q="1", FA_WAIT_TIMEOUT_MS="300", FA_ROOT=ROOT)
    out = subprocess.run([sys.executable, "-c", CODE], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "FIRST FA_ERR_TIMEOUT" in out.stdout, out.stdout
    assert "SECOND OK" in out.stdout, out.stdout


def test_noalloc_bounded_wait_reports_timeout_and_next_call_is_correct():
    env = dict(os.environ, FA_TEST_DROP_FIRST_Q="1", FA_WAIT_TIMEOUT_MS="300", FA_ROOT=ROOT)
    out = subprocess.run([sys.executable, "-c", CODE_NOALLOC], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "FIRST FA_ERR_TIMEOUT" in out.stdout, out.stdout
    assert "CLEARED FA_OK" in out.stdout, out.stdout
    assert "SECOND OK" in out.stdout, out.stdout
