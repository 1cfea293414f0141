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


def test_bounded_wait_reports_timeout_and_context_survives():
    env = dict(os.environ, FA_TEST_DROP_FIRST_Q="1", FA_WAIT_TIMEOUT_MS="300", FA_ROOT=ROOT)
    out = subprocess.run([sys.executable, "-c", CODE], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "FIRST FA_ERR_TIMEOUT" in out.stdout, out.stdout
    assert "SECOND OK" in out.stdout, out.stdout
