"""GPU parity of the dense-mask occupancy pre-pass and of the attention paths
that use it (sparseMode 1 allMask, sparseMode 0 with an attenMask).

The pre-pass's tile classes and ranges are integer results: they must equal
the oracle's block occupancy of its visibility matrix exactly. The attention
under structured masks (whole hidden / visible blocks, mixed blocks, hidden
rows, a hidden key block between visible ones, one 128-row sub-tile of a
256-row item without a visible key, items without any) is compared with the
fp64 oracle element by element, through fa_fwd, fa_fwd_with_ranges and
fa_fwd_noalloc. At full size, the leftUpCausal problem given as an explicit
lower-triangular allMask must reproduce the closed-form sparseMode 2 result
bit for bit.
"""
import numpy as np
import pytest
import torch

import masked_attention_fa_b200 as fa
import oracle
from masked_attention_fa_b200.workloads import (block_mask, lower_triangular_mask, make_inputs,
                                                named_workloads, random_inputs)
from gpu_helpers import assert_close, check_against_oracle, problem_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()
    assert torch.cuda.is_available()
    fa.load_library()


def _plane_bh(kind, B, N):
    if kind == "SS":
        return [(0, 0)]
    if kind == "B1SS":
        return [(b, 0) for b in range(B)]
    return [(b, h) for b in range(B) for h in range(N)]


def _mask_shape(kind, B, N, Sq, Skv):
    return {"SS": (Sq, Skv), "B1SS": (B, 1, Sq, Skv), "BNSS": (B, N, Sq, Skv)}[kind]


def _hidden_rows_mask(Sq, Skv):
    m = torch.zeros(Sq, Skv, dtype=torch.uint8)
    m[200:400] = 1
    return m


# (mode, mask kind, B, N, Sq, Skv, pre, next, mask builder)
OCC_CASES = [
    (1, "SS", 1, 1, 1000, 1000, 0, 0, lambda s: lower_triangular_mask(1000)),
    (1, "SS", 1, 1, 1024, 1024, 0, 0, lambda s: lower_triangular_mask(1024)),
    (1, "BNSS", 2, 2, 520, 784, 0, 0, lambda s: block_mask(s, 11)),
    (0, "B1SS", 2, 3, 700, 900, 300, 100, lambda s: block_mask(s, 12)),
    (0, "SS", 1, 2, 600, 640, -30, 200, lambda s: torch.zeros(s, dtype=torch.uint8)),
    (1, "SS", 1, 1, 129, 1, 0, 0, lambda s: torch.zeros(s, dtype=torch.uint8)),
    (1, "SS", 1, 1, 512, 512, 0, 0, lambda s: _hidden_rows_mask(512, 512)),
    (1, "B1SS", 2, 1, 384, 1040, 0, 0, lambda s: block_mask(s, 13, weights=[1, 0, 0, 1, 0, 0])),
]


@pytest.mark.parametrize("case", range(len(OCC_CASES)))
def test_occupancy_matches_oracle_exactly(case):
    mode, kind, B, N, Sq, Skv, pre, nxt, make = OCC_CASES[case]
    shape = _mask_shape(kind, B, N, Sq, Skv)
    mask = make(shape).to(torch.uint8).reshape(shape).contiguous()
    desc = fa.make_desc("BNSD", B, N, Sq, Skv, 64, mode, pre, nxt, None, kind)
    cls, rng = fa.fa_mask_occupancy(desc, mask.cuda())
    torch.cuda.synchronize()
    cls, rng = cls.cpu().numpy(), rng.cpu().numpy()
    kw = dict(layout="BNSD", B=B, N=N, Sq=Sq, Skv=Skv, D=64, sparse_mode=mode,
              pre_tokens=pre, next_tokens=nxt, mask_kind=kind)
    pb = problem_of(kw, mask)
    for p, (b, h) in enumerate(_plane_bh(kind, B, N)):
        want = oracle.tile_classes(pb, b, h)
        assert np.array_equal(cls[p], want), f"plane {p}: tile classes differ"
        assert np.array_equal(rng[p], oracle.tile_ranges(want)), f"plane {p}: ranges differ"


def _structured_mask(Sq, Skv):
    """Blocks of 128 chosen to reach the kernel's scheduling corners:
    rows 0-127 see key block 0 only and rows 128-255 key block 3 only (the
    item's two sub-tiles share no key block, blocks 1-2 are visited by
    neither); rows 256-511 see nothing (an item without key tiles); rows
    512-639 see blocks 0 and 4 with a hidden block between and a mixed
    diagonal block; the rest is a lower triangle."""
    m = torch.triu(torch.ones(Sq, Skv, dtype=torch.uint8), diagonal=1)
    m[0:512] = 1
    m[0:128, 0:128] = 0
    m[128:256, 384:512] = 0
    m[512:640] = 1
    m[512:640, 0:128] = 0
    m[512:640, 512:640] = torch.triu(torch.ones(128, 128, dtype=torch.uint8), diagonal=1)
    m[520, 5] = 1
    return m


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("layout", ["BNSD", "BSND"])
def test_structured_mask_scheduling_corners(layout, D):
    Sq = Skv = 768
    B, N = 1, 2
    inp = random_inputs(layout, B, N, Sq, Skv, D, seed=41)
    inp["mask"] = _structured_mask(Sq, Skv)
    kw = dict(layout=layout, B=B, N=N, Sq=Sq, Skv=Skv, D=D, sparse_mode=1, mask_kind="SS")
    check_against_oracle(kw, inp, what="structured allMask")


BLOCK_CASES = [
    # mode, kind, Sq, Skv, pre, next, seed
    (1, "SS", 640, 768, 0, 0, 21),
    (1, "BNSS", 300, 333, 0, 0, 22),
    (1, "B1SS", 520, 1040, 0, 0, 23),
    (0, "SS", 700, 900, 300, 100, 24),
    (0, "BNSS", 384, 512, 150, -40, 25),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(BLOCK_CASES)))
def test_block_masks_match_oracle(case, D):
    mode, kind, Sq, Skv, pre, nxt, seed = BLOCK_CASES[case]
    B, N = 2, 2
    inp = random_inputs("BNSD", B, N, Sq, Skv, D, seed=seed)
    inp["mask"] = block_mask(_mask_shape(kind, B, N, Sq, Skv), seed)
    kw = dict(layout="BNSD", B=B, N=N, Sq=Sq, Skv=Skv, D=D, sparse_mode=mode,
              pre_tokens=pre, next_tokens=nxt, mask_kind=kind)
    check_against_oracle(kw, inp, what=f"block mask {case}")


def test_with_ranges_and_noalloc_match_fa_fwd_bitwise():
    """The pre-pass run once and its ranges passed to fa_fwd_with_ranges, and
    the allocation-free entry point, give fa_fwd's bits (same kernels)."""
    B, N, Sq, Skv, D = 2, 2, 640, 768, 128
    inp = random_inputs("BNSD", B, N, Sq, Skv, D, seed=31)
    mask = block_mask((B, N, Sq, Skv), 31).cuda()
    q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
    attn = fa.MaskedAttention("BNSD", B, N, Sq, Skv, D, 1, mask_kind="BNSS")
    o1, l1 = attn(q, k, v, atten_mask=mask)
    _, ranges = attn.occupancy(mask)
    o2, l2 = attn(q, k, v, atten_mask=mask, ranges=ranges)
    o3 = torch.empty_like(o1)
    l3 = torch.empty_like(l1)
    fa.fa_fwd_noalloc(attn.desc, q, k, v, o3, l3, atten_mask=mask)
    torch.cuda.synchronize()
    attn.sync_status()
    attn.close()
    for o, l in ((o2, l2), (o3, l3)):
        assert torch.equal(o, o1)
        assert torch.equal(l.isneginf(), l1.isneginf())
        live = ~l1.isneginf()
        assert torch.equal(l[live], l1[live])
    pb = problem_of(dict(layout="BNSD", B=B, N=N, Sq=Sq, Skv=Skv, D=D, sparse_mode=1,
                         mask_kind="BNSS"), mask.cpu())
    o_ref, l_ref = oracle.attention(pb, inp["q"], inp["k"], inp["v"])
    assert_close(o1.float().cpu().double().numpy(), l1.cpu().double().numpy(), o_ref, l_ref)


def test_ranges_entry_point_rejects_bad_arguments():
    attn = fa.MaskedAttention("BNSD", 1, 1, 256, 256, 64, 1, mask_kind="SS")
    q = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16, device="cuda")
    mask = torch.zeros(256, 256, dtype=torch.uint8, device="cuda")
    _, ranges = attn.occupancy(mask)
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 256, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_with_ranges(attn.handle, q, q, q, o, lse, mask,
                              ranges.view(-1).view(torch.uint8)[4:])  # 4 bytes off
    assert e.value.status == 2
    attn.close()
    causal = fa.MaskedAttention("BNSD", 1, 1, 256, 256, 64, 2)
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd_with_ranges(causal.handle, q, q, q, o, lse, mask, ranges)
    assert e.value.status == 2
    causal.close()


def test_allmask_causal_full_size_equals_closed_form_causal():
    """B=2, N=16, S=4096, D=128: the lower-triangular allMask through the
    pre-pass visits the same tiles, masks the same keys and so reproduces
    the closed-form leftUpCausal output bit for bit; the pre-pass's classes
    are the triangle's (oracle, plane 0), and sampled rows match the fp64
    oracle."""
    wm = named_workloads()["allmask_causal_4k"]
    wc = named_workloads()["leftup_causal_4k"]
    inp = make_inputs(wm)
    q, k, v = (inp[x].cuda() for x in ("q", "k", "v"))
    mask = inp["mask"].cuda()
    am = fa.MaskedAttention(wm.layout, wm.B, wm.N, wm.Sq, wm.Skv, wm.D, 1, mask_kind="SS")
    ac = fa.MaskedAttention(wc.layout, wc.B, wc.N, wc.Sq, wc.Skv, wc.D, 2)
    om, lm = am(q, k, v, atten_mask=mask)
    oc, lc = ac(q, k, v)
    cls, rng = am.occupancy(mask)
    torch.cuda.synchronize()
    am.sync_status()
    ac.sync_status()
    am.close()
    ac.close()
    assert torch.equal(om, oc)
    assert torch.equal(lm, lc)
    nb = wm.Sq // 128
    qt, kt = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    want = np.where(kt < qt, 2, np.where(kt == qt, 1, 0)).astype(np.uint8)
    assert np.array_equal(cls[0].cpu().numpy(), want)
    pb = problem_of(dict(layout="BNSD", B=1, N=1, Sq=wm.Sq, Skv=wm.Skv, D=wm.D, sparse_mode=1,
                         mask_kind="SS"), inp["mask"])
    assert np.array_equal(cls[0].cpu().numpy(), oracle.tile_classes(pb, 0))
    rows = [0, 1, 127, 128, 255, 2047, 2048, 4095]
    for b, h in ((0, 0), (1, 15)):
        o_ref, l_ref = oracle.attention_rows(pb, inp["q"][b:b + 1, h:h + 1],
                                             inp["k"][b:b + 1, h:h + 1],
                                             inp["v"][b:b + 1, h:h + 1],
                                             [(0, 0, i) for i in rows])
        got = om[b, h, rows].float().cpu().double().numpy()
        gl = lm[b, h, rows].cpu().double().numpy()
        assert_close(got, gl, o_ref, l_ref, what=f"sampled rows b={b} h={h}")


# The device-side work-list rebuild has three paths: a parallel rank (at most
# 1024 items, at most 128 cost buckets), a counting sort placed by one warp
# (more items or buckets) and the unsorted enumeration (more than 65536
# items). Each must give exactly the result of the closed-form path for the
# same visible set (the kernels compute every item the same way; only the
# order the CTAs take them in differs).
SCHEDULE_CASES = [
    # name, (B, N, Sq, Skv, D), closed-form mode, mask ("causal" | "zero")
    ("buckets_over_128", (1, 2, 512, 8320, 64), 2, "causal"),
    ("items_over_1024", (1, 65, 4096, 4096, 64), 2, "causal"),
    ("items_over_65536", (257, 1, 65536, 128, 64), 0, "zero"),
]


@pytest.mark.parametrize("case", range(len(SCHEDULE_CASES)))
def test_schedule_paths_match_closed_form_bitwise(case):
    name, (B, N, Sq, Skv, D), mode, kind = SCHEDULE_CASES[case]
    g = torch.Generator(device="cuda").manual_seed(100 + case)
    q = torch.randn(B, N, Sq, D, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, N, Skv, D, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, N, Skv, D, generator=g, device="cuda").to(torch.bfloat16)
    if kind == "causal":
        mask = torch.triu(torch.ones(Sq, Skv, dtype=torch.uint8, device="cuda"), diagonal=1)
    else:
        mask = torch.zeros(Sq, Skv, dtype=torch.uint8, device="cuda")
    dense = fa.MaskedAttention("BNSD", B, N, Sq, Skv, D, 1, mask_kind="SS")
    closed = fa.MaskedAttention("BNSD", B, N, Sq, Skv, D, mode)
    od, ld = dense(q, k, v, atten_mask=mask)
    oc, lc = closed(q, k, v)
    torch.cuda.synchronize()
    dense.sync_status()
    closed.sync_status()
    dense.close()
    closed.close()
    assert torch.equal(od, oc), name
    assert torch.equal(ld, lc), name
