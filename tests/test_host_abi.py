"""Host-side checks of the C-ABI library (no GPU needed, no device work).

- the library loads and exports every entry point include/fa.h declares;
- validation returns the documented status for each constraint of the
  Ascend "sparseMode参数说明" page (sparseMode=0 notes, =4, =7, =8);
- the scheduler's visible-pair count and tile classes agree with the fp64
  oracle's explicit masks.
"""
import os
import re
import subprocess
import sys

import numpy as np
import pytest

import masked_attention_fa_b200 as fa
import oracle
from oracle import Problem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from masked_attention_fa_b200 import build
    build.build()


def test_library_exports_every_declared_entry_point():
    with open(os.path.join(ROOT, "include", "fa.h")) as f:
        header = f.read()
    declared = set(re.findall(r"^\s*(?:fa_status_t|int32_t|const char\*)\s+(fa_\w+)\s*\(",
                              header, re.M))
    assert declared >= {"fa_create", "fa_fwd", "fa_destroy", "fa_last_error"}
    lib = fa.load_library()
    for name in declared:
        assert hasattr(lib, name), name
    assert set(fa.EXPORTED) == declared
    assert fa.fa_version() == 1


def _status(**kw):
    arrays = {k: kw.pop(k) for k in ("prefix", "actual_seq_qlen", "actual_seq_kvlen", "has_mask")
              if k in kw}
    return fa.STATUS[fa.fa_validate(fa.make_desc(**kw), **arrays)]


BASE = dict(layout="BNSD", B=1, N=2, Sq=64, Skv=64, D=128)


def test_valid_descriptors():
    assert _status(**BASE, sparse_mode=2) == "FA_OK"
    assert _status(**BASE, sparse_mode=0) == "FA_OK"
    assert _status(**dict(BASE, D=64), sparse_mode=3) == "FA_OK"
    assert _status(**BASE, sparse_mode=4, pre_tokens=2147483647, next_tokens=2147483647) == "FA_OK"


@pytest.mark.parametrize("kw,status", [
    (dict(layout=7), "FA_ERR_PARAM_INVALID"),
    (dict(sparse_mode=9), "FA_ERR_PARAM_INVALID"),
    (dict(B=0), "FA_ERR_SHAPE"),
    (dict(Sq=-1), "FA_ERR_SHAPE"),
    (dict(D=96), "FA_ERR_UNSUPPORTED"),
    (dict(D=256), "FA_ERR_UNSUPPORTED"),
    (dict(scale=0.0), "FA_ERR_PARAM_INVALID"),
    (dict(scale=float("nan")), "FA_ERR_PARAM_INVALID"),
    (dict(sparse_mode=2, mask_kind="SS"), "FA_ERR_PARAM_INVALID"),
    (dict(sparse_mode=1), "FA_ERR_PARAM_INVALID"),
    (dict(sparse_mode=7), "FA_ERR_PARAM_INVALID"),
])
def test_descriptor_errors(kw, status):
    args = dict(BASE)
    args.update(kw)
    args.setdefault("sparse_mode", 0)
    assert _status(**args) == status


def test_mode0_negative_pre_next_constraints():
    """sparseMode=0 notes: next < 0 needs pre >= |next| and |next| < Skv;
    pre < 0 needs next >= |pre| and |pre| < Sq (only when a mask is given)."""
    m = dict(BASE, sparse_mode=0, mask_kind="SS", has_mask=True)
    assert _status(**m, pre_tokens=9, next_tokens=-3) == "FA_OK"
    assert _status(**m, pre_tokens=3, next_tokens=-3) == "FA_OK"
    assert _status(**m, pre_tokens=2, next_tokens=-3) == "FA_ERR_PARAM_INVALID"
    assert _status(**m, pre_tokens=100, next_tokens=-64) == "FA_ERR_PARAM_INVALID"
    assert _status(**m, pre_tokens=-3, next_tokens=7) == "FA_OK"
    assert _status(**m, pre_tokens=-3, next_tokens=2) == "FA_ERR_PARAM_INVALID"
    assert _status(**m, pre_tokens=-64, next_tokens=100) == "FA_ERR_PARAM_INVALID"
    # without a mask pre/next are ignored
    assert _status(**BASE, sparse_mode=0, pre_tokens=2, next_tokens=-3) == "FA_OK"
    # a mask pointer with mask_kind NONE cannot be interpreted
    assert _status(**BASE, sparse_mode=0, has_mask=True) == "FA_ERR_PARAM_INVALID"
    assert _status(**dict(BASE, mask_kind="SS"), sparse_mode=1) == "FA_ERR_NULLPTR"


def test_mode4_band_must_intersect():
    assert _status(**BASE, sparse_mode=4, pre_tokens=3, next_tokens=-3) == "FA_OK"
    assert _status(**BASE, sparse_mode=4, pre_tokens=3, next_tokens=-4) == "FA_ERR_PARAM_INVALID"


def test_prefix_and_varlen_arrays():
    assert _status(**BASE, sparse_mode=5) == "FA_ERR_NULLPTR"
    assert _status(**BASE, sparse_mode=5, prefix=[65]) == "FA_ERR_PARAM_INVALID"
    assert _status(**BASE, sparse_mode=6, prefix=[64]) == "FA_OK"
    t = dict(layout="TND", B=2, N=1, Sq=5, Skv=9, D=64, sparse_mode=3)
    assert _status(**t) == "FA_ERR_NULLPTR"
    assert _status(**t, actual_seq_qlen=[3, 5], actual_seq_kvlen=[3, 9]) == "FA_OK"
    assert _status(**t, actual_seq_qlen=[3, 4], actual_seq_kvlen=[3, 9]) == "FA_ERR_SHAPE"
    assert _status(**t, actual_seq_qlen=[6, 5], actual_seq_kvlen=[3, 9]) == "FA_ERR_SHAPE"
    assert _status(**dict(t, mask_kind="SS", sparse_mode=0)) == "FA_ERR_UNSUPPORTED"


def test_mode7_mode8_worked_examples_validate():
    """The two cards of each worked split on the sparseMode page validate,
    and breaking each listed condition is rejected."""
    c7 = dict(layout="TND", B=2, N=1, Sq=5, Skv=9, D=64, sparse_mode=7)
    arr7 = dict(actual_seq_qlen=[3, 5], actual_seq_kvlen=[3, 9])
    assert _status(**c7, pre_tokens=6, next_tokens=-2, **arr7) == "FA_OK"
    assert _status(**c7, pre_tokens=5, next_tokens=-2, **arr7) == "FA_ERR_PARAM_INVALID"
    assert _status(**c7, pre_tokens=6, next_tokens=1, **arr7) == "FA_ERR_PARAM_INVALID"
    assert _status(**c7, pre_tokens=6, next_tokens=-5, **arr7) == "FA_ERR_PARAM_INVALID"
    # a non-band sequence with Sq > Skv
    assert _status(**dict(c7, Skv=8), pre_tokens=6, next_tokens=-2, actual_seq_qlen=[3, 5],
                   actual_seq_kvlen=[2, 8]) == "FA_ERR_PARAM_INVALID"
    c8 = dict(layout="TND", B=3, N=1, Sq=12, Skv=13, D=64, sparse_mode=8)
    arr8 = dict(actual_seq_qlen=[3, 8, 12], actual_seq_kvlen=[4, 9, 13])
    assert _status(**c8, pre_tokens=4, next_tokens=1, **arr8) == "FA_OK"
    assert _status(**c8, pre_tokens=3, next_tokens=1, **arr8) == "FA_ERR_PARAM_INVALID"
    assert _status(**c8, pre_tokens=4, next_tokens=-2, **arr8) == "FA_ERR_PARAM_INVALID"
    assert _status(**dict(c8, layout="BNSD"), pre_tokens=4, next_tokens=1) == "FA_ERR_PARAM_INVALID"


def test_create_rejects_and_alloc_injection():
    with pytest.raises(fa.FaError) as e:
        fa.fa_create(fa.make_desc("BNSD", 1, 1, 8, 8, 80, 2))
    assert e.value.name == "FA_ERR_UNSUPPORTED" and "D=80" in str(e.value)
    h = fa.fa_create(fa.make_desc("BNSD", 1, 1, 8, 8, 64, 2))
    fa.fa_destroy(h)
    fa.fa_destroy(None)
    code = ("import masked_attention_fa_b200 as fa\n"
            "try:\n    fa.fa_create(fa.make_desc('BNSD',1,1,8,8,64,2))\n"
            "except fa.FaError as e:\n    print(e.name)\n")
    env = dict(os.environ, FA_TEST_FAIL_ALLOC="1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                         cwd=ROOT, timeout=120)
    assert out.stdout.strip() == "FA_ERR_ALLOC", out.stderr


# ---------------------------------------------------------------- scheduler vs oracle

def _random_problem(rng, mode):
    """A small random valid call of `mode` with lengths that cross 128-key tiles."""
    N = 1
    if mode in (7, 8):
        nseq = int(rng.integers(1, 4))
        lens = []
        for _ in range(nseq):
            sq = int(rng.integers(0, 300))
            skv = sq + int(rng.integers(0, 200))
            lens.append((sq, skv))
        nonempty = [i for i, (a, _) in enumerate(lens) if a > 0]
        if not nonempty:
            lens[0] = (5, 9)
            nonempty = [0]
        band = nonempty[-1] if mode == 7 else nonempty[0]
        sq, skv = lens[band]
        pre = skv + int(rng.integers(0, 50))
        if mode == 7:
            nxt = int(rng.integers(sq - skv, 1))
        else:
            nxt = sq - skv + int(rng.integers(0, 100))
        cu_q = np.cumsum([a for a, _ in lens]).tolist()
        cu_k = np.cumsum([b for _, b in lens]).tolist()
        return dict(layout="TND", B=nseq, N=N, Sq=cu_q[-1], Skv=cu_k[-1], D=64, sparse_mode=mode,
                    pre_tokens=pre, next_tokens=nxt, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_k)
    Sq = int(rng.integers(1, 400))
    Skv = int(rng.integers(1, 400))
    kw = dict(layout="BNSD", B=2, N=N, Sq=Sq, Skv=Skv, D=64, sparse_mode=mode)
    if mode == 4:
        pre = int(rng.integers(-100, 500))
        kw.update(pre_tokens=pre, next_tokens=int(rng.integers(-pre, 500)))
    if mode in (5, 6):
        kw["prefix"] = [int(rng.integers(0, Skv + 1)) for _ in range(2)]
    return kw


def _split(kw):
    desc_kw = {k: v for k, v in kw.items()
               if k not in ("prefix", "actual_seq_qlen", "actual_seq_kvlen")}
    arrays = {k: kw[k] for k in ("prefix", "actual_seq_qlen", "actual_seq_kvlen") if k in kw}
    return desc_kw, arrays


@pytest.mark.parametrize("mode", [0, 2, 3, 4, 5, 6, 7, 8])
def test_visible_pairs_match_oracle_counts(mode):
    rng = np.random.default_rng(100 + mode)
    for _ in range(6):
        kw = _random_problem(rng, mode)
        desc_kw, arrays = _split(kw)
        assert fa.fa_validate(fa.make_desc(**desc_kw), **arrays) == 0, kw
        got = fa.fa_visible_pairs(fa.make_desc(**desc_kw), **arrays)
        pb = Problem(**kw)
        assert got == oracle.visible_count(pb), kw


@pytest.mark.parametrize("mode", [0, 2, 3, 4, 5, 6, 7, 8])
def test_tile_classes_match_oracle_masks(mode):
    """EMPTY <=> the tile has no visible pair; FULL <=> every stored row sees
    all 128 keys of the tile; PARTIAL otherwise."""
    rng = np.random.default_rng(200 + mode)
    for _ in range(4):
        kw = _random_problem(rng, mode)
        desc_kw, arrays = _split(kw)
        desc = fa.make_desc(**desc_kw)
        pb = Problem(**kw)
        for b in range(pb.B):
            _, _, sq, skv = pb.seq(b)
            if sq == 0:
                continue
            vis = oracle.mask_matrix(pb, b)
            for qt in range((sq + 127) // 128):
                for kt in range((skv + 127) // 128 + 1):
                    blk = vis[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]
                    cls = fa.fa_tile_class(desc, b, qt, kt, **arrays)
                    if blk.size == 0 or not blk.any():
                        want = fa.FA_TILE_EMPTY
                    elif blk.all() and blk.shape[1] == 128:
                        want = fa.FA_TILE_FULL
                    else:
                        want = fa.FA_TILE_PARTIAL
                    assert cls == want, (kw, b, qt, kt)


def test_dense_mask_tiles_are_never_full():
    S = 300
    mask = np.zeros((S, S), np.uint8)
    desc = fa.make_desc("BNSD", 1, 1, S, S, 64, 0, pre_tokens=40, next_tokens=5, mask_kind="SS")
    pb = Problem("BNSD", 1, 1, S, S, 64, sparse_mode=0, pre_tokens=40, next_tokens=5,
                 mask=mask, mask_kind="SS")
    vis = oracle.mask_matrix(pb, 0)
    for qt in range(3):
        for kt in range(3):
            cls = fa.fa_tile_class(desc, 0, qt, kt, has_mask=True)
            blk = vis[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]
            assert cls != fa.FA_TILE_FULL
            assert (cls == fa.FA_TILE_EMPTY) == (not blk.any())


def test_plan_stats_item_count_and_named_workload_counts():
    from masked_attention_fa_b200.workloads import named_workloads
    ws = named_workloads()
    w = ws["leftup_causal_4k"]
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode)
    items, empty, partial, full = fa.fa_plan_stats(d)
    assert items == 2 * 16 * 16
    assert partial == 2 * 16 * 32        # the diagonal tiles
    assert full == 2 * 16 * (32 * 31 // 2)
    assert fa.fa_visible_pairs(d) == 268500992
    w = ws["rightdown_band_2k_8k"]
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode, w.pre_tokens,
                     w.next_tokens)
    assert fa.fa_visible_pairs(d) == 32 * 2048 * 1025
    w = ws["prefix_8k"]
    d = fa.make_desc(w.layout, w.B, w.N, w.Sq, w.Skv, w.D, w.sparse_mode)
    S = 8192
    expect = 16 * sum(P * P + S * (S + 1) // 2 - P * (P + 1) // 2 for P in w.prefix)
    assert fa.fa_visible_pairs(d, prefix=w.prefix) == expect == 2325942272


def test_occupancy_entry_points_validate_before_device_work():
    """fa_mask_occupancy and fa_fwd_with_ranges reject bad arguments on the
    host, before any device query (the pointers below are never touched)."""
    import ctypes
    lib = fa.load_library()
    dev = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10004)
    ss1 = fa.make_desc("BNSD", 1, 1, 256, 256, 64, 1, mask_kind="SS")
    causal = fa.make_desc("BNSD", 1, 1, 256, 256, 64, 2)
    tnd = fa.make_desc("TND", 1, 1, 256, 256, 64, 1, mask_kind="SS")
    occ = lib.fa_mask_occupancy
    assert fa.STATUS[occ(ctypes.byref(ss1), None, dev, dev, None)] == "FA_ERR_NULLPTR"
    assert fa.STATUS[occ(ctypes.byref(ss1), dev, dev, None, None)] == "FA_ERR_NULLPTR"
    assert fa.STATUS[occ(ctypes.byref(causal), dev, dev, dev, None)] == "FA_ERR_PARAM_INVALID"
    assert fa.STATUS[occ(ctypes.byref(tnd), dev, dev, dev, None)] == "FA_ERR_UNSUPPORTED"
    assert fa.STATUS[occ(ctypes.byref(ss1), dev, dev, odd, None)] == "FA_ERR_PARAM_INVALID"
    assert "16-byte" in fa.fa_last_error()
    h1, h2 = fa.fa_create(ss1), fa.fa_create(causal)
    try:
        fwr = lib.fa_fwd_with_ranges
        assert fa.STATUS[fwr(h2, dev, dev, dev, dev, dev, dev, dev, None)] == \
            "FA_ERR_PARAM_INVALID"
        assert fa.STATUS[fwr(h1, dev, dev, dev, None, dev, dev, dev, None)] == \
            "FA_ERR_PARAM_INVALID"
        assert fa.STATUS[fwr(h1, dev, dev, dev, dev, None, dev, dev, None)] == "FA_ERR_NULLPTR"
        assert fa.STATUS[fwr(h1, dev, dev, dev, dev, odd, dev, dev, None)] == \
            "FA_ERR_PARAM_INVALID"
        assert fa.STATUS[fwr(None, dev, dev, dev, dev, dev, dev, dev, None)] == "FA_ERR_NULLPTR"
    finally:
        fa.fa_destroy(h1)
        fa.fa_destroy(h2)


def test_occupancy_output_shapes():
    d = fa.make_desc("BSND", 3, 5, 300, 1000, 128, 0, 10, 10, None, "BNSS")
    assert fa.occupancy_shapes(d) == ((15, 3, 8), (15, 3, 4))
    d = fa.make_desc("BNSD", 3, 5, 128, 129, 128, 1, mask_kind="B1SS")
    assert fa.occupancy_shapes(d) == ((3, 1, 2), (3, 1, 4))
    d = fa.make_desc("BNSD", 3, 5, 1, 1, 64, 1, mask_kind="SS")
    assert fa.occupancy_shapes(d) == ((1, 1, 1), (1, 1, 4))


def test_paged_entry_point_validates_before_device_work():
    """fa_fwd_paged rejects bad handles and arguments on the host (the
    device pointers below are never touched)."""
    import ctypes
    lib = fa.load_library()
    dev = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    I64 = ctypes.c_int64 * 2
    cu_q, cu_kv = I64(1, 2), I64(40, 70)

    def call(h, q=dev, table=dev, nblk=10, bs=16, maxb=3, cq=cu_q, ckv=cu_kv):
        return fa.STATUS[lib.fa_fwd_paged(h, q, dev, dev, table, nblk, bs, maxb, None, cq, ckv,
                                          dev, dev, None)]

    tnd = fa.fa_create(fa.make_desc("TND", 2, 2, 2, 70, 64, 3))
    bsnd = fa.fa_create(fa.make_desc("BSND", 2, 2, 1, 40, 64, 3))
    try:
        assert call(None) == "FA_ERR_NULLPTR"
        assert call(tnd, table=None) == "FA_ERR_NULLPTR"
        assert call(bsnd) == "FA_ERR_UNSUPPORTED"
        assert call(tnd, maxb=2) == "FA_ERR_SHAPE"          # 40 keys need 3 blocks of 16
        assert call(tnd, bs=0) == "FA_ERR_PARAM_INVALID"
        assert call(tnd, nblk=0) == "FA_ERR_PARAM_INVALID"
        assert call(tnd, q=odd) == "FA_ERR_PARAM_INVALID"   # 16-byte alignment
        assert call(tnd, cq=I64(1, 3)) == "FA_ERR_SHAPE"     # last qlen must equal T_q
    finally:
        fa.fa_destroy(tnd)
        fa.fa_destroy(bsnd)


def test_claim_threshold_matches_the_library():
    """The binding's CLAIM_MIN_ITEMS_PER_CTA (used to name the kernel instance a
    call runs) is the library's kClaimMinItemsPerCta."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "masked_attention_fa_b200", "csrc", "fa_kernel.h")) as f:
        m = re.search(r"constexpr int kClaimMinItemsPerCta = (\d+);", f.read())
    assert m is not None
    assert int(m.group(1)) == fa.CLAIM_MIN_ITEMS_PER_CTA


# Work lists of closed-form calls, checked against the oracle's own tile
# ranges (from its visibility definition): every (sequence, head, block of
# 256 query rows) with a query row appears once, the cost keys are
# 8 x (the longer sub-tile's key tiles) + (the shorter's) and never increase
# along the list, so items without a key tile come last (the claiming kernel
# relies on that), and equal keys keep (sequence, block, head) order.
PLAN_CASES = [
    dict(layout="BNSD", B=2, N=3, Sq=700, Skv=900, D=64, sparse_mode=2),
    dict(layout="BNSD", B=1, N=2, Sq=1000, Skv=600, D=64, sparse_mode=3),
    dict(layout="BSND", B=2, N=2, Sq=800, Skv=2000, D=128, sparse_mode=4, pre_tokens=300,
         next_tokens=0),
    dict(layout="BNSD", B=3, N=2, Sq=900, Skv=900, D=64, sparse_mode=5, prefix=[0, 200, 900]),
    dict(layout="BNSD", B=1, N=2, Sq=600, Skv=700, D=64, sparse_mode=0),
    dict(layout="TND", B=6, N=2, Sq=0, Skv=0, D=64, sparse_mode=3,
         qlen=[300, 0, 129, 700, 5, 256], kvlen=[400, 50, 0, 900, 5, 1]),
    dict(layout="TND", B=2, N=2, Sq=5, Skv=9, D=64, sparse_mode=7, pre_tokens=6, next_tokens=-2,
         qlen=[3, 2], kvlen=[3, 6]),
    dict(layout="TND", B=3, N=2, Sq=12, Skv=13, D=64, sparse_mode=8, pre_tokens=4, next_tokens=1,
         qlen=[3, 5, 4], kvlen=[4, 5, 4]),
]


@pytest.mark.parametrize("case", range(len(PLAN_CASES)))
def test_work_list_order_and_keys_match_the_oracle_ranges(case):
    c = dict(PLAN_CASES[case])
    qlen, kvlen = c.pop("qlen", None), c.pop("kvlen", None)
    prefix = c.pop("prefix", None)
    cu_q = cu_kv = None
    if qlen is not None:
        cu_q, cu_kv = np.cumsum(qlen).tolist(), np.cumsum(kvlen).tolist()
        c["Sq"], c["Skv"] = cu_q[-1], cu_kv[-1]
    desc = fa.make_desc(**c)
    items = fa.fa_plan_items(desc, prefix=prefix, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)
    pb = Problem(**c, prefix=prefix, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)
    expected = {}
    for b in range(c["B"]):
        sq = pb.seq(b)[2]
        if sq <= 0:
            continue
        r = oracle.tile_ranges(oracle.tile_classes(pb, b))
        tiles = [int(r[qt, 1] - r[qt, 0]) if qt < len(r) else 0 for qt in range(len(r) + 1)]
        for qb in range((sq + 255) // 256):
            t0, t1 = tiles[2 * qb], tiles[2 * qb + 1]
            for h in range(c["N"]):
                expected[(b, h, qb)] = 8 * max(t0, t1) + min(t0, t1)
    got = {(int(b), int(h), int(qb)): int(key) for b, h, qb, key in items}
    assert len(got) == len(items), "an item appears twice"
    assert got == expected
    keys = items[:, 3]
    assert np.all(keys[:-1] >= keys[1:]), "keys must not increase along the list"
    for m in range(len(items) - 1):
        if keys[m] == keys[m + 1]:
            a, z = items[m], items[m + 1]
            assert (a[0], a[2], a[1]) < (z[0], z[2], z[1]), "ties keep (sequence, block, head) order"


def test_plan_items_reports_its_length_and_rejects_a_short_buffer():
    import ctypes
    desc = fa.make_desc("BNSD", 1, 2, 600, 600, 64, 2)
    lib = fa.load_library()
    n = ctypes.c_int64(-1)
    buf = (ctypes.c_int32 * 8)()
    st = lib.fa_plan_items(ctypes.byref(desc), None, None, None, 148, 2, buf, ctypes.byref(n))
    assert fa.STATUS[st] == "FA_ERR_SHAPE" and n.value == 6   # 3 blocks x 2 heads
    st = lib.fa_plan_items(ctypes.byref(desc), None, None, None, 148, 0, None, None)
    assert fa.STATUS[st] == "FA_ERR_NULLPTR"
    st = lib.fa_plan_items(ctypes.byref(desc), None, None, None, 148, 4, None, ctypes.byref(n))
    assert fa.STATUS[st] == "FA_ERR_NULLPTR"


def test_alibi_descriptor_checks():
    """The descriptor's ALiBi variant: 0..3, and only without an attenMask."""
    for kind in ("right", "sqrt", "left"):
        assert _status(**BASE, sparse_mode=3, alibi=kind) == "FA_OK"
        assert _status(**BASE, sparse_mode=0, alibi=kind) == "FA_OK"
    assert _status(**BASE, sparse_mode=3, alibi=4) == "FA_ERR_PARAM_INVALID"
    assert _status(**BASE, sparse_mode=3, alibi=-1) == "FA_ERR_PARAM_INVALID"
    assert _status(**BASE, sparse_mode=1, mask_kind="SS", alibi="right") == "FA_ERR_UNSUPPORTED"
    assert _status(**BASE, sparse_mode=0, mask_kind="BNSS", alibi="left") == "FA_ERR_UNSUPPORTED"


def test_alibi_entry_points_validate_before_device_work():
    """fa_fwd on an ALiBi handle, fa_fwd_alibi on a plain handle, missing or
    unaligned slopes, and the entry points without slopes (allocation-free,
    paged) are all refused on the host; the device pointers below are never
    touched."""
    import ctypes
    lib = fa.load_library()
    dev = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10002)
    ali = fa.fa_create(fa.make_desc("BNSD", 1, 2, 64, 64, 64, 3, alibi="right"))
    plain = fa.fa_create(fa.make_desc("BNSD", 1, 2, 64, 64, 64, 3))
    tnd = fa.fa_create(fa.make_desc("TND", 1, 2, 1, 64, 64, 3, alibi="right"))
    try:
        st = lambda x: fa.STATUS[x]
        assert st(lib.fa_fwd(ali, dev, dev, dev, None, None, None, None, dev, dev, None)) == \
            "FA_ERR_PARAM_INVALID"
        assert "fa_fwd_alibi" in fa.fa_last_error()
        assert st(lib.fa_fwd_alibi(plain, dev, dev, dev, dev, None, None, None, dev, dev,
                                   None)) == "FA_ERR_PARAM_INVALID"
        assert st(lib.fa_fwd_alibi(ali, dev, dev, dev, None, None, None, None, dev, dev,
                                   None)) == "FA_ERR_NULLPTR"
        assert st(lib.fa_fwd_alibi(ali, dev, dev, dev, odd, None, None, None, dev, dev,
                                   None)) == "FA_ERR_PARAM_INVALID"
        d = fa.make_desc("BNSD", 1, 2, 64, 64, 64, 3, alibi="sqrt")
        assert st(lib.fa_fwd_noalloc(ctypes.byref(d), dev, dev, dev, None, None, None, None,
                                     dev, dev, None)) == "FA_ERR_UNSUPPORTED"
        I64 = ctypes.c_int64 * 1
        assert st(lib.fa_fwd_paged(tnd, dev, dev, dev, dev, 4, 16, 4, None, I64(1), I64(64),
                                   dev, dev, None)) == "FA_ERR_UNSUPPORTED"
    finally:
        for h in (ali, plain, tnd):
            fa.fa_destroy(h)


def _expected_keys(c, prefix, cu_q, cu_kv):
    """Each item's cost key from the oracle's block ranges."""
    pb = Problem(**c, prefix=prefix, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv)
    expected = {}
    for b in range(c["B"]):
        sq = pb.seq(b)[2]
        if sq <= 0:
            continue
        r = oracle.tile_ranges(oracle.tile_classes(pb, b))
        tiles = [int(r[qt, 1] - r[qt, 0]) if qt < len(r) else 0 for qt in range(len(r) + 1)]
        for qb in range((sq + 255) // 256):
            t0, t1 = tiles[2 * qb], tiles[2 * qb + 1]
            for h in range(c["N"]):
                expected[(b, h, qb)] = 8 * max(t0, t1) + min(t0, t1)
    return expected


@pytest.mark.parametrize("num_sms", [148, 8])
def test_claimed_list_order_groups_sequence_and_head_inside_length_buckets(num_sms):
    """A list with at least 8 items per SM (claimed at run time) is ordered for
    L2 locality: items without a key tile last, then buckets of 24 key tiles
    (key // 192) longest first, inside a bucket (sequence, head) ascending,
    then the key descending, then the block; every item once with the oracle's
    key. With fewer items per SM the same call gives the strict order."""
    g = np.random.default_rng(9)
    qlen = g.integers(0, 1500, size=40).tolist()
    kvlen = [q + int(g.integers(0, 300)) for q in qlen]
    kvlen[3] = 0                                        # a sequence without keys
    cu_q, cu_kv = np.cumsum(qlen).tolist(), np.cumsum(kvlen).tolist()
    c = dict(layout="TND", B=40, N=6, Sq=cu_q[-1], Skv=cu_kv[-1], D=64, sparse_mode=3)
    desc = fa.make_desc(**c)
    items = fa.fa_plan_items(desc, actual_seq_qlen=cu_q, actual_seq_kvlen=cu_kv, num_sms=num_sms)
    got = {(int(b), int(h), int(qb)): int(key) for b, h, qb, key in items}
    assert len(got) == len(items) and got == _expected_keys(c, None, cu_q, cu_kv)
    keys = items[:, 3]
    claimed = len(items) >= fa.CLAIM_MIN_ITEMS_PER_CTA * num_sms
    assert claimed == (num_sms == 8)
    if not claimed:
        assert np.all(keys[:-1] >= keys[1:])
        return
    zero = keys == 0
    assert zero.any() and not np.any(zero[:-1] & ~zero[1:]), "items without a key tile last"
    k = keys[~zero]
    it = items[~zero]
    buckets = k // 192
    assert np.all(buckets[:-1] >= buckets[1:])
    for m in range(len(it) - 1):
        if buckets[m] == buckets[m + 1]:
            a, z = it[m], it[m + 1]
            assert (a[0], a[1], -a[3], a[2]) < (z[0], z[1], -z[3], z[2])


def test_trace_build_compiles_and_exports_its_accessors():
    """The per-cycle trace build (-DFA_TRACE=<cta>, masked_attention_fa_b200/trace.py) still
    compiles from the library's sources and exports the traced CTA and the stamp accessors;
    the library itself exports none of them (its kernel has no trace code)."""
    import ctypes
    from masked_attention_fa_b200 import trace
    lib = ctypes.CDLL(trace.build_trace(3))
    for name in ("fa_trace_cta", "fa_trace_clear", "fa_trace_read", "fa_create", "fa_fwd"):
        assert hasattr(lib, name), name
    assert lib.fa_trace_cta() == 3
    prod = fa.load_library()
    assert not hasattr(prod, "fa_trace_read")


def _synthetic_trace(pv_first):
    """Stamp arrays of two warpgroups over 20 turns with fixed phase lengths:
    S wait 100, load 50, max 200, then turn wait 300, exponentials 1000, PV
    wait 80, P store 400 (or, pv_first, PV wait 80 before the turn wait)."""
    import numpy as np
    tiles = np.zeros((8, 8, 1024), dtype=np.int64)
    warps = np.zeros((8, 4, 1024), dtype=np.int64)
    for s in (0, 1):
        t = 1000 + 500 * s
        for i in range(20):
            ev = {0: t, 1: t + 100, 2: t + 150, 3: t + 350}
            if pv_first:
                ev.update({6: t + 430, 4: t + 730, 5: t + 1730, 7: t + 1790})
            else:
                ev.update({4: t + 650, 5: t + 1650, 6: t + 1730, 7: t + 2130})
            for e, v in ev.items():
                tiles[s, e, i] = v
            for wq in range(4):
                warps[4 * s + wq, 0, i] = ev[4]
                warps[4 * s + wq, 1, i] = ev[5]
            t += 3000
    return tiles, warps


@pytest.mark.parametrize("pv_first", [False, True])
def test_trace_summary_phases_follow_the_event_order(pv_first):
    """The trace tool's table lists each turn's phases in the order they
    occur: with the previous PV awaited before the turn (the ALiBi instances)
    its columns follow that order, and every phase length is recovered."""
    from masked_attention_fa_b200.trace import summarize
    tiles, warps = _synthetic_trace(pv_first)
    lines = summarize(tiles, warps).splitlines()
    head = [c.strip() for c in lines[0].strip("|").split("|")]
    row0 = [c.strip() for c in lines[2].strip("|").split("|")]
    got = dict(zip(head[2:-1], (int(v) for v in row0[2:-1])))
    if pv_first:
        assert list(got) == ["S wait", "S load+mask", "row max", "PV wait", "turn wait",
                             "exponentials + P store", "P hand-over"]
        assert got == {"S wait": 100, "S load+mask": 50, "row max": 200, "PV wait": 80,
                       "turn wait": 300, "exponentials + P store": 1000, "P hand-over": 60}
    else:
        assert list(got) == ["S wait", "S load+mask", "row max", "turn wait", "exponentials",
                             "PV wait", "P store"]
        assert got == {"S wait": 100, "S load+mask": 50, "row max": 200, "turn wait": 300,
                       "exponentials": 1000, "PV wait": 80, "P store": 400}
    assert int(row0[-1]) == 3000  # turn period
