"""Oracle for the masked attention forward (fp64, CPU). TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its Python binding) never touches it, and it never touches the product: the
two share only the seeded input generators of
``masked_attention_fa_b200.workloads``, which hold none of the method's
arithmetic.

The arithmetic lives in ``fa_oracle.c`` (plain C, fp64, OpenMP over heads);
this module only builds it with gcc and marshals numpy arrays through ctypes.
Every function of the C file is pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

LAYOUTS = {"BNSD": 0, "BSND": 1, "TND": 2}
# ALiBi variants of the "压缩mask" page's alibi section.
ALIBI = {None: 0, "right": 1, "sqrt": 2, "left": 3}
MASK_KINDS = {None: 0, "SS": 1, "B1SS": 2, "BNSS": 3}


class _Desc(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int32),
        ("sparse_mode", ctypes.c_int32),
        ("mask_kind", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
        ("B", ctypes.c_int64),
        ("N", ctypes.c_int64),
        ("Sq", ctypes.c_int64),
        ("Skv", ctypes.c_int64),
        ("D", ctypes.c_int64),
        ("pre_tokens", ctypes.c_int64),
        ("next_tokens", ctypes.c_int64),
        ("scale", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile fa_oracle.c into liboracle.so next to it (gcc, -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_visible.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, i64, i64, i64, i64]
        lib.oracle_visible.restype = ctypes.c_int
        lib.oracle_attn.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P, P, P, P]
        lib.oracle_attn.restype = ctypes.c_int
        lib.oracle_attn_alibi.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, ctypes.c_int32, P,
                                          P, P, P, P, P]
        lib.oracle_attn_alibi.restype = ctypes.c_int
        lib.oracle_attn_rows.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P, P, i64, P, P, P]
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_rows_alibi.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, ctypes.c_int32,
                                               P, P, P, P, i64, P, P, P]
        lib.oracle_attn_rows_alibi.restype = ctypes.c_int
        lib.oracle_mask.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, i64, i64, P]
        lib.oracle_mask.restype = None
        lib.oracle_tile_classes.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, i64, i64, i64, P]
        lib.oracle_tile_classes.restype = None
        lib.oracle_tile_ranges.argtypes = [P, i64, i64, P]
        lib.oracle_tile_ranges.restype = None
        lib.oracle_attn_paged.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P, P, i64, i64,
                                          P, P]
        lib.oracle_attn_paged.restype = ctypes.c_int
        lib.oracle_visible_count.argtypes = [ctypes.POINTER(_Desc), P, P, P, P]
        lib.oracle_visible_count.restype = ctypes.c_int64
        lib.oracle_flash_tiled.argtypes = [P, P, P, P, i64, i64, i64, i64, ctypes.c_double, P]
        lib.oracle_flash_tiled.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


class Problem:
    """Arguments of one call, in the terms of the Ascend sparseMode page.

    For TND, ``B`` is the number of sequences, ``Sq``/``Skv`` are the token
    totals and ``actual_seq_qlen``/``actual_seq_kvlen`` hold the cumulative
    end offsets (no leading 0).
    """

    def __init__(self, layout, B, N, Sq, Skv, D, sparse_mode=0, pre_tokens=0, next_tokens=0,
                 scale=None, mask=None, mask_kind=None, prefix=None,
                 actual_seq_qlen=None, actual_seq_kvlen=None):
        self.layout = layout
        self.B, self.N, self.Sq, self.Skv, self.D = int(B), int(N), int(Sq), int(Skv), int(D)
        self.sparse_mode = int(sparse_mode)
        self.pre_tokens, self.next_tokens = int(pre_tokens), int(next_tokens)
        self.scale = float(scale) if scale is not None else 1.0 / float(D) ** 0.5
        self.mask = None if mask is None else np.ascontiguousarray(np.asarray(mask, dtype=np.uint8))
        self.mask_kind = mask_kind if self.mask is not None else None
        self.prefix = None if prefix is None else np.ascontiguousarray(np.asarray(prefix, dtype=np.int64))
        self.cu_q = None if actual_seq_qlen is None else np.ascontiguousarray(
            np.asarray(actual_seq_qlen, dtype=np.int64))
        self.cu_kv = None if actual_seq_kvlen is None else np.ascontiguousarray(
            np.asarray(actual_seq_kvlen, dtype=np.int64))
        if self.sparse_mode == 1 and self.mask is None:
            raise ValueError("sparseMode 1 needs an attenMask")

    def desc(self) -> _Desc:
        return _Desc(LAYOUTS[self.layout], self.sparse_mode, MASK_KINDS[self.mask_kind], 0,
                     self.B, self.N, self.Sq, self.Skv, self.D,
                     self.pre_tokens, self.next_tokens, self.scale)

    def seq(self, b):
        """(q_off, kv_off, Sq_b, Skv_b) of sequence b."""
        if self.layout == "TND":
            q0 = 0 if b == 0 else int(self.cu_q[b - 1])
            k0 = 0 if b == 0 else int(self.cu_kv[b - 1])
            return q0, k0, int(self.cu_q[b]) - q0, int(self.cu_kv[b]) - k0
        return 0, 0, self.Sq, self.Skv

    def _ptrs(self):
        def p(a):
            return None if a is None else a.ctypes.data
        return p(self.prefix), p(self.cu_q), p(self.cu_kv), p(self.mask)

    def q_shape(self):
        if self.layout == "BNSD":
            return (self.B, self.N, self.Sq, self.D)
        if self.layout == "BSND":
            return (self.B, self.Sq, self.N, self.D)
        return (self.Sq, self.N, self.D)

    def kv_shape(self):
        if self.layout == "BNSD":
            return (self.B, self.N, self.Skv, self.D)
        if self.layout == "BSND":
            return (self.B, self.Skv, self.N, self.D)
        return (self.Skv, self.N, self.D)

    def lse_shape(self):
        if self.layout == "TND":
            return (self.N, self.Sq)
        return (self.B, self.N, self.Sq)


def _f64(a):
    if hasattr(a, "detach"):  # torch tensor (exact upcast of bf16 values)
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def visible(pb: Problem, b, h, i, j) -> bool:
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    return bool(_load().oracle_visible(ctypes.byref(d), pre, cq, ckv, m, b, h, i, j))


def mask_matrix(pb: Problem, b: int, h: int = 0) -> np.ndarray:
    """Explicit [Sq_b, Skv_b] visibility of sequence b, head h (1 = visible)."""
    _, _, sq, skv = pb.seq(b)
    out = np.zeros((max(sq, 0), max(skv, 0)), dtype=np.uint8)
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    if sq > 0 and skv > 0:
        _load().oracle_mask(ctypes.byref(d), pre, cq, ckv, m, b, h, out.ctypes.data)
    return out


def tile_classes(pb: Problem, b: int, h: int = 0, tile: int = 128) -> np.ndarray:
    """Block occupancy of sequence b, head h: [ceil(Sq_b/tile), ceil(Skv_b/tile)]
    uint8, 0 = no visible pair, 2 = every existing row sees every key of the
    block (all keys existing), 1 = otherwise."""
    _, _, sq, skv = pb.seq(b)
    out = np.zeros(((max(sq, 0) + tile - 1) // tile, (max(skv, 0) + tile - 1) // tile),
                   dtype=np.uint8)
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    if out.size:
        _load().oracle_tile_classes(ctypes.byref(d), pre, cq, ckv, m, b, h, tile,
                                    out.ctypes.data)
    return out


def tile_ranges(classes) -> np.ndarray:
    """Per query block of a class matrix: (lo, hi, full_lo, full_hi) int32."""
    c = np.ascontiguousarray(np.asarray(classes, dtype=np.uint8))
    n_qt, n_kt = c.shape
    out = np.zeros((n_qt, 4), dtype=np.int32)
    if n_qt:
        _load().oracle_tile_ranges(c.ctypes.data, n_qt, n_kt, out.ctypes.data)
    return out


def visible_count(pb: Problem) -> int:
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    return int(_load().oracle_visible_count(ctypes.byref(d), pre, cq, ckv, m))


def attention(pb: Problem, q, k, v, alibi=None, slopes=None):
    """Full forward in fp64: returns (O in Q's layout, lse). With alibi in
    ("right", "sqrt", "left") and slopes [N], each visible score gets
    slopes[h] times that variant's bias added."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    assert q.shape == pb.q_shape() and k.shape == pb.kv_shape() and v.shape == pb.kv_shape()
    o = np.zeros(pb.q_shape(), dtype=np.float64)
    lse = np.full(pb.lse_shape(), -np.inf, dtype=np.float64)
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    if alibi is None:
        err = _load().oracle_attn(ctypes.byref(d), pre, cq, ckv, m, q.ctypes.data,
                                  k.ctypes.data, v.ctypes.data, o.ctypes.data, lse.ctypes.data)
    else:
        sl = np.ascontiguousarray(np.asarray(slopes, dtype=np.float64).reshape(-1))
        assert sl.shape == (pb.N,)
        err = _load().oracle_attn_alibi(ctypes.byref(d), pre, cq, ckv, m, ALIBI[alibi],
                                        sl.ctypes.data, q.ctypes.data, k.ctypes.data,
                                        v.ctypes.data, o.ctypes.data, lse.ctypes.data)
    if err:
        raise MemoryError("oracle_attn: allocation failed")
    return o, lse


def attention_paged(pb: Problem, q, k_cache, v_cache, block_table, block_size: int):
    """Forward of a TND problem with K/V read from paged caches
    [num_blocks, block_size, N, D] through block_table [B, max_blocks]
    (int32): returns (O [T_q, N, D], lse [N, T_q])."""
    assert pb.layout == "TND"
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    assert q.shape == pb.q_shape() and kc.shape == vc.shape and kc.shape[1] == block_size
    o = np.zeros(pb.q_shape(), dtype=np.float64)
    lse = np.full(pb.lse_shape(), -np.inf, dtype=np.float64)
    d = pb.desc()
    pre, cq, ckv, _ = pb._ptrs()
    err = _load().oracle_attn_paged(ctypes.byref(d), pre, cq, ckv, q.ctypes.data, kc.ctypes.data,
                                    vc.ctypes.data, bt.ctypes.data, bt.shape[1], block_size,
                                    o.ctypes.data, lse.ctypes.data)
    if err:
        raise MemoryError("oracle_attn_paged: allocation failed")
    return o, lse


def attention_rows(pb: Problem, q, k, v, rows, alibi=None, slopes=None):
    """Selected rows (b, h, i) only: returns (O rows [n, D], lse [n]); the
    ALiBi arguments are attention()'s."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    n = rows.shape[0]
    o = np.zeros((n, pb.D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    d = pb.desc()
    pre, cq, ckv, m = pb._ptrs()
    sl = None
    if alibi is not None:
        sl = np.ascontiguousarray(np.asarray(slopes, dtype=np.float64).reshape(-1))
        assert sl.shape == (pb.N,)
    err = _load().oracle_attn_rows_alibi(ctypes.byref(d), pre, cq, ckv, m, ALIBI[alibi],
                                         None if sl is None else sl.ctypes.data, q.ctypes.data,
                                         k.ctypes.data, v.ctypes.data, n, rows.ctypes.data,
                                         o.ctypes.data, lse.ctypes.data)
    if err:
        raise MemoryError("oracle_attn_rows: allocation failed")
    return o, lse


def flash_tiled(q, k, v, block_size=4, scale=None, vis=None):
    """The exercise page's tiled online-softmax attention on [B, S, D] inputs."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S, D = q.shape
    scale = 1.0 / float(D) ** 0.5 if scale is None else float(scale)
    out = np.zeros_like(q)
    vptr = None
    if vis is not None:
        vis = np.ascontiguousarray(np.asarray(vis, dtype=np.uint8))
        assert vis.shape == (B, S, S)
        vptr = vis.ctypes.data
    _load().oracle_flash_tiled(q.ctypes.data, k.ctypes.data, v.ctypes.data, vptr, B, S, D,
                               int(block_size), scale, out.ctypes.data)
    return out
