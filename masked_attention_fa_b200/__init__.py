"""Python binding of the B200 masked attention forward C ABI (include/fa.h).

Argument marshalling only: every step of the computation runs in the CUDA
library ``libfa_b200.so`` (built in-tree by ``masked_attention_fa_b200.build``).
PyTorch is used for device memory and streams. If the library is missing the
import of any entry point fails loudly; there is no fallback.

The C entry points keep their names (``fa_create``, ``fa_fwd``, ...). The
``MaskedAttention`` class wraps a handle for convenience.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_BNSD, FA_BSND, FA_TND = 0, 1, 2
LAYOUTS = {"BNSD": FA_BNSD, "BSND": FA_BSND, "TND": FA_TND}
FA_MASK_NONE, FA_MASK_SS, FA_MASK_B1SS, FA_MASK_BNSS = 0, 1, 2, 3
MASK_KINDS = {None: FA_MASK_NONE, "SS": FA_MASK_SS, "B1SS": FA_MASK_B1SS, "BNSS": FA_MASK_BNSS}
STATUS = {0: "FA_OK", 1: "FA_ERR_NULLPTR", 2: "FA_ERR_PARAM_INVALID", 3: "FA_ERR_SHAPE",
          4: "FA_ERR_UNSUPPORTED", 5: "FA_ERR_ALLOC", 6: "FA_ERR_CUDA", 7: "FA_ERR_TIMEOUT",
          8: "FA_ERR_DEVICE"}
FA_TILE_EMPTY, FA_TILE_PARTIAL, FA_TILE_FULL = 0, 1, 2
FA_ALIBI_NONE, FA_ALIBI_RIGHT, FA_ALIBI_SQRT, FA_ALIBI_LEFT = 0, 1, 2, 3
ALIBI = {None: FA_ALIBI_NONE, "right": FA_ALIBI_RIGHT, "sqrt": FA_ALIBI_SQRT,
         "left": FA_ALIBI_LEFT}


class FaError(RuntimeError):
    def __init__(self, status, message):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {message}")


class fa_desc_t(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int32),
        ("sparse_mode", ctypes.c_int32),
        ("mask_kind", ctypes.c_int32),
        ("alibi", ctypes.c_int32),
        ("B", ctypes.c_int64),
        ("N", ctypes.c_int64),
        ("Sq", ctypes.c_int64),
        ("Skv", ctypes.c_int64),
        ("D", ctypes.c_int64),
        ("pre_tokens", ctypes.c_int64),
        ("next_tokens", ctypes.c_int64),
        ("scale", ctypes.c_double),
    ]


class fa_split_part_t(ctypes.Structure):
    _fields_ = [
        ("desc", fa_desc_t),
        ("q_begin", ctypes.c_int64),
        ("q_end", ctypes.c_int64),
        ("kv_begin", ctypes.c_int64),
        ("kv_end", ctypes.c_int64),
    ]


_lib = None


def load_library():
    """Load libfa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m masked_attention_fa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i64p = ctypes.POINTER(ctypes.c_int64)
    dp = ctypes.POINTER(fa_desc_t)
    st = ctypes.c_int32
    lib.fa_create.argtypes = [dp, ctypes.POINTER(P)]
    lib.fa_create.restype = st
    lib.fa_fwd.argtypes = [P, P, P, P, P, i64p, i64p, i64p, P, P, P]
    lib.fa_fwd.restype = st
    lib.fa_fwd_alibi.argtypes = [P, P, P, P, P, i64p, i64p, i64p, P, P, P]
    lib.fa_fwd_alibi.restype = st
    lib.fa_sync_status.argtypes = [P]
    lib.fa_sync_status.restype = st
    lib.fa_destroy.argtypes = [P]
    lib.fa_destroy.restype = st
    lib.fa_last_error.argtypes = []
    lib.fa_last_error.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_version.restype = ctypes.c_int32
    lib.fa_validate.argtypes = [dp, i64p, i64p, i64p, ctypes.c_int32]
    lib.fa_validate.restype = st
    lib.fa_visible_pairs.argtypes = [dp, i64p, i64p, i64p, ctypes.c_int32, i64p]
    lib.fa_visible_pairs.restype = st
    lib.fa_tile_class.argtypes = [dp, i64p, i64p, i64p, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.c_int64, ctypes.c_int64]
    lib.fa_tile_class.restype = ctypes.c_int32
    lib.fa_plan_stats.argtypes = [dp, i64p, i64p, i64p, ctypes.c_int32, i64p]
    lib.fa_plan_stats.restype = st
    lib.fa_plan_items.argtypes = [dp, i64p, i64p, i64p, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.POINTER(ctypes.c_int32), i64p]
    lib.fa_plan_items.restype = st
    lib.fa_fwd_noalloc.argtypes = [dp, P, P, P, P, i64p, i64p, i64p, P, P, P]
    lib.fa_fwd_noalloc.restype = st
    lib.fa_noalloc_sync_status.argtypes = [P]
    lib.fa_noalloc_sync_status.restype = st
    lib.fa_fwd_paged.argtypes = [P, P, P, P, P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                 i64p, i64p, i64p, P, P, P]
    lib.fa_fwd_paged.restype = st
    lib.fa_mask_occupancy.argtypes = [dp, P, P, P, P]
    lib.fa_mask_occupancy.restype = st
    lib.fa_fwd_with_ranges.argtypes = [P, P, P, P, P, P, P, P, P]
    lib.fa_fwd_with_ranges.restype = st
    lib.fa_split_queries.argtypes = [dp, i64p, i64p, ctypes.c_int32, i64p, ctypes.c_int32,
                                     ctypes.POINTER(fa_split_part_t), i64p, i64p]
    lib.fa_split_queries.restype = st
    _lib = lib
    return lib


EXPORTED = ("fa_create", "fa_fwd", "fa_sync_status", "fa_destroy", "fa_last_error",
            "fa_version", "fa_validate", "fa_visible_pairs", "fa_tile_class", "fa_plan_stats",
            "fa_plan_items", "fa_fwd_noalloc", "fa_split_queries", "fa_mask_occupancy",
            "fa_fwd_with_ranges", "fa_fwd_paged", "fa_noalloc_sync_status", "fa_fwd_alibi")


def _check(status):
    if status != 0:
        msg = load_library().fa_last_error().decode(errors="replace")
        raise FaError(status, msg)


# Work-list size per SM from which closed-form calls claim their items at
# run time (the library's kClaimMinItemsPerCta; used to name the kernel
# instance a call runs).
CLAIM_MIN_ITEMS_PER_CTA = 8


def make_desc(layout, B, N, Sq, Skv, D, sparse_mode=0, pre_tokens=0, next_tokens=0, scale=None,
              mask_kind=None, alibi=None) -> fa_desc_t:
    lay = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    mk = MASK_KINDS[mask_kind] if (mask_kind is None or isinstance(mask_kind, str)) else int(mask_kind)
    al = ALIBI[alibi] if (alibi is None or isinstance(alibi, str)) else int(alibi)
    sc = (1.0 / float(D) ** 0.5) if scale is None else float(scale)
    return fa_desc_t(lay, int(sparse_mode), mk, al, int(B), int(N), int(Sq), int(Skv), int(D),
                     int(pre_tokens), int(next_tokens), sc)


class _Arrays:
    """Host int64 arrays for prefix / actual_seq_* kept alive for one call."""

    def __init__(self, prefix, cu_q, cu_kv):
        self.prefix = None if prefix is None else np.ascontiguousarray(prefix, dtype=np.int64)
        self.cu_q = None if cu_q is None else np.ascontiguousarray(cu_q, dtype=np.int64)
        self.cu_kv = None if cu_kv is None else np.ascontiguousarray(cu_kv, dtype=np.int64)

    @staticmethod
    def _p(a):
        if a is None:
            return None
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))

    def ptrs(self):
        return self._p(self.prefix), self._p(self.cu_q), self._p(self.cu_kv)


# ---------------------------------------------------------------- C names

def fa_version() -> int:
    return int(load_library().fa_version())


def fa_last_error() -> str:
    return load_library().fa_last_error().decode(errors="replace")


def fa_validate(desc, prefix=None, actual_seq_qlen=None, actual_seq_kvlen=None, has_mask=False):
    """Status code of the host-side checks (0 = valid)."""
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    return int(load_library().fa_validate(ctypes.byref(desc), *a.ptrs(), int(bool(has_mask))))


def fa_visible_pairs(desc, prefix=None, actual_seq_qlen=None, actual_seq_kvlen=None,
                     has_mask=False) -> int:
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    out = ctypes.c_int64(0)
    _check(load_library().fa_visible_pairs(ctypes.byref(desc), *a.ptrs(), int(bool(has_mask)),
                                           ctypes.byref(out)))
    return int(out.value)


def fa_tile_class(desc, b, qt, kt, prefix=None, actual_seq_qlen=None, actual_seq_kvlen=None,
                  has_mask=False) -> int:
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    return int(load_library().fa_tile_class(ctypes.byref(desc), *a.ptrs(), int(bool(has_mask)),
                                             int(b), int(qt), int(kt)))


def fa_plan_items(desc, prefix=None, actual_seq_qlen=None, actual_seq_kvlen=None, num_sms=148):
    """The closed-form work list in the kernel's order on a device with
    num_sms SMs: int32 array [n, 4] of (sequence, head, 256-row block, cost
    key)."""
    import numpy as np
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    n = ctypes.c_int64(0)
    lib = load_library()
    st = lib.fa_plan_items(ctypes.byref(desc), *a.ptrs(), int(num_sms), 0, None, ctypes.byref(n))
    if n.value == 0:
        _check(st)
        return np.zeros((0, 4), dtype=np.int32)
    out = np.zeros((n.value, 4), dtype=np.int32)
    _check(lib.fa_plan_items(ctypes.byref(desc), *a.ptrs(), int(num_sms), n.value,
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), ctypes.byref(n)))
    return out


def fa_plan_stats(desc, prefix=None, actual_seq_qlen=None, actual_seq_kvlen=None,
                  has_mask=False):
    """(work items, EMPTY, PARTIAL, FULL) of the scheduler for one call."""
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    out = (ctypes.c_int64 * 4)()
    _check(load_library().fa_plan_stats(ctypes.byref(desc), *a.ptrs(), int(bool(has_mask)), out))
    return tuple(int(x) for x in out)


def fa_create(desc) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(load_library().fa_create(ctypes.byref(desc), ctypes.byref(h)))
    return h


def fa_destroy(h):
    _check(load_library().fa_destroy(h))


def fa_sync_status(h) -> int:
    """Raw status of the handle's last call (0 = OK)."""
    return int(load_library().fa_sync_status(h))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def fa_fwd(h, q, k, v, o, lse, atten_mask=None, prefix=None, actual_seq_qlen=None,
           actual_seq_kvlen=None, stream=None):
    """Enqueue one forward on `stream` (torch.cuda.Stream, raw handle int, or
    None = torch's current stream). Tensors must be CUDA tensors."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    _check(load_library().fa_fwd(h, _ptr(q), _ptr(k), _ptr(v), _ptr(atten_mask), *a.ptrs(),
                                 _ptr(o), _ptr(lse), ctypes.c_void_p(int(stream))))


def fa_fwd_alibi(h, q, k, v, slopes, o, lse, prefix=None, actual_seq_qlen=None,
                 actual_seq_kvlen=None, stream=None):
    """fa_fwd for a handle with an ALiBi variant; slopes: fp32 CUDA tensor [N]."""
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    _check(load_library().fa_fwd_alibi(h, _ptr(q), _ptr(k), _ptr(v), _ptr(slopes), *a.ptrs(),
                                       _ptr(o), _ptr(lse),
                                       ctypes.c_void_p(_stream_int(stream, q.device))))


def _stream_int(stream, device):
    import torch
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


def occupancy_shapes(desc):
    """Shapes of fa_mask_occupancy's outputs: (tile classes, ranges)."""
    planes = {1: 1, 2: int(desc.B), 3: int(desc.B) * int(desc.N)}[int(desc.mask_kind)]
    n_qt = (int(desc.Sq) + 127) // 128
    n_kt = (int(desc.Skv) + 127) // 128
    return (planes, n_qt, n_kt), (planes, n_qt, 4)


def fa_mask_occupancy(desc, atten_mask, tile_class=None, ranges=None, stream=None):
    """The dense-mask pre-pass alone (see include/fa.h): returns the uint8
    tile classes [P, ceil(Sq/128), ceil(Skv/128)] and the int32 ranges
    [P, ceil(Sq/128), 4] as CUDA tensors (allocated unless given)."""
    import torch
    cshape, rshape = occupancy_shapes(desc)
    dev = atten_mask.device
    if tile_class is None:
        tile_class = torch.empty(cshape, dtype=torch.uint8, device=dev)
    if ranges is None:
        ranges = torch.empty(rshape, dtype=torch.int32, device=dev)
    _check(load_library().fa_mask_occupancy(ctypes.byref(desc), _ptr(atten_mask),
                                            _ptr(tile_class), _ptr(ranges),
                                            ctypes.c_void_p(_stream_int(stream, dev))))
    return tile_class, ranges


def fa_fwd_with_ranges(h, q, k, v, o, lse, atten_mask, ranges, stream=None):
    """fa_fwd for a dense-mask handle with the pre-pass's ranges supplied."""
    _check(load_library().fa_fwd_with_ranges(h, _ptr(q), _ptr(k), _ptr(v), _ptr(atten_mask),
                                             _ptr(ranges), _ptr(o), _ptr(lse),
                                             ctypes.c_void_p(_stream_int(stream, q.device))))


def fa_fwd_paged(h, q, k_cache, v_cache, block_table, o, lse, actual_seq_qlen,
                 actual_seq_kvlen, prefix=None, stream=None):
    """Forward of a TND handle reading K/V from paged caches
    [num_blocks, block_size, N, D] through block_table [B, max_blocks] (int32)."""
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    num_blocks, block_size = int(k_cache.shape[0]), int(k_cache.shape[1])
    max_blocks = int(block_table.shape[1])
    _check(load_library().fa_fwd_paged(h, _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(block_table), num_blocks, block_size, max_blocks,
                                       *a.ptrs(), _ptr(o), _ptr(lse),
                                       ctypes.c_void_p(_stream_int(stream, q.device))))


def fa_fwd_noalloc(desc, q, k, v, o, lse, atten_mask=None, prefix=None, actual_seq_qlen=None,
                   actual_seq_kvlen=None, stream=None):
    """The allocation-free forward: no handle, the work list lives in the
    library's fixed device array (see include/fa.h). Same arguments as
    fa_fwd plus the descriptor."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    a = _Arrays(prefix, actual_seq_qlen, actual_seq_kvlen)
    _check(load_library().fa_fwd_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(atten_mask), *a.ptrs(), _ptr(o), _ptr(lse),
                                         ctypes.c_void_p(int(stream))))


def fa_noalloc_sync_status(stream=None, raise_on_error=True):
    """Wait for `stream` and read the error word of the allocation-free
    path's fixed array (see include/fa.h); returns the status code, or
    raises FaError for a non-OK status when raise_on_error."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    elif hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    lib = load_library()
    st = lib.fa_noalloc_sync_status(ctypes.c_void_p(int(stream)))
    if raise_on_error:
        _check(st)
    return st


def fa_split_queries(desc, actual_seq_qlen, actual_seq_kvlen, n_parts, part, cuts=None):
    """Part `part` of the query split of a TND mode-2/3 job (see include/fa.h).

    Returns a dict with the part's descriptor, its query token range
    [q_begin, q_end) and key range [kv_begin, kv_end) in the unsplit tensors,
    and its cumulative length arrays.
    """
    a = _Arrays(None, actual_seq_qlen, actual_seq_kvlen)
    c = None if cuts is None else np.ascontiguousarray(cuts, dtype=np.int64)
    out = fa_split_part_t()
    oq = np.zeros(int(desc.B), dtype=np.int64)
    ok = np.zeros(int(desc.B), dtype=np.int64)
    _, pq, pk = a.ptrs()
    _check(load_library().fa_split_queries(
        ctypes.byref(desc), pq, pk, int(n_parts), _Arrays._p(c), int(part), ctypes.byref(out),
        _Arrays._p(oq), _Arrays._p(ok)))
    nb = int(out.desc.B)
    return {"desc": out.desc, "q_begin": int(out.q_begin), "q_end": int(out.q_end),
            "kv_begin": int(out.kv_begin), "kv_end": int(out.kv_end),
            "actual_seq_qlen": oq[:nb].tolist(), "actual_seq_kvlen": ok[:nb].tolist()}


# ---------------------------------------------------------------- helper class

class MaskedAttention:
    """A handle for one problem shape: ``o, lse = attn(q, k, v, ...)``."""

    def __init__(self, layout, B, N, Sq, Skv, D, sparse_mode=0, pre_tokens=0, next_tokens=0,
                 scale=None, mask_kind=None, alibi=None):
        self.layout = layout
        self.desc = make_desc(layout, B, N, Sq, Skv, D, sparse_mode, pre_tokens, next_tokens,
                              scale, mask_kind, alibi)
        self.handle = fa_create(self.desc)

    def out_shapes(self):
        d = self.desc
        if self.layout == "BNSD":
            return (d.B, d.N, d.Sq, d.D), (d.B, d.N, d.Sq)
        if self.layout == "BSND":
            return (d.B, d.Sq, d.N, d.D), (d.B, d.N, d.Sq)
        return (d.Sq, d.N, d.D), (d.N, d.Sq)

    def __call__(self, q, k, v, atten_mask=None, prefix=None, actual_seq_qlen=None,
                 actual_seq_kvlen=None, out=None, lse=None, stream=None, ranges=None,
                 slopes=None):
        import torch
        oshape, lshape = self.out_shapes()
        if out is None:
            out = torch.empty(oshape, dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty(lshape, dtype=torch.float32, device=q.device)
        for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
                raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
        if not lse.is_contiguous() or lse.dtype != torch.float32:
            raise ValueError("lse must be a contiguous fp32 tensor")
        if atten_mask is not None:
            if atten_mask.dtype not in (torch.uint8, torch.bool) or not atten_mask.is_contiguous():
                raise ValueError("atten_mask must be a contiguous uint8/bool tensor")
        if slopes is not None:
            if slopes.dtype != torch.float32 or not slopes.is_contiguous() or not slopes.is_cuda:
                raise ValueError("slopes must be a contiguous fp32 CUDA tensor")
            fa_fwd_alibi(self.handle, q, k, v, slopes, out, lse, prefix, actual_seq_qlen,
                         actual_seq_kvlen, stream)
        elif ranges is not None:
            fa_fwd_with_ranges(self.handle, q, k, v, out, lse, atten_mask, ranges, stream)
        else:
            fa_fwd(self.handle, q, k, v, out, lse, atten_mask, prefix, actual_seq_qlen,
                   actual_seq_kvlen, stream)
        return out, lse

    def paged(self, q, k_cache, v_cache, block_table, actual_seq_qlen, actual_seq_kvlen,
              prefix=None, out=None, lse=None, stream=None):
        """O, lse of a TND handle with K/V in paged caches (see fa_fwd_paged)."""
        import torch
        oshape, lshape = self.out_shapes()
        if out is None:
            out = torch.empty(oshape, dtype=torch.bfloat16, device=q.device)
        if lse is None:
            lse = torch.empty(lshape, dtype=torch.float32, device=q.device)
        for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or not t.is_cuda:
                raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
        if block_table.dtype != torch.int32 or not block_table.is_contiguous():
            raise ValueError("block_table must be a contiguous int32 tensor")
        d = self.desc
        if (k_cache.dim() != 4 or tuple(v_cache.shape) != tuple(k_cache.shape)
                or k_cache.shape[2] != d.N or k_cache.shape[3] != d.D):
            raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, N, D]")
        if block_table.dim() != 2 or block_table.shape[0] != d.B:
            raise ValueError("block_table must be [B, max_blocks]")
        if tuple(q.shape) != tuple(oshape):
            raise ValueError(f"q must be {tuple(oshape)}")
        fa_fwd_paged(self.handle, q, k_cache, v_cache, block_table, out, lse, actual_seq_qlen,
                     actual_seq_kvlen, prefix, stream)
        return out, lse

    def occupancy(self, atten_mask, stream=None):
        """Run the dense-mask pre-pass on its own: (tile classes, ranges);
        pass the ranges back as ``attn(..., ranges=ranges)`` to skip it."""
        return fa_mask_occupancy(self.desc, atten_mask, stream=stream)

    def sync_status(self):
        st = fa_sync_status(self.handle)
        if st != 0:
            raise FaError(st, fa_last_error())

    def close(self):
        if self.handle is not None:
            fa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
