"""ctypes binding of libkascade.so (the C ABI in include/kascade.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are torch CUDA tensors (used for device memory and
streams); the library raises if it was not built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

__all__ = ["Shape", "KascadeError", "lib", "OP_SELECT", "OP_SPARSE_DECODE", "OP_SPARSE_PREFILL",
           "OP_DENSE", "workspace_bytes", "index_count", "index_offsets", "Workspace", "select",
           "sparse_decode", "sparse_prefill", "dense_ref", "status_str", "launch_count", "EXPORTS", "LIB_PATH",
           "select_decode_static", "select_decode_static_error", "refine_select", "OP_REFINE",
           "index_overlap", "plan_anchors", "sparse_decode_paged", "select_varlen", "sparse_decode_varlen"]

LIB_PATH = os.environ.get("KASCADE_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkascade.so")

OP_SELECT, OP_SPARSE_DECODE, OP_SPARSE_PREFILL, OP_DENSE, OP_REFINE, OP_SELECT_VARLEN = 0, 1, 2, 3, 4, 5
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TOO_LARGE = 0, 1, 2, 3, 4, 5
FLAG_PDL, FLAG_INPUTS_STABLE, FLAG_CHECK_INDICES, FLAG_TEST_DROP_LOAD = 1, 2, 4, 1 << 30
DEVERR_SCORE_POOL, DEVERR_DECODE_MERGE, DEVERR_PREFILL_ATTN, DEVERR_DECODE_SELECT = 2, 3, 4, 5
DEVERR_DECODE_GATHER, DEVERR_INDEX_LIST = 6, 7
SELECT_GQA, SELECT_PER_HEAD, SELECT_ALL_HEADS = 0, 1, 2
DTYPE_BF16, DTYPE_F32, DTYPE_F16 = 0, 1, 2

EXPORTS = ("kascade_workspace_bytes", "kascade_index_count", "kascade_index_offsets",
           "kascade_workspace_init", "kascade_select", "kascade_sparse_decode",
           "kascade_sparse_prefill", "kascade_dense_ref", "kascade_workspace_error",
           "kascade_status_str", "kascade_select_decode_static", "kascade_select_decode_static_max_bytes",
           "kascade_launch_count", "kascade_select_decode_static_error", "kascade_refine_select",
           "kascade_index_overlap", "kascade_plan_anchors", "kascade_sparse_decode_paged",
           "kascade_select_varlen", "kascade_sparse_decode_varlen")


class KascadeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_str(status)} (status {status})")
        self.status = status


class Shape(ctypes.Structure):
    """kascade_shape: B, Hq, Hkv, d, q_len (1 = decode), kv_len, tile, frac."""
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("q_len", ctypes.c_int32), ("kv_len", ctypes.c_int32), ("tile", ctypes.c_int32),
                ("topk_num", ctypes.c_int32), ("topk_den", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("select_mode", ctypes.c_int32), ("dtype", ctypes.c_int32)]

    @classmethod
    def make(cls, batch, hq, hkv, d, q_len, kv_len, frac=(10, 100), tile=32, flags=0, mode=0, dtype=0):
        return cls(batch, hq, hkv, d, q_len, kv_len, tile, frac[0], frac[1], flags, mode, dtype)

    def with_flags(self, flags: int) -> "Shape":
        return Shape(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim, self.q_len,
                     self.kv_len, self.tile, self.topk_num, self.topk_den, flags, self.select_mode, self.dtype)

    @property
    def n_lists(self) -> int:
        """Index lists per batch row under the shape's selection mode."""
        return {SELECT_PER_HEAD: self.num_q_heads, SELECT_ALL_HEADS: 1}.get(self.select_mode, self.num_kv_heads)

    @property
    def decode(self) -> bool:
        return self.q_len == 1


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m sparse_attention_long_anchor_b200.build`")
    so = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    SP = ctypes.POINTER(Shape)
    so.kascade_workspace_bytes.argtypes = [SP, ctypes.c_int]
    so.kascade_workspace_bytes.restype = ctypes.c_size_t
    so.kascade_index_count.argtypes = [SP]
    so.kascade_index_count.restype = ctypes.c_int64
    so.kascade_index_offsets.argtypes = [SP, ctypes.POINTER(ctypes.c_int64)]
    so.kascade_index_offsets.restype = ctypes.c_int
    so.kascade_workspace_init.argtypes = [P, ctypes.c_size_t, P]
    so.kascade_workspace_init.restype = ctypes.c_int
    so.kascade_select.argtypes = [SP, P, P, P, P, ctypes.c_size_t, P]
    so.kascade_select.restype = ctypes.c_int
    for fn in (so.kascade_sparse_decode, so.kascade_sparse_prefill):
        fn.argtypes = [SP, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        fn.restype = ctypes.c_int
    so.kascade_dense_ref.argtypes = [SP, P, P, P, ctypes.c_int, P, P, P, ctypes.c_size_t, P]
    so.kascade_dense_ref.restype = ctypes.c_int
    so.kascade_workspace_error.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.c_int, P]
    so.kascade_workspace_error.restype = ctypes.c_int
    so.kascade_select_varlen.argtypes = [SP, P, P, P, P, P, ctypes.c_size_t, P]
    so.kascade_select_varlen.restype = ctypes.c_int
    so.kascade_sparse_decode_varlen.argtypes = [SP, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    so.kascade_sparse_decode_varlen.restype = ctypes.c_int
    so.kascade_sparse_decode_paged.argtypes = [SP, P, P, P, P, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P,
                                               ctypes.c_size_t, P]
    so.kascade_sparse_decode_paged.restype = ctypes.c_int
    so.kascade_index_overlap.argtypes = [SP, P, P, P, P]
    so.kascade_index_overlap.restype = ctypes.c_int
    so.kascade_plan_anchors.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.c_int32, ctypes.c_int32,
                                        ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)]
    so.kascade_plan_anchors.restype = ctypes.c_int
    so.kascade_refine_select.argtypes = [SP, P, P, P, ctypes.c_int32, P, P, P, ctypes.c_size_t, P]
    so.kascade_refine_select.restype = ctypes.c_int
    so.kascade_select_decode_static.argtypes = [SP, P, P, P, P]
    so.kascade_select_decode_static.restype = ctypes.c_int
    so.kascade_select_decode_static_error.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int, P]
    so.kascade_select_decode_static_error.restype = ctypes.c_int
    so.kascade_select_decode_static_max_bytes.argtypes = []
    so.kascade_select_decode_static_max_bytes.restype = ctypes.c_size_t
    so.kascade_launch_count.argtypes = [SP, ctypes.c_int]
    so.kascade_launch_count.restype = ctypes.c_int
    so.kascade_status_str.argtypes = [ctypes.c_int]
    so.kascade_status_str.restype = ctypes.c_char_p
    return so


lib = _load()


def status_str(status: int) -> str:
    return lib.kascade_status_str(status).decode()


def launch_count(shape: "Shape", op: int) -> int:
    """Kernels that `op` launches for `shape` on the current device."""
    n = lib.kascade_launch_count(ctypes.byref(shape), op)
    if n < 0:
        raise KascadeError(ERR_INVALID_ARG, "kascade_launch_count")
    return n


def _check(status: int, where: str):
    if status != OK:
        raise KascadeError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


# the raw handle of the current stream without building a Stream object
# (a per-call host cost of the eager API); the public call where absent
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def workspace_bytes(shape: Shape, op: int) -> int:
    return int(lib.kascade_workspace_bytes(ctypes.byref(shape), op))


def index_count(shape: Shape) -> int:
    n = int(lib.kascade_index_count(ctypes.byref(shape)))
    if n < 0:
        raise KascadeError(ERR_INVALID_ARG, "kascade_index_count")
    return n


def index_offsets(shape: Shape) -> np.ndarray:
    """Tile offsets of one index row (the call's tiles: a rolling chunk's own)."""
    n_t = 1 if shape.decode else -(-shape.kv_len // 32) - (shape.kv_len - shape.q_len) // 32
    out = np.zeros(n_t + 1, dtype=np.int64)
    _check(lib.kascade_index_offsets(ctypes.byref(shape), out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))),
           "kascade_index_offsets")
    return out


class Workspace:
    """A zero-initialised device workspace large enough for the given ops."""

    def __init__(self, shape: Shape, ops=(OP_SELECT, OP_SPARSE_DECODE, OP_SPARSE_PREFILL, OP_DENSE, OP_REFINE),
                 device="cuda", nbytes=None):
        need = nbytes if nbytes is not None else max([workspace_bytes(shape, op) for op in ops] + [256])
        self.buf = torch.zeros(need + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256
        self.nbytes = need

    def args(self):
        return self.ptr, self.nbytes

    def error(self, clear=True, stream=None) -> int:
        """The device error word (0 = no kernel gave up on a bounded wait)."""
        out = ctypes.c_int(0)
        _check(lib.kascade_workspace_error(self.ptr, ctypes.byref(out), int(clear), _stream(stream)),
               "kascade_workspace_error")
        return out.value


def _ws(ws, shape, op):
    if ws is None:
        if op != OP_SELECT and not shape.flags & FLAG_CHECK_INDICES:
            return None, 0       # attention calls run without an error word
        ws = Workspace(shape, (op,))
    return ws.args()


def select(shape: Shape, q, k, idx=None, ws=None, stream=None):
    """kascade_select: anchor Top-k index sets (int32, ascending)."""
    if idx is None:
        idx = torch.empty(index_count(shape), dtype=torch.int32, device=q.device)
    p, n = _ws(ws, shape, OP_SELECT)
    _check(lib.kascade_select(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(idx), p, n, _stream(stream)),
           "kascade_select")
    return idx


def refine_select(shape: Shape, q, k, pool, pool_len: int, head_map=None, idx=None, ws=None, stream=None):
    """kascade_refine_select: a refined decode layer's own Top-k from the
    proposal layer's pool [B, Hkv, pool_len]."""
    if idx is None:
        idx = torch.empty(index_count(shape), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = Workspace(shape, (OP_REFINE,))
    p, n = ws.args()
    _check(lib.kascade_refine_select(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(pool), int(pool_len),
                                     _ptr(head_map), _ptr(idx), p, n, _stream(stream)), "kascade_refine_select")
    return idx


def index_overlap(shape: Shape, a, b, counts=None, stream=None):
    """kascade_index_overlap: |a and b| per (batch row, list), summed over tiles."""
    if counts is None:
        counts = torch.empty(shape.batch * shape.n_lists, dtype=torch.int64, device=a.device)
    _check(lib.kascade_index_overlap(ctypes.byref(shape), _ptr(a), _ptr(b), _ptr(counts), _stream(stream)),
           "kascade_index_overlap")
    return counts


def plan_anchors(sim, n_anchors: int):
    """kascade_plan_anchors: (anchor layers, objective) for a host
    similarity matrix sim[a][l]."""
    sim = np.ascontiguousarray(np.asarray(sim, dtype=np.float64))
    n = sim.shape[0]
    out = (ctypes.c_int32 * max(n_anchors, 1))()
    obj = ctypes.c_double(0.0)
    _check(lib.kascade_plan_anchors(sim.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), n, n_anchors, out,
                                    ctypes.byref(obj)), "kascade_plan_anchors")
    return list(out)[:n_anchors], obj.value


def select_decode_static(shape: Shape, q, k, idx=None, stream=None):
    """kascade_select_decode_static: decode anchor selection with the library's
    fixed scratch array instead of a workspace (nothing is allocated)."""
    if idx is None:
        idx = torch.empty(index_count(shape), dtype=torch.int32, device=q.device)
    _check(lib.kascade_select_decode_static(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(idx), _stream(stream)),
           "kascade_select_decode_static")
    return idx


def select_decode_static_error(clear=True, stream=None) -> int:
    """The device error word of kascade_select_decode_static on the current
    device (0 = no kernel gave up on a bounded wait)."""
    out = ctypes.c_int(0)
    _check(lib.kascade_select_decode_static_error(ctypes.byref(out), int(clear), _stream(stream)),
           "kascade_select_decode_static_error")
    return out.value


def _attn(fn, name, shape, q, k, v, idx, head_map, o, lse, ws, stream, op):
    if o is None:
        o = torch.empty_like(q)
    p, n = _ws(ws, shape, op)
    _check(fn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(head_map), _ptr(o),
              _ptr(lse), p, n, _stream(stream)), name)
    return o


def sparse_decode(shape: Shape, q, k, v, idx, head_map=None, o=None, lse=None, ws=None, stream=None):
    """kascade_sparse_decode: kv head h attends over anchor list head_map[h]."""
    return _attn(lib.kascade_sparse_decode, "kascade_sparse_decode", shape, q, k, v, idx, head_map, o, lse,
                 ws, stream, OP_SPARSE_DECODE)


def select_varlen(shape: Shape, q, k, kv_lens, idx=None, ws=None, stream=None):
    """kascade_select_varlen: decode selection with a context length per batch
    row (lists padded with -1 to the layout of kv_len)."""
    if idx is None:
        idx = torch.empty(index_count(shape), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = Workspace(shape, (OP_SELECT_VARLEN,))
    p, n = ws.args()
    _check(lib.kascade_select_varlen(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(kv_lens), _ptr(idx), p, n,
                                     _stream(stream)), "kascade_select_varlen")
    return idx


def sparse_decode_varlen(shape: Shape, q, k, v, kv_lens, idx, head_map=None, o=None, lse=None, ws=None,
                         stream=None):
    """kascade_sparse_decode_varlen: sparse (idx None: dense) decode with a
    context length per batch row."""
    if o is None:
        o = torch.empty_like(q)
    p, n = _ws(ws, shape, OP_SPARSE_DECODE)
    _check(lib.kascade_sparse_decode_varlen(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens),
                                            _ptr(idx), _ptr(head_map), _ptr(o), _ptr(lse), p, n, _stream(stream)),
           "kascade_sparse_decode_varlen")
    return o


def sparse_decode_paged(shape: Shape, q, k_pages, v_pages, page_table, page_size: int, idx, head_map=None, o=None,
                        lse=None, ws=None, stream=None):
    """kascade_sparse_decode_paged: sparse (or, with idx None, dense) decode
    over pages [num_pages, Hkv, page_size, d] named by page_table [B, max_pages]."""
    if o is None:
        o = torch.empty_like(q)
    p, n = _ws(ws, shape, OP_SPARSE_DECODE)
    _check(lib.kascade_sparse_decode_paged(ctypes.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                                           _ptr(page_table), int(page_size), int(page_table.shape[-1]), _ptr(idx),
                                           _ptr(head_map), _ptr(o), _ptr(lse), p, n, _stream(stream)),
           "kascade_sparse_decode_paged")
    return o


def sparse_prefill(shape: Shape, q, k, v, idx, head_map=None, o=None, lse=None, ws=None, stream=None):
    """kascade_sparse_prefill: causal tile-level sparse attention."""
    return _attn(lib.kascade_sparse_prefill, "kascade_sparse_prefill", shape, q, k, v, idx, head_map, o,
                 lse, ws, stream, OP_SPARSE_PREFILL)


def dense_ref(shape: Shape, q, k, v, causal=True, o=None, lse=None, ws=None, stream=None):
    """kascade_dense_ref: dense (causal) attention."""
    if o is None:
        o = torch.empty_like(q)
    p, n = _ws(ws, shape, OP_DENSE)
    _check(lib.kascade_dense_ref(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), int(bool(causal)), _ptr(o),
                                 _ptr(lse), p, n, _stream(stream)), "kascade_dense_ref")
    return o
