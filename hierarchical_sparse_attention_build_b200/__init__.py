"""Python binding of librecsa: RecSA tree build and level-wise sparse attend on B200.

Thin ctypes marshalling over the C ABI declared in ``include/recsa.h``; every step of
the computation runs in the library's CUDA kernels.  PyTorch supplies device memory
and the current CUDA stream.  Importing this module fails loudly when the compiled
library is missing: there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librecsa.so")

HEAD_DIM = 128
TOPK_ALL = 0x7FFFFFFF
MAX_LEVELS = 40
MAX_CANDIDATES = 4096

STATUS = {
    0: "RECSA_OK",
    1: "RECSA_ERR_INVALID_ARGUMENT",
    2: "RECSA_ERR_UNSUPPORTED",
    3: "RECSA_ERR_WORKSPACE_TOO_SMALL",
    4: "RECSA_ERR_CAPACITY",
    5: "RECSA_ERR_CUDA",
    6: "RECSA_ERR_DEVICE_CHECK",
    7: "RECSA_ERR_TIMEOUT",
}


class RecsaError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS.get(code, code)}: {message}")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("branching", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("rope_base", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
    ]


class Tree(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
        ("length", ctypes.c_int64),
        ("k_tok", ctypes.c_void_p),
        ("v_tok", ctypes.c_void_p),
        ("k_node", ctypes.c_void_p),
        ("v_node", ctypes.c_void_p),
        ("pooler", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
    ]


class Debug(ctypes.Structure):
    _fields_ = [
        ("sel_idx", ctypes.c_void_p),
        ("entries", ctypes.c_void_p),
        ("sel_levels", ctypes.c_int32),
        ("kernel", ctypes.c_int32),
        ("cluster_size", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


KERNEL_AUTO, KERNEL_CTA, KERNEL_WARP, KERNEL_LEAN = 0, 1, 2, 3


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -c 'import __graft_entry__ as g; g.build()'` (nvcc, sm_100a)"
        )
    lib = ctypes.CDLL(LIB_PATH)
    P, T, D = ctypes.POINTER(Params), ctypes.POINTER(Tree), ctypes.POINTER(Debug)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "recsa_tree_layout": [P, i32, i64, ctypes.POINTER(i64), ctypes.POINTER(i32), ctypes.POINTER(i64)],
        "recsa_workspace_size": [P, i64, ctypes.POINTER(sz)],
        "recsa_workspace_init": [P, i64, vp, sz, vp],
        "recsa_build_tree": [P, T, vp],
        "recsa_decode": [P, T, vp, i32, vp, i32, vp, sz, D, vp],
        "recsa_decode_host": [P, T, vp, i32, vp, i32, vp, vp, vp, sz, D, vp],
        "recsa_append": [P, T, vp, vp, i32, vp],
        "recsa_decode_step": [P, T, vp, vp, vp, vp, i32, vp, sz, vp],
        "recsa_prefill_chunk": [P, T, vp, vp, vp, i32, vp, i32, vp, sz, D, vp],
        "recsa_check_device_errors": [vp, vp],
        "recsa_decode_no_alloc": [P, T, vp, i32, vp, i32, vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.recsa_status_string.argtypes = [ctypes.c_int]
    lib.recsa_status_string.restype = ctypes.c_char_p
    lib.recsa_last_error.argtypes = []
    lib.recsa_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def _check(code: int) -> None:
    if code != 0:
        raise RecsaError(code, _lib.recsa_last_error().decode())


def _stream(stream=None) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t) -> ctypes.c_void_p | None:
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def params(num_kv_heads: int, num_q_heads: int, branching: int, top_k: int, rope_base: float = 1.0e6,
           softmax_scale: float = 0.0, head_dim: int = HEAD_DIM) -> Params:
    return Params(head_dim, num_kv_heads, num_q_heads, branching, top_k, rope_base, softmax_scale)


def tree_layout(p: Params, batch: int, capacity: int):
    """(node_rows, levels, level_row_offsets[0..levels]) of the node arena."""
    rows = ctypes.c_int64()
    levels = ctypes.c_int32()
    offs = (ctypes.c_int64 * (MAX_LEVELS + 1))()
    _check(_lib.recsa_tree_layout(ctypes.byref(p), batch, capacity, ctypes.byref(rows), ctypes.byref(levels), offs))
    return rows.value, levels.value, list(offs[: levels.value + 1])


def workspace_size(p: Params, capacity: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib.recsa_workspace_size(ctypes.byref(p), capacity, ctypes.byref(n)))
    return n.value


class RecsaTree:
    """A layer's token caches plus its node arena (torch tensors) and the C struct over them."""

    def __init__(self, p: Params, k_tok: torch.Tensor, v_tok: torch.Tensor, pooler: torch.Tensor, length: int,
                 k_node: torch.Tensor | None = None, v_node: torch.Tensor | None = None,
                 seq_len: torch.Tensor | None = None, page_table: torch.Tensor | None = None):
        """k_tok, v_tok: contiguous caches [batch][Hkv][capacity][128], or with page_table (int32
        [batch][pages per sequence] device tensor) a page pool [num_pages][Hkv][page_size][128].
        seq_len: optional int64 [batch] device tensor of per-sequence lengths (length is then
        the longest); the library advances it on the device when it appends."""
        assert k_tok.dtype == torch.bfloat16 and v_tok.dtype == torch.bfloat16 and pooler.dtype == torch.float32
        assert k_tok.is_contiguous() and v_tok.is_contiguous() and pooler.is_contiguous()
        assert v_tok.shape == k_tok.shape and k_tok.shape[3] == HEAD_DIM and k_tok.shape[1] == p.num_kv_heads
        if page_table is None:
            batch, _, capacity, _ = k_tok.shape
            num_pages = page_size = 0
        else:
            assert page_table.dtype == torch.int32 and page_table.is_contiguous() and page_table.dim() == 2
            num_pages, _, page_size, _ = k_tok.shape
            batch = page_table.shape[0]
            capacity = page_table.shape[1] * page_size
        self.p = p
        rows, self.levels, self.level_offsets = tree_layout(p, batch, capacity)
        if k_node is None:
            k_node = torch.empty(max(rows, 1), HEAD_DIM, dtype=torch.bfloat16, device=k_tok.device)
            v_node = torch.empty_like(k_node)
        self.k_tok, self.v_tok, self.k_node, self.v_node, self.pooler = k_tok, v_tok, k_node, v_node, pooler
        self.node_rows = rows
        if seq_len is not None:
            assert seq_len.dtype == torch.int64 and seq_len.is_contiguous() and seq_len.numel() == batch
        self.seq_len = seq_len
        self.page_table = page_table
        self.c = Tree(batch, 0, capacity, length, k_tok.data_ptr(), v_tok.data_ptr(), k_node.data_ptr(),
                      v_node.data_ptr(), pooler.data_ptr(), seq_len.data_ptr() if seq_len is not None else None,
                      page_table.data_ptr() if page_table is not None else None, page_size, num_pages)

    @property
    def length(self) -> int:
        return self.c.length

    @length.setter
    def length(self, v: int) -> None:
        self.c.length = v

    @property
    def batch(self) -> int:
        return self.c.batch

    @property
    def capacity(self) -> int:
        return self.c.capacity

    def level_rows(self, level: int) -> torch.Tensor:
        """Node-arena rows of `level` as [batch][Hkv][slots][128] views (K, V)."""
        slots = -(-self.capacity // self.p.branching ** level)
        o = self.level_offsets[level]
        n = self.batch * self.p.num_kv_heads * slots
        shape = (self.batch, self.p.num_kv_heads, slots, HEAD_DIM)
        return self.k_node[o:o + n].view(shape), self.v_node[o:o + n].view(shape)


class Workspace:
    """Device workspace (RoPE table + error word) initialised for a params/capacity pair."""

    def __init__(self, p: Params, capacity: int, device, stream=None, buffer: torch.Tensor | None = None):
        self.nbytes = workspace_size(p, capacity)
        self.buf = buffer if buffer is not None else torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        workspace_init(p, capacity, self.buf, stream)


def workspace_init(p: Params, capacity: int, buf: torch.Tensor, stream=None) -> None:
    _check(_lib.recsa_workspace_init(ctypes.byref(p), capacity, _ptr(buf), buf.numel() * buf.element_size(),
                                     _stream(stream)))


def build_tree(p: Params, tree: RecsaTree, stream=None) -> None:
    _check(_lib.recsa_build_tree(ctypes.byref(p), ctypes.byref(tree.c), _stream(stream)))


def _debug(sel_idx=None, sel_levels=0, cluster_size=0, entries=None, kernel=0):
    if sel_idx is None and entries is None and cluster_size == 0 and kernel == 0:
        return None
    return Debug(sel_idx.data_ptr() if sel_idx is not None else None,
                 entries.data_ptr() if entries is not None else None, sel_levels, kernel, cluster_size, 0)


def decode(p: Params, tree: RecsaTree, q: torch.Tensor, out: torch.Tensor, ws: Workspace, sel_idx=None,
           sel_levels: int = 0, entries=None, cluster_size: int = 0, kernel: int = 0, stream=None) -> None:
    """recsa_decode: q [B][Q][Hq][128] bf16 -> out [B][Q][Hq][128] (fp32 or bf16)."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and out.is_contiguous()
    nq = q.shape[1]
    dbg = _debug(sel_idx, sel_levels, cluster_size, entries, kernel)
    _check(_lib.recsa_decode(ctypes.byref(p), ctypes.byref(tree.c), _ptr(q), nq, _ptr(out),
                             int(out.dtype == torch.float32), _ptr(ws.buf), ws.nbytes,
                             ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))


def decode_host(p: Params, tree: RecsaTree, q_host: torch.Tensor, out_host: torch.Tensor, q_dev: torch.Tensor,
                out_dev: torch.Tensor, ws: Workspace, stream=None) -> None:
    """recsa_decode_host: host q -> device staging -> decode -> host out, queued in one call."""
    for t in (q_host, out_host):
        assert t.device.type == "cpu" and t.is_contiguous()
    assert q_host.dtype == torch.bfloat16 and q_dev.shape == q_host.shape and out_dev.shape == out_host.shape
    assert out_dev.dtype == out_host.dtype and q_dev.is_contiguous() and out_dev.is_contiguous()
    _check(_lib.recsa_decode_host(ctypes.byref(p), ctypes.byref(tree.c), _ptr(q_host), q_host.shape[1],
                                  _ptr(out_host), int(out_host.dtype == torch.float32), _ptr(q_dev), _ptr(out_dev),
                                  _ptr(ws.buf), ws.nbytes, None, _stream(stream)))


def append(p: Params, tree: RecsaTree, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
    """recsa_append: append [B][C][Hkv][128] K/V to every sequence and rebuild the nodes over them."""
    for t in (k_new, v_new):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    _check(_lib.recsa_append(ctypes.byref(p), ctypes.byref(tree.c), _ptr(k_new), _ptr(v_new), k_new.shape[1],
                             _stream(stream)))


def decode_step(p: Params, tree: RecsaTree, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                out: torch.Tensor, ws: Workspace, stream=None) -> None:
    """recsa_decode_step: append one token per sequence at its device length, advance the
    lengths, decode the token's query; graph-capturable (needs tree.seq_len)."""
    for t in (k_new, v_new, q):
        assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.shape[1] == 1
    _check(_lib.recsa_decode_step(ctypes.byref(p), ctypes.byref(tree.c), _ptr(k_new), _ptr(v_new), _ptr(q),
                                  _ptr(out), int(out.dtype == torch.float32), _ptr(ws.buf), ws.nbytes,
                                  _stream(stream)))


def prefill_chunk(p: Params, tree: RecsaTree, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                  out: torch.Tensor, ws: Workspace, sel_idx=None, sel_levels: int = 0, entries=None,
                  cluster_size: int = 0, kernel: int = 0, stream=None) -> None:
    """recsa_prefill_chunk: append [B][C][Hkv][128] K/V, extend the tree, attend the C queries causally."""
    for t in (k_new, v_new, q):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    chunk = q.shape[1]
    dbg = _debug(sel_idx, sel_levels, cluster_size, entries, kernel)
    _check(_lib.recsa_prefill_chunk(ctypes.byref(p), ctypes.byref(tree.c), _ptr(k_new), _ptr(v_new), _ptr(q), chunk,
                                    _ptr(out), int(out.dtype == torch.float32), _ptr(ws.buf), ws.nbytes,
                                    ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))


def decode_no_alloc(p: Params, tree: RecsaTree, q: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """recsa_decode_no_alloc: recsa_decode with its scratch in the library's fixed device array."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and out.is_contiguous()
    _check(_lib.recsa_decode_no_alloc(ctypes.byref(p), ctypes.byref(tree.c), _ptr(q), q.shape[1], _ptr(out),
                                      int(out.dtype == torch.float32), _stream(stream)))


def check_device_errors(ws: Workspace, stream=None) -> None:
    _check(_lib.recsa_check_device_errors(_ptr(ws.buf), _stream(stream)))


def status_string(code: int) -> str:
    return _lib.recsa_status_string(code).decode()


def last_error() -> str:
    return _lib.recsa_last_error().decode()


def raw_library() -> ctypes.CDLL:
    """The loaded CDLL (for callers that marshal their own arguments)."""
    return _lib
