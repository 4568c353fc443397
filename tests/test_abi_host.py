"""Host-side checks of the C ABI (no CUDA device needed, no kernel launched).

Every call here fails argument validation before the library touches CUDA, or is a
pure host computation (layout, workspace size), so these run on any machine.
"""

import ctypes
import os
import re

import pytest

import hierarchical_sparse_attention_build_b200 as R
from oracle import recsa_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "recsa.h")
lib = R.raw_library()

OK, INVALID, UNSUPPORTED, WS_SMALL, CAPACITY = 0, 1, 2, 3, 4
FAKE = 0x7F0000000000  # aligned, never dereferenced: every call below fails validation first


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"RECSA_API\s+[^;()]*?\b(recsa_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert set(names) == {"recsa_tree_layout", "recsa_workspace_size", "recsa_workspace_init", "recsa_build_tree",
                          "recsa_decode", "recsa_prefill_chunk", "recsa_check_device_errors", "recsa_status_string",
                          "recsa_last_error", "recsa_decode_no_alloc", "recsa_decode_host", "recsa_append",
                          "recsa_decode_step"}, names
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings():
    for code, name in R.STATUS.items():
        assert R.status_string(code) == name


def _p(**kw):
    d = dict(num_kv_heads=8, num_q_heads=32, branching=16, top_k=8)
    d.update(kw)
    return R.params(**d)


@pytest.mark.parametrize("cap,b", [(4096, 8), (1 << 20, 16), (532480, 16), (2 << 20, 16), (17, 16), (1000, 3),
                                   (16, 16), (5, 2)])
def test_tree_layout_matches_level_counts(cap, b):
    p = _p(branching=b, num_kv_heads=2, num_q_heads=8)
    batch = 3
    rows, levels, offs = R.tree_layout(p, batch, cap)
    want = O.level_counts(cap, b)  # independent statement of the level rule
    assert levels == len(want) - 1
    acc = 0
    for l in range(1, levels + 1):
        assert offs[l] == acc
        acc += batch * 2 * want[l]
    assert rows == acc


def test_workspace_size_covers_positions():
    # RoPE positions 0 .. max(b, min((k+1)*b, capacity)), capped at the candidate limit
    p = _p()
    assert R.workspace_size(p, 1 << 20) == 256 + (9 * 16 + 1) * 64 * 8
    assert R.workspace_size(_p(top_k=R.TOPK_ALL, branching=8), 4096) == 256 + (4096 + 1) * 64 * 8
    assert R.workspace_size(_p(top_k=0), 100) == 256 + (16 + 1) * 64 * 8


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), UNSUPPORTED),
    (dict(num_q_heads=30), INVALID),
    (dict(num_q_heads=8 * 16), UNSUPPORTED),
    (dict(branching=1), INVALID),
    (dict(top_k=-1), INVALID),
    (dict(rope_base=0.0), INVALID),
    (dict(softmax_scale=-1.0), INVALID),
])
def test_bad_params_rejected(kw, code):
    p = _p(**kw)
    n = ctypes.c_size_t()
    assert lib.recsa_workspace_size(ctypes.byref(p), 4096, ctypes.byref(n)) == code
    assert R.last_error()


def _tree(**kw):
    d = dict(batch=1, reserved=0, capacity=4096, length=4096, k_tok=FAKE, v_tok=FAKE, k_node=FAKE, v_node=FAKE,
             pooler=FAKE)
    d.update(kw)
    return R.Tree(**d)


def _decode(p, t, q=FAKE, nq=1, out=FAKE, ws=FAKE, ws_bytes=1 << 30, dbg=None):
    return lib.recsa_decode(ctypes.byref(p), ctypes.byref(t), q, nq, out, 1, ws, ws_bytes,
                            ctypes.byref(dbg) if dbg else None, None)


@pytest.mark.parametrize("tkw,code", [
    (dict(k_tok=0), INVALID),
    (dict(v_node=0), INVALID),
    (dict(pooler=0), INVALID),
    (dict(k_node=FAKE + 8), INVALID),
    (dict(length=0), INVALID),
    (dict(length=5000), INVALID),
    (dict(batch=0), INVALID),
    (dict(capacity=(1 << 30) + 1, length=1), UNSUPPORTED),
])
def test_decode_bad_tree_rejected(tkw, code):
    assert _decode(_p(), _tree(**tkw)) == code


def test_decode_host_checks_everything_before_queuing():
    # each of these fails validation, so no copy is queued and no CUDA call is made
    p, t = _p(), _tree()
    host = ctypes.create_string_buffer(64)

    def call(q_host=host, out_host=host, q_dev=FAKE, out_dev=FAKE, ws_bytes=1 << 30, p=p, t=t, nq=1):
        return lib.recsa_decode_host(ctypes.byref(p), ctypes.byref(t), q_host, nq, out_host, 1, q_dev, out_dev,
                                     FAKE, ws_bytes, None, None)

    assert call(q_host=None) == INVALID
    assert call(out_host=None) == INVALID
    assert call(q_dev=0) == INVALID
    assert call(out_dev=FAKE + 8) == INVALID
    assert call(nq=0) == INVALID
    assert call(ws_bytes=100) == WS_SMALL
    assert call(p=_p(num_q_heads=30)) == INVALID
    assert call(t=_tree(length=0)) == INVALID


def test_decode_bad_call_arguments_rejected():
    p, t = _p(), _tree()
    assert _decode(p, t, q=0) == INVALID
    assert _decode(p, t, out=FAKE + 4) == INVALID
    assert _decode(p, t, nq=0) == INVALID
    assert _decode(p, t, ws=0) == INVALID
    assert _decode(p, t, ws_bytes=100) == WS_SMALL
    assert _decode(_p(top_k=65), t, dbg=R.Debug(FAKE, 0, 4, 0, 0, 0), ws_bytes=100) == WS_SMALL
    p65 = _p(top_k=65)
    ws = R.workspace_size(p65, 4096)
    assert _decode(p65, t, dbg=R.Debug(FAKE, 0, 4, 0, 0, 0), ws_bytes=ws) == INVALID
    assert _decode(p, t, dbg=R.Debug(0, 0, 0, 0, 3, 0), ws_bytes=R.workspace_size(p, 4096)) == INVALID
    assert _decode(p, t, dbg=R.Debug(0, 0, 0, 5, 0, 0), ws_bytes=R.workspace_size(p, 4096)) == INVALID
    # k = all at a long context needs more candidates per level than the kernel holds
    pall = _p(top_k=R.TOPK_ALL)
    big = _tree(capacity=1 << 16, length=1 << 16)
    assert _decode(pall, big, ws_bytes=R.workspace_size(pall, 1 << 16)) == UNSUPPORTED


def test_prefill_capacity_and_arguments_rejected():
    p = _p()
    t = _tree(length=4000)
    ws = R.workspace_size(p, 4096)
    call = lambda t, chunk=64, **kw: lib.recsa_prefill_chunk(
        ctypes.byref(p), ctypes.byref(t), kw.get("k", FAKE), kw.get("v", FAKE), kw.get("q", FAKE), chunk,
        kw.get("out", FAKE), 1, FAKE, kw.get("ws", ws), None, None)
    assert call(t, chunk=200) == CAPACITY
    assert call(t, chunk=0) == INVALID
    assert call(t, k=0) == INVALID
    assert call(t, v=FAKE + 2) == INVALID
    assert call(t, ws=10) == WS_SMALL
    assert t.length == 4000  # unchanged on failure


def test_append_capacity_and_arguments_rejected():
    p = _p()
    t = _tree(length=4000)
    call = lambda t, count=64, **kw: lib.recsa_append(ctypes.byref(p), ctypes.byref(t), kw.get("k", FAKE),
                                                      kw.get("v", FAKE), count, None)
    assert call(t, count=97) == CAPACITY
    assert call(t, count=0) == INVALID
    assert call(t, count=-3) == INVALID
    assert call(t, k=0) == INVALID
    assert call(t, v=FAKE + 8) == INVALID
    assert call(_tree(length=4000, k_node=0)) == INVALID
    assert call(_tree(length=4000, seq_len=FAKE + 4)) == INVALID  # per-sequence lengths need 8-byte alignment
    assert lib.recsa_append(ctypes.byref(_p(top_k=-1)), ctypes.byref(t), FAKE, FAKE, 1, None) == INVALID
    assert t.length == 4000  # unchanged on failure


@pytest.mark.parametrize("kw", [
    dict(page_size=3),                     # not a power of two
    dict(page_size=0),
    dict(page_size=1 << 17),               # above 65536
    dict(page_size=8, capacity=4100),      # capacity not a multiple of the page size
    dict(page_size=8, num_pages=0),
    dict(page_size=8, page_table=FAKE + 2),  # misaligned table
])
def test_paged_cache_arguments_rejected(kw):
    p = _p()
    d = dict(length=100, page_table=FAKE, page_size=8, num_pages=16)
    d.update(kw)
    assert lib.recsa_build_tree(ctypes.byref(p), ctypes.byref(_tree(**d)), None) == INVALID


def test_decode_step_checks_everything_before_queuing():
    p = _p()
    ws = R.workspace_size(p, 4096)
    call = lambda t, **kw: lib.recsa_decode_step(ctypes.byref(p), ctypes.byref(t), kw.get("k", FAKE), kw.get("v", FAKE),
                                                 kw.get("q", FAKE), kw.get("out", FAKE), 1, FAKE, kw.get("ws", ws), None)
    assert call(_tree(length=100)) == INVALID                     # no per-sequence lengths
    with_len = _tree(length=100, seq_len=FAKE)
    assert call(with_len, q=0) == INVALID
    assert call(with_len, k=FAKE + 4) == INVALID
    assert call(with_len, ws=10) == WS_SMALL
    assert call(_tree(length=100, seq_len=FAKE + 4)) == INVALID   # misaligned lengths


def test_layout_and_build_reject_bad_input():
    p = _p()
    rows = ctypes.c_int64()
    lv = ctypes.c_int32()
    offs = (ctypes.c_int64 * 41)()
    assert lib.recsa_tree_layout(ctypes.byref(p), 0, 100, ctypes.byref(rows), ctypes.byref(lv), offs) == INVALID
    assert lib.recsa_tree_layout(ctypes.byref(p), 1, 0, ctypes.byref(rows), ctypes.byref(lv), offs) == INVALID
    assert lib.recsa_build_tree(ctypes.byref(p), ctypes.byref(_tree(v_tok=0)), None) == INVALID
    assert lib.recsa_build_tree(ctypes.byref(p), None, None) == INVALID
    assert lib.recsa_check_device_errors(None, None) == INVALID
    assert lib.recsa_workspace_init(ctypes.byref(p), 4096, FAKE, 10, None) == WS_SMALL
