"""The C ABI without a GPU: the library loads, exports what include/gdr.h
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_147_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")

# fake, 16-byte aligned device addresses: validation fails before they are used
P = 1 << 20
NULL = None


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:gdr_status|const char\*|int|size_t)\s+(gdr_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.gdr_version() == (1 << 16)
    assert _lib.status_string(0) == "GDR_OK"
    assert _lib.status_string(3) == "GDR_ERR_MISALIGNED"


def test_library_is_in_tree():
    assert os.path.dirname(_lib.library_path()) == os.path.join(ROOT, "gated_delta_rule_147_b200")


def chunk(**kw):
    a = dict(q=P, k=P, v=P, alpha=P, b=P, w=NULL, ak=1, bk=1, wk=3, S0=NULL, o=P, ST=P, ws=NULL,
             ws_bytes=0, B=1, T=64, H=1, dk=128, dv=128, chunk=64, dtype=0)
    a.update(kw)
    lib = _lib.load()
    return lib.gdr_chunk_fwd(a["q"], a["k"], a["v"], a["alpha"], a["b"], a["w"], a["ak"], a["bk"],
                             a["wk"], a["S0"], a["o"], a["ST"], a["ws"], a["ws_bytes"], a["B"],
                             a["T"], a["H"], a["dk"], a["dv"], a["chunk"], a["dtype"], None, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), _lib.GDR_ERR_INVALID_ARG),
    (dict(H=0), _lib.GDR_ERR_INVALID_ARG),
    (dict(T=-1), _lib.GDR_ERR_INVALID_ARG),
    (dict(dk=0), _lib.GDR_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.GDR_ERR_INVALID_ARG),
    (dict(ak=9), _lib.GDR_ERR_INVALID_ARG),
    (dict(ak=3), _lib.GDR_ERR_INVALID_ARG),             # alpha cannot be tied
    (dict(alpha=NULL), _lib.GDR_ERR_INVALID_ARG),        # scalar alpha needs data
    (dict(ak=0), _lib.GDR_ERR_INVALID_ARG),              # NONE alpha must be NULL
    (dict(w=P), _lib.GDR_ERR_INVALID_ARG),               # tied w must be NULL
    (dict(bk=0, b=NULL), _lib.GDR_ERR_INVALID_ARG),      # tied to an absent b
    (dict(q=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(o=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(chunk=32), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dtype=1, dk=512), _lib.GDR_ERR_UNSUPPORTED),
    (dict(q=P + 8), _lib.GDR_ERR_MISALIGNED),
    (dict(o=P + 2), _lib.GDR_ERR_MISALIGNED),
    (dict(ST=P + 4), _lib.GDR_ERR_MISALIGNED),
    (dict(ak=2, alpha=P + 2), _lib.GDR_ERR_MISALIGNED),
    (dict(ws=P, ws_bytes=1024), _lib.GDR_ERR_INVALID_ARG),          # workspace too small
    (dict(ws=P + 16, ws_bytes=1 << 30), _lib.GDR_ERR_MISALIGNED),   # workspace not 256-aligned
])
def test_chunk_fwd_rejects_bad_arguments(kw, expect):
    assert chunk(**kw) == expect


def decode(**kw):
    a = dict(q=P, k=P, v=P, alpha=P, b=P, w=P, ak=2, bk=2, wk=2, S=P, o=P, B=2, H=2, dk=128, dv=128,
             dtype=0)
    a.update(kw)
    return _lib.load().gdr_decode_step(a["q"], a["k"], a["v"], a["alpha"], a["b"], a["w"], a["ak"],
                                       a["bk"], a["wk"], a["S"], a["o"], a["B"], a["H"], a["dk"],
                                       a["dv"], a["dtype"], None, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), _lib.GDR_ERR_INVALID_ARG),
    (dict(S=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(wk=3), _lib.GDR_ERR_INVALID_ARG),              # tied w must be NULL
    (dict(bk=5), _lib.GDR_ERR_INVALID_ARG),
    (dict(dv=48), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dk=512), _lib.GDR_ERR_UNSUPPORTED),
    (dict(S=P + 4), _lib.GDR_ERR_MISALIGNED),
])
def test_decode_step_rejects_bad_arguments(kw, expect):
    assert decode(**kw) == expect


def test_binding_raises_on_error_status():
    with pytest.raises(_lib.GdrError):
        _lib.gdr_chunk_fwd(P, P, P, P, P, None, 1, 1, 3, None, P, P, None, 0, 0, 64, 1, 128, 128,
                           64, 0, stream=0)


@pytest.mark.parametrize("shape,kinds,expect", [
    # GDN form: per-token rows of -W (d_k), P (d_v) and the chunk's Aq block (64)
    ((4, 4096, 16, 128, 128), (1, 1, 3), 4 * 4096 * 16 * (128 + 128 + 64) * 2),
    ((1, 100, 2, 128, 64), (1, 1, 3), 1 * 100 * 2 * (128 + 64 + 64) * 2),
    ((1, 64, 1, 128, 256), (1, 1, 3), 0),          # d_v > 128: single pass only
    # d_k = 256, GDN form: -W (256), P (d_v), Aq (64) and K~ = Diag(g_{n-1}/g) K (256)
    ((2, 100, 3, 256, 256), (1, 1, 3), 2 * 100 * 3 * (256 + 256 + 64 + 256) * 2),
    ((1, 65, 1, 256, 64), (1, 1, 3), 65 * (256 + 64 + 64 + 256) * 2),
    ((1, 64, 1, 256, 320), (1, 1, 3), 0),          # d_v > 256: exact path
    ((1, 64, 1, 256, 128), (2, 1, 3), 0),          # d_k = 256, other gate forms: exact path
    ((1, 64, 1, 128, 128), (2, 1, 3), 3 * 16384 + 8192 + 16384 + 512 + 65536),   # KDA form
    ((1, 100, 2, 128, 64), (2, 2, 2), 4 * 51200 + 3 * 25600 + 2048 + 65536),      # GDN-2 form
    ((1, 64, 1, 128, 128), (2, 0, 0), 0),          # no erase: single pass only
    ((1, 64, 1, 64, 64), (1, 1, 3), 0),            # not the tensor-core shape
    ((1, 0, 1, 128, 128), (1, 1, 3), 0),
])
def test_workspace_size(shape, kinds, expect):
    B, T, H, dk, dv = shape
    assert _lib.gdr_chunk_fwd_workspace_size(B, T, H, dk, dv, *kinds, 0) == expect


def test_grouped_entry_points_reject_bad_head_counts():
    lib = _lib.load()
    st = lib.gdr_chunk_fwd_grouped(P, P, P, P, P, None, 1, 1, 3, None, P, P, None, 0,
                                   1, 64, 3, 4, 128, 128, 64, 0, None, None)   # 4 % 3 != 0
    assert st == _lib.GDR_ERR_INVALID_ARG
    st = lib.gdr_chunk_fwd_grouped(P, P, P, P, P, None, 1, 1, 3, None, P, P, None, 0,
                                   1, 64, 0, 4, 128, 128, 64, 0, None, None)   # H_qk = 0
    assert st == _lib.GDR_ERR_INVALID_ARG
    st = lib.gdr_decode_step_grouped(P, P, P, P, P, P, 2, 2, 2, P, P, 2, 3, 4, 128, 128, 0,
                                     None, None)
    assert st == _lib.GDR_ERR_INVALID_ARG


def bwd(**kw):
    a = dict(q=P, k=P, v=P, alpha=P, b=P, w=NULL, ak=1, bk=1, wk=3, S0=NULL, dO=P, dST=NULL, dq=P,
             dk_=P, dv_=P, dal=P, db=P, dw=NULL, dS0=P, ws=P, ws_bytes=1 << 30, B=1, T=64, H=1,
             dk=128, dv=128, chunk=64, dtype=0)
    a.update(kw)
    return _lib.load().gdr_chunk_bwd(a["q"], a["k"], a["v"], a["alpha"], a["b"], a["w"], a["ak"],
                                     a["bk"], a["wk"], a["S0"], a["dO"], a["dST"], a["dq"],
                                     a["dk_"], a["dv_"], a["dal"], a["db"], a["dw"], a["dS0"],
                                     a["ws"], a["ws_bytes"], a["B"], a["T"], a["H"], a["dk"],
                                     a["dv"], a["chunk"], a["dtype"], None, None)


# every case fails on the host, before any launch
@pytest.mark.parametrize("kw,expect", [
    (dict(B=0), _lib.GDR_ERR_INVALID_ARG),
    (dict(T=-1), _lib.GDR_ERR_INVALID_ARG),
    (dict(dtype=3), _lib.GDR_ERR_INVALID_ARG),
    (dict(dO=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(dq=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(dal=NULL), _lib.GDR_ERR_INVALID_ARG),          # scalar alpha needs its gradient
    (dict(dw=P), _lib.GDR_ERR_INVALID_ARG),              # tied w has no gradient of its own
    (dict(ak=0, alpha=NULL), _lib.GDR_ERR_INVALID_ARG),  # absent alpha: dalpha must be NULL
    (dict(ws=NULL), _lib.GDR_ERR_INVALID_ARG),
    (dict(ws_bytes=1024), _lib.GDR_ERR_INVALID_ARG),     # workspace too small
    (dict(chunk=32), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dk=320), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dv=264), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dv=44), _lib.GDR_ERR_UNSUPPORTED),
    (dict(dO=P + 8), _lib.GDR_ERR_MISALIGNED),
    (dict(dS0=P + 4), _lib.GDR_ERR_MISALIGNED),
    (dict(ws=P + 16), _lib.GDR_ERR_MISALIGNED),
])
def test_chunk_bwd_rejects_bad_arguments(kw, expect):
    assert bwd(**kw) == expect


def r256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("shape,expect", [
    # checkpoints of S and G, r and dr per token, scalar-gate partials (16 row blocks of
    # 8), and at d_k = d_v = 128 the forward's -W and P rows (bf16)
    ((4, 4096, 16, 128, 128), 2 * 4 * 16 * 64 * 128 * 128 * 4 + 2 * 4 * 4096 * 16 * 128 * 4
     + 3 * 16 * 4 * 4096 * 16 * 4 + 4 * 4096 * 16 * (128 + 128 + 64) * 2),
    # d_v = 32: 4 threads per row, 32 rows per block, 2 blocks
    ((1, 65, 2, 64, 32), 2 * 2 * 2 * 64 * 32 * 4 + 2 * r256(65 * 2 * 32 * 4) + r256(3 * 2 * 65 * 2 * 4)),
    ((1, 0, 2, 64, 32), 0),
])
def test_bwd_workspace_size(shape, expect):
    assert _lib.gdr_chunk_bwd_workspace_size(*shape) == expect


def test_grouped_backward_rejects_bad_head_counts_and_sizes_its_workspace():
    lib = _lib.load()
    args = [P, P, P, P, P, None, 1, 1, 3, None, P, None, P, P, P, P, P, None, P, P, 1 << 30]
    st = lib.gdr_chunk_bwd_grouped(*args, 1, 64, 3, 4, 128, 128, 64, 0, None, None)  # 4 % 3 != 0
    assert st == _lib.GDR_ERR_INVALID_ARG
    st = lib.gdr_chunk_bwd_grouped(*args, 1, 64, 0, 4, 128, 128, 64, 0, None, None)  # H_qk = 0
    assert st == _lib.GDR_ERR_INVALID_ARG
    base = _lib.gdr_chunk_bwd_grouped_workspace_size(1, 64, 4, 4, 128, 128)
    assert base == _lib.gdr_chunk_bwd_workspace_size(1, 64, 4, 128, 128)
    # grouped: per-value-head dq and dk in the workspace
    assert _lib.gdr_chunk_bwd_grouped_workspace_size(1, 64, 2, 4, 128, 128) == base + 2 * 64 * 4 * 128 * 4
    assert _lib.gdr_chunk_bwd_grouped_workspace_size(1, 64, 3, 4, 128, 128) == 0
