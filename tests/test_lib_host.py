"""Host-side checks of the C-ABI library that need no GPU: it loads, it exports every
entry point include/sparse_attn.h declares, and host-side argument errors are
returned as codes without touching the device."""
import ctypes
import os
import re

import pytest

from index_sparse_attention_b200 import _lib
from index_sparse_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "sizeof")))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(_lib.EXPORTS) <= set(names), names
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"


def test_header_constants_match_the_binding():
    """Every integer SA_* constant the header defines has the same value in the binding."""
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "sparse_attn.h")).read()
    defs = {}
    for name, expr in re.findall(r"^#define (SA_[A-Z0-9_]+) ([^/\n]+)", hdr, re.M):
        expr = expr.strip()
        if re.fullmatch(r"[-+*()0-9u\s]+", expr):  # integer expressions only
            defs[name] = eval(expr.replace("u", ""))
    assert len(defs) >= 20
    for name, value in defs.items():
        assert hasattr(_lib, name), f"{name} missing from the binding"
        assert getattr(_lib, name) == value, (name, getattr(_lib, name), value)


def test_error_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -7, 12345):
        assert isinstance(_lib.error_string(code), str)
    assert "aligned" in _lib.error_string(_lib.SA_ERR_ALIGN)


def test_null_arguments_are_rejected_on_host(lib):
    p = _lib.ParamsStruct()
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_INVALID
    assert lib.sparse_attn_bwd(ctypes.byref(p), None, 0, None) == _lib.SA_ERR_INVALID
    s = _lib.BlockSparseStruct()
    assert lib.block_mask_to_block_sparse(ctypes.byref(s), None) == _lib.SA_ERR_INVALID
    assert lib.index_to_block_sparse(None, 4, ctypes.byref(s), None, None) == _lib.SA_ERR_INVALID


def _fake_params(**kw):
    """Parameters with non-null (never dereferenced) pointers for host-side checks."""
    s = _lib.BlockSparseStruct(_lib.SA_MODE_DENSE, 0, 1, 2, 256, 256, 128, 0, 0, None, None,
                               0x1000, 0x1000, 0x1000, 0x1000)
    p = _lib.ParamsStruct(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000,
                          0x1000, 1, 4, 2, 128, 128, 256, 256, 0.125, ctypes.pointer(s), None)
    for k, v in kw.items():
        setattr(p, k, v)
    return p, s


def test_unsupported_and_inconsistent_shapes(lib):
    p, s = _fake_params(Dqk=96, Dv=96)
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_UNSUPPORTED
    p, s = _fake_params(HQ=5)
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_INVALID
    p, s = _fake_params(Sq=384)  # lists were built for Sq = 256
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_INVALID
    p, s = _fake_params(q=0x1008)  # not 16-byte aligned
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_ALIGN
    p, s = _fake_params(softmax_scale=0.0)
    assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_INVALID


def test_zero_extents_are_refused_on_host(lib):
    """A problem with a zero extent is refused before any launch, by every entry point."""
    for field in ("B", "HQ", "HK", "Sq", "Sk"):
        p, s = _fake_params(**{field: 0})
        assert lib.sparse_attn_fwd(ctypes.byref(p), None) == _lib.SA_ERR_INVALID, field
        assert lib.sparse_attn_bwd(ctypes.byref(p), 0x2000, 1 << 30, None) == _lib.SA_ERR_INVALID, field
        if field in ("B", "HQ", "Sq"):  # the workspace holds per-query-row data only
            assert lib.sparse_attn_bwd_workspace_size(ctypes.byref(p)) == 0, field
    for field in ("B", "HK", "Sq", "Sk"):
        p, s = _fake_params()
        setattr(s, field, 0)
        assert lib.block_mask_to_block_sparse(ctypes.byref(s), None) == _lib.SA_ERR_INVALID, field


def test_bwd_workspace_is_checked_on_host(lib):
    p, s = _fake_params()
    need = lib.sparse_attn_bwd_workspace_size(ctypes.byref(p))
    # Delta [1,4,256] fp32, the dQ accumulator [1,256,4,128] fp32 and the deterministic
    # mode's turn counters [1,4,2,2] int32, each 256-B rounded
    assert need == 4 * 256 * 4 + 256 * 4 * 128 * 4 + 256
    for fn in (lib.sparse_attn_bwd, lib.sparse_attn_bwd_deterministic):
        assert fn(ctypes.byref(p), None, 0, None) == _lib.SA_ERR_WORKSPACE
        assert fn(ctypes.byref(p), 0x2000, need - 1, None) == _lib.SA_ERR_WORKSPACE


def test_block_mask_validation(lib):
    s = _lib.BlockSparseStruct(_lib.SA_MODE_BLOCK, 0, 1, 2, 256, 256, 32, 8, 8, 0x1000, None,
                               0x1000, 0x1000, 0x1000, 0x1000)
    assert lib.block_mask_to_block_sparse(ctypes.byref(s), None) == _lib.SA_ERR_UNSUPPORTED
    s.bs, s.Mb, s.Nb = 64, 2, 4  # Mb * bs < Sq
    assert lib.block_mask_to_block_sparse(ctypes.byref(s), None) == _lib.SA_ERR_INVALID


def test_instrumentation_setters(lib):
    """The test-only knob: the wait limit of the bounded pipeline waits."""
    assert lib.sparse_attn_set_wait_limit_ns(1000) == _lib.SA_OK
    assert lib.sparse_attn_set_wait_limit_ns(0) == _lib.SA_OK


def test_backward_form_setter(lib):
    """The (192,128) backward's key-tile form: the three SA_BWD_FORM_* values are accepted,
    anything else is refused with SA_ERR_INVALID; the binding maps the names and refuses
    unknown ones."""
    import index_sparse_attention_b200 as sa
    for code in (_lib.SA_BWD_FORM_SPLIT, _lib.SA_BWD_FORM_WHOLE, _lib.SA_BWD_FORM_AUTO):
        assert lib.sparse_attn_set_backward_form(code) == _lib.SA_OK
    for bad in (-1, 3, 1 << 20):
        assert lib.sparse_attn_set_backward_form(bad) == _lib.SA_ERR_INVALID
    for name in ("split", "whole", "auto"):
        sa.sparse_attn_set_backward_form(name)
    with pytest.raises(ValueError):
        sa.sparse_attn_set_backward_form("halves")


def test_forward_form_setter(lib):
    """The forward's head-to-CTA form: the four SA_FWD_FORM_* values are accepted,
    anything else is refused with SA_ERR_INVALID; the binding maps the names and refuses
    unknown ones."""
    import index_sparse_attention_b200 as sa
    for code in (_lib.SA_FWD_FORM_ONE_HEAD, _lib.SA_FWD_FORM_CTA_PAIR, _lib.SA_FWD_FORM_TWO_HEADS,
                 _lib.SA_FWD_FORM_TWO_TILES, _lib.SA_FWD_FORM_AUTO):
        assert lib.sparse_attn_set_forward_form(code) == _lib.SA_OK
    for bad in (-1, 5, 1 << 20):
        assert lib.sparse_attn_set_forward_form(bad) == _lib.SA_ERR_INVALID
    for name in ("one_head", "cta_pair", "two_heads", "two_tiles", "auto"):
        sa.sparse_attn_set_forward_form(name)
    with pytest.raises(ValueError):
        sa.sparse_attn_set_forward_form("sometimes")
