"""The C ABI library on the host: it loads, exports every declared symbol, and rejects
bad arguments before touching a GPU (CPU only; nothing here launches a kernel)."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

import rank_state_read_b200 as rs
from rank_state_read_b200 import build as rbuild


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rs.load()


def declared_functions(root):
    text = open(os.path.join(root, "include", "sketchssm.h")).read()
    return sorted(set(re.findall(r"\b(sketchssm_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_exports(root):
    assert declared_functions(root) == sorted(rs.EXPORTS)


def test_library_exports_every_declared_symbol(root, lib):
    out = subprocess.run(["nm", "-D", "--defined-only", rbuild.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (sketchssm_\w+)", out))
    for name in declared_functions(root):
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code, text in [(0, b"ok"), (1, b"invalid argument"), (2, b"misaligned tensor"),
                       (3, b"unsupported shape"), (4, b"CUDA error"), (5, b"timeout")]:
        assert lib.sketchssm_status_string(code) == text


def _create(lib, **over):
    d = dict(kind=0, batch=4, heads=8, qk_heads=1, key_dim=128, value_dim=80, window=16, groups=1,
             basis_rows=128, rank_cap=128)
    d.update({k: v for k, v in over.items() if k != "group_table"})
    desc = rs.Desc(*[d[f] for f, _ in rs.Desc._fields_])
    ranks = (ctypes.c_int32 * d["heads"])(*([6] * d["heads"]))
    out = ctypes.c_void_p()
    group = over.get("group_table")
    gp = None if group is None else ctypes.cast((ctypes.c_int32 * d["heads"])(*group), ctypes.c_void_p)
    st = lib.sketchssm_plan_create(ctypes.byref(desc), ctypes.cast(ranks, ctypes.c_void_p), gp, None,
                                   ctypes.byref(out))
    return st, out, lib.sketchssm_last_error().decode()


@pytest.mark.parametrize("over,status", [
    (dict(kind=7), 1), (dict(batch=0), 1), (dict(heads=6, groups=4), 1), (dict(heads=8, qk_heads=3), 1),
    (dict(basis_rows=129), 1), (dict(rank_cap=129), 1), (dict(key_dim=64, basis_rows=64, rank_cap=64), 3),
    (dict(value_dim=72), 3), (dict(value_dim=272), 3), (dict(window=33), 3),
    (dict(heads=64, groups=1, qk_heads=64), 3), (dict(heads=8, groups=2, qk_heads=1), 3),
])
def test_plan_create_rejects_bad_descriptors(lib, over, status):
    st, out, msg = _create(lib, **over)
    assert st == status, msg
    assert not out.value
    assert msg


def test_plan_create_rejects_bad_ranks(lib):
    desc = rs.Desc(0, 4, 4, 1, 128, 80, 16, 1, 79, 49)
    out = ctypes.c_void_p()
    for bad in ([6, 0, 6, 6], [6, 50, 6, 6], [6, -2, 6, 6]):
        ranks = (ctypes.c_int32 * 4)(*bad)
        st = lib.sketchssm_plan_create(ctypes.byref(desc), ctypes.cast(ranks, ctypes.c_void_p), None, None,
                                       ctypes.byref(out))
        assert st == 1 and not out.value
        assert b"rank[1]" in lib.sketchssm_last_error()
    assert lib.sketchssm_plan_create(ctypes.byref(desc), None, None, None, ctypes.byref(out)) == 1
    assert lib.sketchssm_plan_create(None, None, None, None, ctypes.byref(out)) == 1


@pytest.mark.parametrize("group,status", [
    ([0, 0, 1, 1, 2, 2, 3, 3][::-1], 3),   # groups in reverse order
    ([0, 1, 0, 1, 2, 3, 2, 3], 3),         # interleaved
    ([0, 0, 0, 1, 1, 2, 3, 3], 3),         # unequal runs
    ([0, 0, 1, 1, 2, 2, 3, 4], 1),         # a group outside 0..G-1
    ([0, 0, 1, 1, 2, 2, -1, 3], 1),
])
def test_plan_create_group_table_checked_on_the_host(lib, group, status):
    """Only the contiguous head-to-group map is supported; any other is refused before
    anything is allocated or launched, with the offending head named."""
    st, out, msg = _create(lib, heads=8, groups=4, qk_heads=4, group_table=group)
    assert st == status, msg
    assert not out.value
    assert "group[" in msg


def test_calls_without_a_plan(lib):
    assert lib.sketchssm_flush(None, None, None, None, None, None, None, 0, None, None) == 1
    assert lib.sketchssm_decode(None, 0, *([None] * 13), None) == 1
    assert lib.sketchssm_dense_decode(None, 0, *([None] * 11), None) == 1
    assert lib.sketchssm_plan_query(None, None, None, None, 1, None, None) == 1
    assert lib.sketchssm_plan_set_wait_limit(None, 1000) == 1
    assert lib.sketchssm_decode_rows(None, *([None] * 14), None) == 1
    assert lib.sketchssm_flush_rows(None, *([None] * 8), None) == 1
    assert lib.sketchssm_prefill(None, 0, *([None] * 7), None) == 1
    assert lib.sketchssm_plan_check(None, None) == 1
    assert lib.sketchssm_plan_destroy(None) == 0


def test_python_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    import rank_state_read_b200._binding as b
    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        b.load()
