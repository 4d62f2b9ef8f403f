"""The C-ABI library without a GPU: it builds, loads, exports every entry
point include/tria.h declares, and rejects bad arguments on the host before
any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import key_retention_scoring_b200 as T
from key_retention_scoring_b200 import build as tria_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    tria_build.build()


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "tria.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(tria_[a-z_]+)\s*\(", txt)))


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 12, names
    lib = ctypes.CDLL(T.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(T.EXPORTS) == names


def test_status_strings_and_version():
    assert T.tria_version().startswith("tria")
    for code, name in T.STATUS_NAMES.items():
        assert T.tria_status_string(code).startswith(name)


def _stats_arrays(L=1, H=4, F=64):
    a = np.ones((L, H, F), np.float32)
    return a, a, 2 * a


def _load(desc, arrs, mask=None):
    out = ctypes.c_void_p()
    m = None if mask is None else np.ascontiguousarray(mask, np.float32)
    return T.lib().tria_load_stats(ctypes.byref(desc), arrs[0].ctypes.data, arrs[1].ctypes.data,
                                   arrs[2].ctypes.data, None if m is None else m.ctypes.data,
                                   None, ctypes.byref(out))


def test_load_stats_host_validation():
    arrs = _stats_arrays()
    lib = T.lib()
    out = ctypes.c_void_p()
    d = T.model_desc(1, 4, 2, T.PAIR_NEOX, 1e4)
    assert lib.tria_load_stats(None, None, None, None, None, None, ctypes.byref(out)) == 1
    assert lib.tria_load_stats(ctypes.byref(d), None, None, None, None, None, ctypes.byref(out)) == 1
    assert _load(T.model_desc(1, 4, 2, T.PAIR_NEOX, 1e4, head_dim=64), arrs) == 2
    assert _load(T.model_desc(1, 6, 2, T.PAIR_NEOX, 1e4), arrs) == 2       # G = 3
    assert _load(T.model_desc(1, 4, 3, T.PAIR_NEOX, 1e4), arrs) == 1       # Hq % Hkv
    assert _load(T.model_desc(1, 4, 2, 7, 1e4), arrs) == 1                 # pairing
    assert _load(T.model_desc(1, 4, 2, T.PAIR_NEOX, 1.0), arrs) == 1       # theta
    assert _load(T.model_desc(1, 4, 2, T.PAIR_NEOX, 1e4, offset_log2_max=31), arrs) == 1
    assert _load(T.model_desc(0, 4, 2, T.PAIR_NEOX, 1e4), arrs) == 1
    bad = [a.copy() for a in arrs]
    bad[0][0, 0, 3] = np.nan
    assert _load(d, bad) == 1
    assert _load(d, arrs, mask=np.full(64, np.inf)) == 1


def test_pass_entry_points_reject_null_arguments():
    lib = T.lib()
    size = ctypes.c_size_t()
    assert lib.tria_workspace_size(None, None, None, 0, 1, ctypes.byref(size)) == 1
    assert lib.tria_score(None, None, None, 0, 1, None, None, None, 0, None) == 1
    assert lib.tria_select(None, None, None, None, 0, 1, None, None, 0, None) == 1
    assert lib.tria_compact(None, None, None, None, 0, 1, None, None, None) == 1
    assert lib.tria_compress_pass(None, None, None, None, None, None, None, 0, None) == 1
    flags = ctypes.c_int32()
    assert lib.tria_read_device_status(None, None, ctypes.byref(flags)) == 1
    assert lib.tria_stats_desc(None, None) == 1
    assert lib.tria_free_stats(None) == 0
    assert lib.tria_set_pass_events(None) == 0


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(T, "_lib", None)
    monkeypatch.setattr(T, "LIB_PATH", "/nonexistent/libtria.so")
    with pytest.raises(RuntimeError):
        T.lib()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "key_retention_scoring_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in src.replace("oracle/", ""), f


def test_newer_entry_points_reject_missing_objects_on_the_host():
    # budget variants and decode attention validate before any CUDA call
    lib = T.lib()
    b = (ctypes.c_int * 4)()
    row = ctypes.c_int()
    assert lib.tria_layer_budgets(None, None, None, b, ctypes.byref(row)) == 1
    size = ctypes.c_size_t()
    assert lib.tria_decode_workspace_size(None, None, ctypes.byref(size)) == 1
    assert lib.tria_decode_attention(None, None, 0, None, 1.0, None, None, None, None, 0, None) == 1
    prm = T.params(2048, 256, 0, budget_pct=50.0, layer_budget_scales=[1.0, 0.5], interval=128)
    assert abs(prm.budget_pct - 50.0) < 1e-6 and prm.interval == 128
    assert abs(prm.layer_budget_scales[1] - 0.5) < 1e-7
