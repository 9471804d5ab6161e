"""The C-ABI library loads and exports every entry point the headers declare;
host-side argument checks (no GPU needed)."""
import ctypes
import os
import re

import pytest

from dynamic_layer_wise_b200 import build, dcu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def libs():
    out = build.build_all()
    return out


def _declared(header):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|void|const char\s*\*)\s*(\w+)\s*\(", src, flags=re.M)))


def test_headers_declare_entry_points():
    names = _declared("dcu.h")
    for n in ("dcu_create", "dcu_full_forward", "dcu_step", "commit_select", "dcu_destroy", "dcu_last_error",
              "dcu_select_tokens", "dcu_budget_split", "dcu_commit_rule", "dcu_cosine_distance"):
        assert n in names


@pytest.mark.parametrize("header,lib", [("dcu.h", "dcu"), ("dcu_gen.h", "gen")])
def test_library_exports_every_declared_symbol(libs, header, lib):
    so = ctypes.CDLL(libs[lib])
    missing = [n for n in _declared(header) if not hasattr(so, n)]
    assert not missing, missing


def test_binding_signatures_cover_header(libs):
    assert set(_declared("dcu.h")) <= set(dcu._SIGS)


def _cfg(**kw):
    base = dict(n_layers=2, d_model=64, n_heads=2, n_kv_heads=2, head_dim=32, d_ffn=128, vocab=100, mask_id=99,
                max_batch=1, max_seq=16, dtype=dcu.DCU_F32, rms_eps=1e-5, rope_theta=10000.0, window_mode=0)
    base.update(kw)
    return dcu.dcu_cfg(**base)


@pytest.mark.parametrize("bad", [dict(d_model=60), dict(head_dim=24), dict(n_kv_heads=3), dict(max_seq=20000),
                                 dict(mask_id=100), dict(dtype=7), dict(window_mode=5), dict(n_layers=0),
                                 dict(rms_eps=0.0)])
def test_create_rejects_bad_cfg_on_host(libs, bad):
    L = dcu.lib()
    w = dcu.dcu_weights()
    h = ctypes.c_void_p(0)
    rc = L.dcu_create(ctypes.byref(w), ctypes.byref(_cfg(**bad)), ctypes.byref(h))
    assert rc == dcu.DCU_EINVAL
    assert b"bad cfg" in L.dcu_last_error(None)
    assert not h.value


def test_create_rejects_null_weights_on_host(libs):
    L = dcu.lib()
    w = dcu.dcu_weights()
    h = ctypes.c_void_p(0)
    assert L.dcu_create(ctypes.byref(w), ctypes.byref(_cfg()), ctypes.byref(h)) == dcu.DCU_EINVAL
    assert L.dcu_create(None, ctypes.byref(_cfg()), ctypes.byref(h)) == dcu.DCU_EINVAL


def test_stateless_entry_points_reject_bad_args_on_host(libs):
    L = dcu.lib()
    assert L.dcu_budget_split(None, 1, 4, 8, 0, None, None) == dcu.DCU_EINVAL
    assert L.dcu_select_tokens(None, None, None, None, 1, 8, 4, 0, None, None, None, None, None) == dcu.DCU_EINVAL
    assert L.dcu_commit_rule(9, 0.1, None, None, None, None, 1, 8, None, None, None) == dcu.DCU_EINVAL
    assert L.dcu_cosine_distance(None, None, None, 4, 12, 0, None, None) == dcu.DCU_EINVAL
    assert L.dcu_full_forward(None, None, 1, 8, None) == dcu.DCU_EINVAL
    assert L.dcu_step(None, None, None, None, 1, 1, None) == dcu.DCU_EINVAL
    assert L.commit_select(None, 0, 0.1, None, None, None, None, None) == dcu.DCU_EINVAL
    assert L.dcu_set_option(None, dcu.DCU_OPT_ATTENTION, dcu.DCU_ATTN_TCGEN05) == dcu.DCU_EINVAL
    assert dcu.dcu_kernel_class_name(dcu.DCU_K_GEMM) == "gemm"
