"""libzo.so loads on a CPU-only host and exports every function include/zo.h declares;
argument checks that need no device behave as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(zo_[a-z0-9_]+)\s*\(", src))
    return names


def test_header_declares_the_boundary():
    names = _declared()
    for required in ["zo_create", "zo_perturb", "zo_restore", "zo_step", "zo_destroy",
                     "zo_quad_loss", "zo_mlp_loss", "zo_update"]:
        assert required in names


def test_library_exports_every_declared_symbol(zo):
    lib = ctypes.CDLL(zo.LIB_PATH)
    missing = [n for n in sorted(_declared()) if not hasattr(lib, n)]
    assert not missing, missing


def test_status_names(zo):
    assert zo.zo_status_name(0) == "ZO_OK"
    assert zo.zo_status_name(5) == "ZO_ERR_NONFINITE"
    assert zo.zo_status_name(99) == "ZO_ERR_UNKNOWN"


def test_create_rejects_bad_arguments_before_touching_a_device(zo):
    h = ctypes.c_void_p()
    L = zo.lib
    assert L.zo_create(None, 16, 10, 0, 0, None) == zo.ZO_ERR_INVALID
    assert L.zo_create(ctypes.byref(h), None, 10, 0, 0, None) == zo.ZO_ERR_INVALID
    assert L.zo_create(ctypes.byref(h), 16, 0, 0, 0, None) == zo.ZO_ERR_INVALID
    assert L.zo_create(ctypes.byref(h), 16, 10, 7, 0, None) == zo.ZO_ERR_INVALID
    assert L.zo_create(ctypes.byref(h), 17, 10, 0, 0, None) == zo.ZO_ERR_INVALID  # misaligned
    assert L.zo_create(ctypes.byref(h), 16, 1 << 40, 0, 0, None) == zo.ZO_ERR_INVALID
    assert not h.value
    assert L.zo_destroy(None) == zo.ZO_OK
    assert L.zo_perturb(None, 1, 1e-3, 0) == zo.ZO_ERR_INVALID
    assert L.zo_step(None, None, None, 1, None, 0.1, 1e-3, 0.0) == zo.ZO_ERR_INVALID


def test_product_path_has_no_oracle_dependency():
    """The CUDA library's package and sources never reference the oracle."""
    pkg = os.path.join(ROOT, "zero_order_forward_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "oracle" not in txt.lower(), os.path.join(dirpath, fn)


def test_model_param_count_matches_both_layouts(zo):
    """zo_model_param_count is host-only: the flat layouts of both decoder families agree in
    size with the oracle's, and invalid configurations are rejected."""
    import oracle
    import synth
    for cfg in synth.OPT_CONFIGS.values():
        assert zo.zo_model_param_count(cfg) == oracle.opt.param_count(cfg)
    for cfg in synth.QWEN_CONFIGS.values():
        assert zo.zo_model_param_count(cfg) == oracle.qwen.param_count(cfg)
    q = dict(synth.QWEN_CONFIGS["qwen3-1.7b"])
    for bad in (dict(n_kv_heads=3), dict(head_dim=96), dict(rope_theta=0.0), dict(d_model=2000),
                dict(d_ffn=6145), dict(class_ids=(0, q["vocab"]))):
        with pytest.raises(zo.ZoError):
            zo.zo_model_param_count({**q, **bad})
