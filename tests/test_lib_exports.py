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
    n = ctypes.c_int64(-1)
    assert L.zo_launch_count(None, ctypes.byref(n)) == zo.ZO_ERR_INVALID
    assert n.value == -1
    assert L.zo_kernel_times(None, None, None) == zo.ZO_ERR_INVALID
    assert L.zo_enable_kernel_timing(None, 1) == zo.ZO_ERR_INVALID
    assert L.zo_set_loss_location(None, 0) == zo.ZO_ERR_INVALID
    assert L.zo_pack_probe(None, 0, 0, 0, 1, None) == zo.ZO_ERR_INVALID
    assert L.zo_model_step_host(None, None, None, 1, 1, 1, 1, 1e-3, 0.1, 0.0, 1, None) == zo.ZO_ERR_INVALID


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


def test_header_is_plain_c_and_links_from_c(zo, tmp_path):
    """include/zo.h compiles as pedantic C99; a C program linked against libzo.so calls the
    host-only entry points (no device needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "zo.h"
int main(void) {
  zo_model_cfg c;
  int64_t M = 0;
  memset(&c, 0, sizeof c);
  c.n_layers = 12; c.d_model = 768; c.n_heads = 12; c.d_ffn = 3072; c.vocab = 50272;
  c.max_pos = 2048; c.class_ids[0] = 1000; c.class_ids[1] = 2000; c.family = ZO_FAMILY_OPT;
  if (zo_model_param_count(&c, &M) != ZO_OK) return 1;
  printf("%lld %s %s\n", (long long)M, zo_status_name(ZO_OK), zo_status_name(ZO_ERR_TIMEOUT));
  return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(zo.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lzo", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert out == ["125239296", "ZO_OK", "ZO_ERR_TIMEOUT"]
