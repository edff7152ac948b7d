"""The C-ABI library loads and exports every entry point include/dreamer.h declares (no GPU
calls)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "depth_recurrent_attention_b200")


@pytest.fixture(scope="module")
def built():
    from depth_recurrent_attention_b200 import build
    return build.build()


def declared(header):
    txt = open(os.path.join(ROOT, "include", header)).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dreamer_\w+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    names = declared("dreamer.h")
    for n in ("dreamer_init", "dreamer_core_forward", "dreamer_decode_step",
              "dreamer_route_counts", "dreamer_route_experts", "dreamer_bias_update",
              "dreamer_destroy", "dreamer_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(built):
    lib = ctypes.CDLL(os.path.join(PKG, "libdreamer.so"))
    for header in os.listdir(os.path.join(ROOT, "include")):
        for n in declared(header):
            assert hasattr(lib, n), f"{n} declared in {header} but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(PKG, "libdreamer.so")],
                         capture_output=True, text=True).stdout
    for n in declared("dreamer.h"):
        assert re.search(rf"\bT {n}\b", out), n


def test_strerror_without_gpu(built):
    lib = ctypes.CDLL(os.path.join(PKG, "libdreamer.so"))
    lib.dreamer_strerror.restype = ctypes.c_char_p
    assert lib.dreamer_strerror(0) == b"ok"
    assert lib.dreamer_strerror(-1) == b"invalid argument"
    assert lib.dreamer_strerror(-5) == b"device wait timed out"


def test_argument_errors_without_gpu(built):
    """Entry points reject a NULL handle before touching the device (through the binding's
    argument types)."""
    from depth_recurrent_attention_b200.dreamer import ERR_ARG, lib
    L = lib()
    assert L.dreamer_bias_update_counts(None, ctypes.c_float(0.01), None, 1, None, None) == ERR_ARG
    assert L.dreamer_bias_update(None, ctypes.c_float(0.01), None, None) == ERR_ARG
    assert L.dreamer_route_balance(None, -1, None, None, None) == ERR_ARG


def test_product_does_not_reference_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower() or f == "inputs.py", f
    lib_txt = open(os.path.join(PKG, "dreamer.py")).read()
    assert "import oracle" not in lib_txt


@pytest.mark.parametrize("kw,bf16_code", [
    ({}, "ARG"),                                        # valid shapes: fails only at the weights
    (dict(n_heads=16, head_dim=32), "UNSUPPORTED"),     # no tcgen05 GEMM / flash SA for d = 32
    (dict(expert_hidden=48), "UNSUPPORTED"),            # expert FFN kernels: m 16, 32 or 64
    (dict(router_dim=32), "UNSUPPORTED"),               # router: d_r 64 or 128
    (dict(hidden=384, n_heads=6), "UNSUPPORTED"),       # N tiles of 256 columns
    (dict(n_experts=6, top_k=2), "UNSUPPORTED"),        # router scorer: E a multiple of 4
    (dict(n_heads=64, head_dim=64, hidden=4096), "UNSUPPORTED"),  # DA: a warp per head, <= 32
])
def test_bf16_shapes_without_a_tcgen05_kernel_are_refused(built, kw, bf16_code):
    """bfloat16 mode has no CUDA-core fallback: dreamer_init refuses a shape its kernels do not
    take (before any device call), while float32 mode takes it (and fails only at the NULL
    weights here)."""
    import depth_recurrent_attention_b200.dreamer as D
    from depth_recurrent_attention_b200 import configs
    cfg = configs.SMALL.with_(**kw)
    h = ctypes.c_void_p()
    rc = D.lib().dreamer_init(ctypes.byref(D.config_c(cfg)), None, None, ctypes.byref(h))
    assert rc == getattr(D, "ERR_" + bf16_code), (kw, rc)
    rc32 = D.lib().dreamer_init(ctypes.byref(D.config_c(cfg.with_(dtype="fp32"))), None, None,
                                ctypes.byref(h))
    assert rc32 == D.ERR_ARG, (kw, rc32)


def test_only_the_test_hook_library_exports_the_injection(built):
    """dreamer_test_inject (the timeout test's hook) exists in the test-hook build only."""
    from depth_recurrent_attention_b200 import dreamer as D
    assert not hasattr(ctypes.CDLL(D.LIB_PATH), "dreamer_test_inject")
    assert hasattr(ctypes.CDLL(D.TESTHOOKS_PATH), "dreamer_test_inject")
