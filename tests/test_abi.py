"""The C-ABI library loads, exports every symbol include/gpt2.h declares, and
rejects bad host-side arguments before touching the device (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(gpt2_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    import transformer_decoder_lm_b200.binding as B
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(B.lib, n), n          # ctypes resolves the symbol in libgpt2.so
        assert n in B.SIGNATURES, n          # and the binding marshals it


def test_binding_names_match_header():
    import transformer_decoder_lm_b200 as pkg
    for n in header_functions():
        assert callable(getattr(pkg.binding, n)), n
        assert callable(getattr(pkg, n)), n         # re-exported by the package


def test_workspace_bytes_and_config_checks():
    import transformer_decoder_lm_b200.binding as B
    ok = B.make_config(12, 12, 768, 50257, 1024, B.GPT2_BF16)
    n = B.gpt2_workspace_bytes(ok, 4, 1024)
    M, C = 4096, 768
    assert n >= M * C * 4 + M * C * 2 * (1 + 3 + 1 + 4)
    assert n % 256 == 0
    assert B.gpt2_workspace_bytes(ok, 0, 1024) == 0
    bad = [
        B.make_config(12, 10, 768, 50257, 1024, B.GPT2_BF16),    # C % H != 0
        B.make_config(12, 6, 768, 50257, 1024, B.GPT2_BF16),     # d_head 128
        B.make_config(12, 12, 768, 50257, 1024, 7),              # dtype
        B.make_config(0, 12, 768, 50257, 1024, B.GPT2_BF16),     # no layers
        B.make_config(2, 2, 96, 512, 32, B.GPT2_BF16),           # bf16 needs C % 64 == 0
    ]
    for c in bad:
        assert B.gpt2_workspace_bytes(c, 1, 1) == 0
    # key/value cache: [n_layer][max_B][n_ctx][2C] elements of the dtype
    assert B.gpt2_kv_cache_bytes(ok, 4) == 12 * 4 * 1024 * 2 * 768 * 2
    f32 = B.make_config(2, 2, 64, 512, 32, B.GPT2_FP32)
    assert B.gpt2_kv_cache_bytes(f32, 3) == 2 * 3 * 32 * 2 * 64 * 4
    assert B.gpt2_kv_cache_bytes(ok, 0) == 0 and B.gpt2_kv_cache_bytes(bad[0], 1) == 0
    # flags: the tanh-GELU bit is accepted, any other bit rejected
    assert B.gpt2_workspace_bytes(B.make_config(12, 12, 768, 50257, 1024, B.GPT2_BF16, B.GPT2_FLAG_GELU_TANH), 4, 1024) == n
    assert B.gpt2_workspace_bytes(B.make_config(12, 12, 768, 50257, 1024, B.GPT2_BF16, 2), 4, 1024) == 0


def test_create_rejects_bad_arguments_on_the_host():
    import transformer_decoder_lm_b200.binding as B
    h = ctypes.c_void_p()
    cfg = B.make_config(12, 10, 768, 50257, 1024, B.GPT2_BF16)
    w = B.gpt2_weights_t()
    rc = B.lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(256), 1 << 30, 4, 1024, ctypes.byref(h))
    assert rc == B.ERR_CODE["GPT2_ERR_UNSUPPORTED"]
    cfg = B.make_config(2, 2, 64, 512, 32, B.GPT2_FP32)
    rc = B.lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(w), None, 1 << 30, 4, 32, ctypes.byref(h))
    assert rc == B.ERR_CODE["GPT2_ERR_INVALID_ARG"]
    rc = B.lib.gpt2_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(256), 16, 4, 32, ctypes.byref(h))
    assert rc == B.ERR_CODE["GPT2_ERR_WORKSPACE"]
    assert B.lib.gpt2_forward(None, None, 1, 1, None, None) == B.ERR_CODE["GPT2_ERR_INVALID_ARG"]
    assert B.lib.gpt2_status(None, None) == B.ERR_CODE["GPT2_ERR_INVALID_ARG"]
    assert B.gpt2_error_string(6) == "a bounded device wait timed out"
    assert B.gpt2_op_lmhead_ce_workspace_bytes(B.GPT2_BF16, 4096, 50257) >= 4096 * 786 * 8


def test_product_path_does_not_import_the_oracle():
    """The package and its sources never name the oracle package."""
    pkg = os.path.join(ROOT, "transformer_decoder_lm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\b(import\s+oracle|from\s+oracle)\b", text), f
