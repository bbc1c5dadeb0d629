"""The C-ABI library loads on a machine without a GPU, exports every function
include/blockffn.h declares, and rejects bad arguments on the host before any
CUDA call (no compute runs here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "blockffn.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(blockffn_[a-z_0-9]+)\s*\(", text)))


def test_header_is_plain_c(tmp_path):
    """The public header compiles on its own as C11 (and C++17), warnings as errors."""
    import shutil
    import subprocess
    for cc, std, ext in (("gcc", "c11", "c"), ("g++", "c++17", "cpp")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not installed")
        src = tmp_path / f"use.{ext}"
        src.write_text('#include "blockffn.h"\nint main(void) { return (int)blockffn_version(); }\n')
        subprocess.run([cc, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                        "-I" + os.path.join(ROOT, "include"), str(src)], check=True)


@pytest.fixture(scope="module")
def lib():
    from chunk_sparse_moe_b200 import build
    build.build()
    from chunk_sparse_moe_b200 import _lib
    return _lib


def test_header_declares_the_calls():
    names = declared_functions()
    for must in ("blockffn_route", "blockffn_chunk_union", "blockffn_forward",
                 "blockffn_forward_workspace_bytes", "blockffn_get_device_status"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in blockffn.h but not exported"
        assert name in lib.SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings(lib):
    for code in range(6):
        assert lib.lib.blockffn_status_string(code)
    assert lib.lib.blockffn_version() >= 100


@pytest.mark.parametrize("T,d_h,E,d_e,n,dt", [
    (32, 2048, 64, 128, 0, 1),      # n < 1
    (32, 2048, 64, 128, 33, 1),     # n > 32
    (32, 2048, 0, 128, 32, 1),      # E < 1
    (32, 2048, 257, 128, 32, 1),    # E > 256
    (-1, 2048, 64, 128, 32, 1),     # T < 0
    (32, 2000, 64, 128, 32, 1),     # bf16 d_h % 128
    (32, 2048, 64, 64, 32, 1),      # bf16 d_e % 128
    (32, 2048, 64, 1024, 32, 1),    # bf16 d_e > 512
    (32, 2048, 64, 128, 32, 7),     # unknown dtype
])
def test_forward_rejects_bad_shapes_on_host(lib, T, d_h, E, d_e, n, dt):
    L = lib.lib
    assert L.blockffn_forward_workspace_bytes(T, d_h, E, d_e, n, dt, 0) == 0
    st = L.blockffn_forward(16, 16, None, None, None, 0.0, None, None, None, 16, 16, T, d_h, E, d_e,
                            n, dt, None, 16, 16, 1 << 30, None)
    assert st in (lib.ERR_INVALID_ARG, lib.ERR_UNSUPPORTED)
    assert L.blockffn_last_error_message()


def test_forward_gating_source_is_exclusive(lib):
    L = lib.lib
    # (T = 32 > 0: with T = 0 the call is a no-op before this check)
    # gates and router weights together
    st = L.blockffn_forward(16, 16, 16, None, None, 0.0, None, None, None, 16, 16, 32, 2048, 64, 128,
                            32, 1, None, 16, 16, 1 << 30, None)
    assert st == lib.ERR_INVALID_ARG
    # neither
    st = L.blockffn_forward(16, None, None, None, None, 0.0, None, None, None, 16, 16, 32, 2048, 64,
                            128, 32, 1, None, 16, 16, 1 << 30, None)
    assert st == lib.ERR_INVALID_ARG


def test_forward_union_tables_all_or_none(lib):
    """counts, idx and tmask come together or not at all, only with injected gates,
    and 16-byte aligned; each refusal is made on the host."""
    L = lib.lib
    args = (16, 16, 32, 2048, 64, 128, 32, 1, None, 16, 16, 1 << 30, None)
    # two of the three
    assert L.blockffn_forward(16, 16, None, None, None, 0.0, 16, 16, None, *args) == lib.ERR_INVALID_ARG
    assert L.blockffn_forward(16, 16, None, None, None, 0.0, None, None, 16, *args) == lib.ERR_INVALID_ARG
    # with the router
    assert L.blockffn_forward(16, None, 16, None, 16, 0.0, 16, 16, 16, *args) == lib.ERR_INVALID_ARG
    assert b"injected" in L.blockffn_last_error_message()
    # misaligned table
    assert L.blockffn_forward(16, 16, None, None, None, 0.0, 16, 20, 16, *args) == lib.ERR_INVALID_ARG


def test_forward_layer_options_checked_on_host(lib):
    """Expert biases and the LayerNorm (blockffn_layer_opts): misaligned pointers and
    a bad ln_eps are refused on the host; unknown workspace flags size nothing."""
    import ctypes
    L = lib.lib
    args = (16, 16, 32, 2048, 64, 128, 32, 1)
    tail = (16, 16, 1 << 30, None)

    def call(opts):
        return L.blockffn_forward(16, 16, None, None, None, 0.0, None, None, None, *args,
                                  ctypes.byref(opts), *tail)

    assert call(lib.LayerOpts(20, None, None, None, 0.0)) == lib.ERR_INVALID_ARG        # b_in
    assert call(lib.LayerOpts(None, 24, None, None, 0.0)) == lib.ERR_INVALID_ARG        # b_out
    assert call(lib.LayerOpts(None, None, 20, None, 1e-5)) == lib.ERR_INVALID_ARG       # ln_weight
    assert call(lib.LayerOpts(None, None, 16, 20, 1e-5)) == lib.ERR_INVALID_ARG         # ln_bias
    assert call(lib.LayerOpts(None, None, 16, None, -1.0)) == lib.ERR_INVALID_ARG       # ln_eps < 0
    assert call(lib.LayerOpts(None, None, 16, None, float("inf"))) == lib.ERR_INVALID_ARG
    assert b"ln_eps" in L.blockffn_last_error_message()
    assert L.blockffn_forward_workspace_bytes(32, 2048, 64, 128, 32, 1, 4) == 0          # unknown flag


def test_union_and_route_reject_bad_args(lib):
    L = lib.lib
    assert L.blockffn_chunk_union(16, 32, 64, 0, 16, 16, 16, None) == lib.ERR_INVALID_ARG
    assert L.blockffn_chunk_union(16, 32, 300, 8, 16, 16, 16, None) == lib.ERR_INVALID_ARG
    assert L.blockffn_chunk_union(None, 32, 64, 8, 16, 16, 16, None) == lib.ERR_INVALID_ARG
    assert L.blockffn_route(16, 16, None, 16, -1.0, 32, 64, 16, 1, 16, None) == lib.ERR_INVALID_ARG
    assert L.blockffn_route(16, 16, None, 16, 0.0, 32, 60, 16, 1, 16, None) == lib.ERR_UNSUPPORTED
    # misaligned pointers
    assert L.blockffn_route(17, 16, None, 16, 0.0, 32, 64, 16, 1, 16, None) == lib.ERR_INVALID_ARG


def test_residual_layernorm_rejects_bad_args(lib):
    L = lib.lib
    f = L.blockffn_residual_layernorm
    assert f(16, 16, 16, 16, 1e-5, 4, 64, 7, 16, None) == lib.ERR_INVALID_ARG          # unknown dtype
    assert f(16, 16, 16, 16, 1e-5, -1, 64, lib.BF16, 16, None) == lib.ERR_INVALID_ARG  # T < 0
    assert f(16, 16, 16, 16, 1e-5, 4, 0, lib.BF16, 16, None) == lib.ERR_INVALID_ARG    # d_h < 1
    assert f(16, 16, 16, 16, -1.0, 4, 64, lib.BF16, 16, None) == lib.ERR_INVALID_ARG   # eps < 0
    assert f(16, 16, 16, 16, float("nan"), 4, 64, lib.F32, 16, None) == lib.ERR_INVALID_ARG
    assert f(None, 16, 16, 16, 1e-5, 4, 64, lib.BF16, 16, None) == lib.ERR_INVALID_ARG  # null y
    assert f(16, 16, None, 16, 1e-5, 4, 64, lib.BF16, 16, None) == lib.ERR_INVALID_ARG  # null scale
    # no rows: nothing to do, nothing launched, no pointer needed
    assert f(None, None, None, None, 1e-5, 0, 64, lib.BF16, None, None) == lib.OK


def test_empty_inputs_are_no_ops(lib):
    L = lib.lib
    # T = 0: nothing to do, nothing launched, no pointer needed
    assert L.blockffn_chunk_union(None, 0, 64, 32, None, None, None, None) == lib.OK
    assert L.blockffn_route(None, None, None, None, 0.0, 0, 64, 16, 1, None, None) == lib.OK
    assert L.blockffn_forward(None, 16, None, None, None, 0.0, None, None, None, None, None, 0, 2048,
                              64, 128, 32, 1, None, None, None, 0, None) == lib.OK
