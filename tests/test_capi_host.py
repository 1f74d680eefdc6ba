"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
symbol include/moe.h declares, and rejects bad arguments synchronously before any
CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

import sparse_moe_layer_02_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_library_builds_and_loads():
    from sparse_moe_layer_02_b200 import build
    build.build()
    lib = moe.load_library()
    assert lib.moe_version() >= 100


def test_every_declared_symbol_is_exported():
    declared = _declared_functions()
    assert set(declared) == set(moe.EXPORTED_SYMBOLS)
    out = subprocess.run(["nm", "-D", "--defined-only", moe.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(moe_[a-z_]+)$", out, flags=re.M))
    missing = set(declared) - exported
    assert not missing, missing
    lib = moe.load_library()
    for name in declared:
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_status_strings():
    for code in range(-8, 1):
        s = moe.moe_status_string(code)
        assert s and s != "unknown status"
    assert moe.moe_status_string(-99) == "unknown status"


@pytest.mark.parametrize("E,G,tg,k", [(16, 3, 1, 2), (16, 16, 2, 2), (16, 4, 1, 8), (8, 1, 1, 9),
                                      (600, 1, 1, 8), (16, 4, 0, 2), (16, 4, 5, 2), (64, 1, 1, 33)])
def test_router_rejects_bad_shapes(E, G, tg, k):
    lib = moe.load_library()
    rc = lib.moe_router(None, 1, None, 1, None, 10, 64, E, G, tg, k, 1, 1.0, None, None, None)
    assert rc == -2


def test_router_rejects_bad_dtype_and_null_pointers():
    lib = moe.load_library()
    assert lib.moe_router(None, 7, None, 1, None, 10, 64, 16, 1, 1, 2, 1, 1.0, None, None, None) == -3
    assert lib.moe_router(None, 1, None, 1, None, 10, 64, 16, 1, 1, 2, 1, 1.0, None, None, None) == -1
    # N = 0 is a no-op even without buffers
    assert lib.moe_router(None, 1, None, 1, None, 0, 64, 16, 1, 1, 2, 1, 1.0, None, None, None) == 0


def test_forward_rejects_bad_arguments():
    lib = moe.load_library()
    call = lambda **kw: lib.moe_forward(*([None] * 8), kw.get("N", 10), kw.get("D", 64),
                                        kw.get("E", 16), kw.get("d", 32), kw.get("dsh", 32),
                                        kw.get("k", 2), kw.get("dt", 1), None, None,
                                        kw.get("ws", 0), None)
    assert call(dt=5) == -3
    assert call(D=60) == -2          # bf16 rows must be 16-byte multiples
    assert call(d=20) == -2
    assert call(k=0) == -2
    assert call(E=1000) == -2
    assert call() == -1              # null pointers
    assert call(N=0) == 0            # no-op


def test_workspace_sizes():
    lib = moe.load_library()
    w = lambda *a: lib.moe_forward_workspace(*a)
    assert w(0, 64, 16, 32, 32, 2, 1) > 0
    assert w(10, 64, 16, 32, 32, 2, 9) == 0
    assert w(100, 64, 16, 32, 32, 2, 1) < w(1000, 64, 16, 32, 32, 2, 1)
    big = w(16384, 6144, 256, 2048, 2048, 8, 1)
    # x_perm + slot (rows_max x D bf16 each) dominate: rows_max = 16384*8 + 127*256 padded
    rows_max = (16384 * 8 + 127 * 256 + 127) // 128 * 128
    assert big > rows_max * 6144 * 2 * 2
    assert big < 6 * 2 ** 30


def test_layer_workspace_adds_router_parts_for_fp32_matrix_only():
    lib = moe.load_library()
    fw = lambda *a: lib.moe_forward_workspace(*a)
    lw = lambda *a: lib.moe_layer_forward_workspace(*a)
    for N, D, E in [(8192, 5120, 160), (300, 520, 48), (32, 4096, 128)]:
        base = fw(N, D, E, 256, 256, 8, 1)
        # fp32 W_g: three bf16 parts of E x D, 256-byte aligned
        parts = (3 * E * D * 2 + 255) // 256 * 256
        assert lw(N, D, E, 256, 256, 8, 1, 0) == base + parts
        assert lw(N, D, E, 256, 256, 8, 1, 1) == base       # bf16 W_g: no split
    assert lw(10, 64, 16, 32, 32, 2, 1, 7) == 0            # bad router dtype
    assert lw(10, 64, 16, 32, 32, 2, 9, 0) == 0            # bad dtype


def test_layer_call_rejects_bad_arguments_before_any_launch():
    lib = moe.load_library()
    call = lambda **kw: lib.moe_layer_forward(
        16, kw.get("W_g", 16), kw.get("wdt", 1), 16, kw.get("N", 10), kw.get("D", 64),
        kw.get("E", 16), kw.get("G", 1), kw.get("tg", 1), kw.get("k", 2), 1, 1.0, 16, 16, 16, 16,
        16, kw.get("d", 32), 32, kw.get("dt", 1), 16, 16, 16, kw.get("ws", 256),
        kw.get("wsb", 1 << 30), None)
    assert call(G=3) == -2                 # router shape
    assert call(k=40) == -2
    assert call(wdt=7) == -3               # router dtype
    assert call(dt=5) == -3                # forward dtype
    assert call(d=20) == -2                # forward shape (bf16 rows of 16 bytes)
    assert call(W_g=0) == -1               # null router matrix
    assert call(ws=0) == -4
    assert call(wsb=16) == -4
    assert call(N=0) == 0                  # no-op


def test_debug_hooks_reject_bad_arguments():
    lib = moe.load_library()
    assert lib.moe_debug_set_pair_mode(5) == -1
    assert lib.moe_debug_set_pair_mode(-2) == -1
    assert lib.moe_debug_set_pair_mode(-1) == 0
    assert lib.moe_debug_capture_scores(8, 16) == -1      # misaligned buffer
    assert lib.moe_debug_capture_scores(16, 0) == -1      # empty buffer
    assert lib.moe_debug_capture_scores(None, 0) == 0     # off


def test_bias_update_rejects_bad_arguments():
    lib = moe.load_library()
    assert lib.moe_bias_update(None, 4, 2, 600, 1e-3, 16, None, None) == -2      # E > 512
    assert lib.moe_bias_update(None, 4, 0, 16, 1e-3, 16, None, None) == -2       # k
    assert lib.moe_bias_update(None, 4, 2, 16, float("nan"), 16, None, None) == -1
    assert lib.moe_bias_update(None, 4, 2, 16, 1e-3, None, None, None) == -1     # null b
    assert lib.moe_bias_update(None, 4, 2, 16, 1e-3, 16, None, None) == -1       # null ids
