"""CPU-side checks of the C ABI: the library loads, exports every function the
header declares, sizes workspaces and rejects bad arguments before touching
the GPU."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

from coreset_attention_approximation_b200 import wildcat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wildcat.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wc_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(wildcat.LIB_PATH):
        from coreset_attention_approximation_b200 import build

        build.build()
    return wildcat.lib()


def test_header_declares_the_expected_calls():
    names = declared_functions()
    for want in ["wc_select", "wc_weights", "wc_attend", "wc_forward", "wc_workspace_bytes",
                 "wc_check_device_status", "wc_status_string"]:
        assert want in names


def test_library_exports_every_declared_function(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", wildcat.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (wc_\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    assert set(wildcat.EXPORTS) <= exported


def test_debug_library_exports_the_same_functions(lib):
    """The bounds-checked build (libwildcat_debug.so) is the same ABI."""
    path = os.path.join(os.path.dirname(wildcat.LIB_PATH), "libwildcat_debug.so")
    if not os.path.exists(path):
        from coreset_attention_approximation_b200 import build

        build.build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (wc_\w+)$", out, flags=re.M))
    assert not [n for n in declared_functions() if n not in exported]
    d = ctypes.CDLL(path)
    d.wc_status_string.restype = ctypes.c_char_p
    assert d.wc_status_string(7) == b"index outside its buffer (debug build)"


def test_status_strings(lib):
    assert lib.wc_status_string(0) == b"ok"
    assert lib.wc_status_string(5) == b"workspace too small"
    assert lib.wc_status_string(7) == b"index outside its buffer (debug build)"
    assert lib.wc_status_string(99) == b"unknown status"


def test_f_ld_rounds_to_sixty_four(lib):
    assert [wildcat.f_ld(n) for n in (1, 63, 64, 65, 1000, 131072)] == [64, 64, 64, 128, 1024, 131072]


def test_workspace_sizes(lib):
    s = wildcat.make_shape(1, 8, 8, 131072, 131072, 128, 128, 2048, torch.bfloat16)
    scratch, full = wildcat.workspace_bytes(s), wildcat.forward_workspace_bytes(s)
    assert scratch > 8 * 128 * 131072 * 2          # holds the transposed keys
    assert full - scratch >= 8 * 2048 * 131072 * 4  # and room for F when not given
    assert scratch % 256 == 0 and full % 256 == 0


@pytest.mark.parametrize("field,value", [
    ("r", 0), ("r", 600), ("d", 12), ("dv", 0), ("hq", 3), ("n_k", 0), ("dtype", 7), ("batch", 0),
    ("scale", -1.0), ("eps_stop", float("nan")), ("d", 264),
])
def test_invalid_shapes_are_rejected_without_a_gpu(lib, field, value):
    s = wildcat.make_shape(1, 2, 2, 512, 16, 64, 64, 32, torch.float32)
    setattr(s, field, value)
    assert wildcat.workspace_bytes(s) == 0
    dummy = ctypes.c_void_p(256)
    code = lib.wc_select(ctypes.byref(s), dummy, dummy, dummy, dummy, dummy, 1 << 30, None)
    assert code == 1


def test_null_and_misaligned_pointers_are_rejected(lib):
    s = wildcat.make_shape(1, 1, 1, 512, 16, 64, 64, 32, torch.float32)
    ok = ctypes.c_void_p(1 << 20)
    assert lib.wc_select(ctypes.byref(s), None, ok, ok, ok, ok, 1 << 30, None) == 1
    assert lib.wc_select(ctypes.byref(s), ctypes.c_void_p((1 << 20) + 4), ok, ok, ok, ok, 1 << 30, None) == 1
    # workspace not 256-byte aligned, then too small
    assert lib.wc_select(ctypes.byref(s), ok, ok, ok, ok, ctypes.c_void_p((1 << 20) + 16), 1 << 30, None) == 1
    assert lib.wc_select(ctypes.byref(s), ok, ok, ok, ok, ok, 1024, None) == 5
    assert lib.wc_selftest_wait_timeout(ok, 100, 10, None) == 1


def test_product_path_does_not_import_the_oracle():
    # the binding and the library sources never reach the oracle
    pkg = os.path.join(ROOT, "coreset_attention_approximation_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "wc_oracle" not in text, f


def test_every_entry_point_checks_its_arguments(lib):
    """weights, attend, forward and the allocation-free attend refuse null and
    misaligned pointers, short workspaces and invalid shapes before any
    launch, so no GPU is needed to see the codes."""
    s = wildcat.make_shape(1, 2, 1, 512, 16, 64, 64, 32, torch.bfloat16)
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 30
    # weights: K, V, piv, F, rank, Ks, W
    assert lib.wc_weights(ctypes.byref(s), None, ok, ok, ok, ok, ok, ok, ok, big, None) == 1
    assert lib.wc_weights(ctypes.byref(s), ok, ok, ok, ok, ok, ok, mis, ok, big, None) == 1
    assert lib.wc_weights(ctypes.byref(s), ok, ok, ok, ok, ok, ok, ok, ok, 1024, None) == 5
    # attend: Q, Ks, W, rank, out
    assert lib.wc_attend(ctypes.byref(s), None, ok, ok, ok, ok, ok, big, None) == 1
    assert lib.wc_attend(ctypes.byref(s), ok, ok, ok, ok, mis, ok, big, None) == 1
    assert lib.wc_attend(ctypes.byref(s), ok, ok, ok, ok, ok, ok, 1024, None) == 5
    # forward: Q, K, V, out, piv, rank, F, Ks, W (the last five nullable, then the workspace must hold them)
    assert lib.wc_forward(ctypes.byref(s), ok, None, ok, ok, None, None, None, None, None, ok, big, None) == 1
    assert lib.wc_forward(ctypes.byref(s), ok, ok, ok, ok, None, None, None, None, None, ok,
                          wildcat.workspace_bytes(s), None) == 5
    # allocation-free attend
    assert lib.wc_attend_noalloc(ctypes.byref(s), None, ok, ok, ok, ok, None) == 1
    # an invalid shape is refused by every call
    bad = wildcat.make_shape(1, 3, 2, 512, 16, 64, 64, 32, torch.bfloat16)   # hq not a multiple of hkv
    assert lib.wc_weights(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, ok, ok, big, None) == 1
    assert lib.wc_attend(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, big, None) == 1
    assert lib.wc_forward(ctypes.byref(bad), ok, ok, ok, ok, ok, ok, ok, ok, ok, ok, big, None) == 1
    assert lib.wc_attend_noalloc(ctypes.byref(bad), ok, ok, ok, ok, ok, None) == 1
    # bins and centring: n and r must be multiples of bins; center is 0 or 1
    for field, value in (("bins", 3), ("bins", -1), ("center", 2), ("unit_base", -1)):
        b2 = wildcat.make_shape(1, 2, 1, 512, 16, 64, 64, 32, torch.bfloat16)
        setattr(b2, field, value)
        assert wildcat.workspace_bytes(b2) == 0
        assert lib.wc_select(ctypes.byref(b2), ok, ok, ok, ok, ok, big, None) == 1


def test_one_workspace_holds_every_calls_scratch(lib):
    """A workspace sized for the whole problem (queries and values included)
    holds the scratch of select (no queries, the binding's 8-wide placeholder
    values), weights (no queries) and attend, with and without bins, centring
    and the decode-sized attention split."""
    cases = [
        (1, 8, 8, 131072, 131072, 128, 128, 2048, {}),
        (1, 32, 8, 32768, 256, 128, 128, 1024, {}),            # decode-sized: attention splits
        (2, 16, 16, 4096, 4096, 64, 64, 256, {"center": True}),
        (1, 8, 8, 131072, 131072, 128, 128, 2048, {"bins": 8}),
        (1, 1, 1, 512, 512, 64, 64, 32, {}),
    ]
    for b, hq, hkv, n, nq, d, dv, r, kw in cases:
        full = wildcat.workspace_bytes(wildcat.make_shape(b, hq, hkv, n, nq, d, dv, r, torch.bfloat16, **kw))
        select = wildcat.workspace_bytes(wildcat.make_shape(b, hkv, hkv, n, 0, d, 8, r, torch.bfloat16, **kw))
        weights = wildcat.workspace_bytes(wildcat.make_shape(b, hkv, hkv, n, 0, d, dv, r, torch.bfloat16, **kw))
        assert 0 < select <= full and 0 < weights <= full, (n, r, kw)
