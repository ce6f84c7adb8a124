"""C-ABI checks that need no GPU: the library builds and loads, exports every
symbol include/dora.h declares, plans workspaces, and rejects bad arguments
before launching anything.

Every call below that passes placeholder pointers fails an argument check, so
no kernel is ever launched with them (also when this file runs on a GPU machine).
"""
import ctypes
import os
import re
import subprocess

import pytest

import dora_weight_decomposed_b200 as dw
from dora_weight_decomposed_b200 import build as dbuild
from dora_inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dora.h")


@pytest.fixture(scope="module")
def lib():
    dbuild.build()
    return dw.load_library()


def _header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DORA_API\s+[\w\s\*]+?\b(dora_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert _header_symbols() == sorted(dw.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", dw.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in _header_symbols():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # Internal helpers stay hidden.
    assert not any(n.startswith("_ZN4dora") for n in exported)


def test_version(lib):
    assert dw.dora_version() >= 100


def _desc(d_out=256, d_in=512, r=16, dtype=0, s=2.0):
    return dw.DoraDesc(d_out, d_in, r, dtype, s)


@pytest.mark.parametrize("key", sorted(WORKLOADS))
def test_workspace_plans(lib, key):
    wl = WORKLOADS[key]
    dt = 0 if wl.dtype == "bf16" else 1
    d = _desc(wl.d_out, wl.d_in, wl.r, dt, wl.s)
    sizes = [lib.dora_workspace_size(ctypes.byref(d), wl.T, op) for op in (0, 1, 2)]
    assert all(s > 0 for s in sizes)
    # Backward holds at least dz (T x d_out) in the storage type.
    assert sizes[2] >= wl.T * wl.d_out * (2 if dt == 0 else 4)
    # No batch, no forward/backward scratch.
    assert lib.dora_workspace_size(ctypes.byref(d), 0, 1) == 0
    assert lib.dora_workspace_size(ctypes.byref(d), 0, 2) == 0


def test_workspace_grows_with_tokens(lib):
    d = _desc(4096, 4096, 64)
    prev = 0
    for T in (1, 100, 1000, 5000):
        cur = lib.dora_workspace_size(ctypes.byref(d), T, 2)
        assert cur >= prev
        prev = cur


@pytest.mark.parametrize("bad", [dict(d_out=250), dict(d_in=100), dict(r=12), dict(r=520), dict(r=0),
                                 dict(d_out=0), dict(dtype=7), dict(s=float("nan"))])
def test_invalid_descriptors(lib, bad):
    d = _desc(**bad)
    assert lib.dora_workspace_size(ctypes.byref(d), 16, 0) == 0
    fake = ctypes.c_void_p(4096)
    st = lib.dora_norm(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == 1, dw.STATUS_NAMES.get(st)
    assert dw.dora_last_error()


def test_null_and_misaligned_pointers_rejected(lib):
    d = _desc()
    fake = ctypes.c_void_p(4096)
    # NULL W0
    st = lib.dora_norm(ctypes.byref(d), None, fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert st == 1 and "W0" in dw.dora_last_error()
    # misaligned A (bf16 needs 16 bytes)
    st = lib.dora_norm(ctypes.byref(d), fake, ctypes.c_void_p(4096 + 8), fake, fake, fake, fake, fake, fake,
                       1 << 30, None)
    assert st == 1 and "aligned" in dw.dora_last_error()
    # backward requires the saved forward tensors
    st = lib.dora_backward(ctypes.byref(d), 8, fake, fake, fake, fake, fake, fake, fake, None, fake, fake, fake,
                           fake, fake, fake, 1 << 30, None)
    assert st == 1 and "su_save" in dw.dora_last_error()
    # negative token count
    st = lib.dora_forward(ctypes.byref(d), -1, fake, fake, fake, fake, fake, fake, None, None, fake, 1 << 30, None)
    assert st == 1


def test_workspace_checks(lib):
    d = _desc()
    fake = ctypes.c_void_p(4096)
    need = lib.dora_workspace_size(ctypes.byref(d), 0, 0)
    assert need > 0
    st = lib.dora_norm(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, None, 0, None)
    assert st == 3 and "workspace" in dw.dora_last_error()
    st = lib.dora_norm(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, fake, need - 1, None)
    assert st == 3
    st = lib.dora_norm(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, ctypes.c_void_p(4096 + 16),
                       need, None)
    assert st == 1 and "256" in dw.dora_last_error()


def test_device_status_rejects_null(lib):
    assert lib.dora_device_status(None, None) == 1


def test_merge_validation(lib):
    d = _desc()
    fake = ctypes.c_void_p(4096)
    # The merge needs no workspace.
    assert lib.dora_workspace_size(ctypes.byref(d), 0, 3) == 0
    assert lib.dora_workspace_size(ctypes.byref(d), 0, 4) == 0
    st = lib.dora_merge(ctypes.byref(d), fake, fake, fake, fake, None, None, 0, None)
    assert st == 1 and "W_out" in dw.dora_last_error()
    st = lib.dora_merge(ctypes.byref(d), fake, fake, ctypes.c_void_p(4096 + 8), fake, fake, None, 0, None)
    assert st == 1 and "aligned" in dw.dora_last_error()
    bad = _desc(r=12)
    st = lib.dora_merge(ctypes.byref(bad), fake, fake, fake, fake, fake, None, 0, None)
    assert st == 1


@pytest.mark.parametrize("key", sorted(WORKLOADS))
def test_full_backward_workspace(lib, key):
    wl = WORKLOADS[key]
    dt = 0 if wl.dtype == "bf16" else 1
    d = _desc(wl.d_out, wl.d_in, wl.r, dt, wl.s)
    det = lib.dora_workspace_size(ctypes.byref(d), wl.T, 2)
    full = lib.dora_workspace_size(ctypes.byref(d), wl.T, 4)
    # The full gradient adds kappa, kappa * B and the Q = W' A^T partials (at least d_out x r fp32).
    assert full >= det + wl.d_out * wl.r * 4
    assert lib.dora_workspace_size(ctypes.byref(d), 0, 4) == 0


def test_full_backward_validation(lib):
    d = _desc()
    fake = ctypes.c_void_p(4096)
    st = lib.dora_backward_full(ctypes.byref(d), 8, fake, fake, fake, fake, fake, fake, fake, None, fake, fake, fake,
                                fake, fake, fake, 1 << 30, None)
    assert st == 1 and "su_save" in dw.dora_last_error()


def test_selftest_timeout_validation(lib):
    # Limits outside 1 us .. 1 s and a NULL scratch word are rejected before any launch.
    fake = ctypes.c_void_p(4096)
    assert lib.dora_selftest_timeout(0, fake, None) == 1
    assert lib.dora_selftest_timeout(1000001, fake, None) == 1
    assert lib.dora_selftest_timeout(1000, None, None) == 1 and "scratch" in dw.dora_last_error()
