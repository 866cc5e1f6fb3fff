"""The C-ABI library builds, loads and exports every declared entry point;
host-side argument checks answer without a GPU (no compute is launched)."""

import ctypes
import os
import re

import pytest

from frame_wise_gated_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
        assert n in api.SIGNATURES, n


def test_version_and_status_strings(lib):
    assert lib.gdn_version() >= 100
    assert lib.gdn_status_string(0) == b"ok"
    assert lib.gdn_status_string(-4) == b"device wait timed out"


def test_workspace_bytes(lib):
    f = api.scan_flags(bf16=True)
    n = api.workspace_bytes(1, 16, 121, 3600, 128, f)
    # A, U and per-frame states (3 x 64 KiB per frame-head) plus span scratch
    assert n >= 3 * 1936 * 128 * 128 * 4
    assert api.workspace_bytes(1, 1, 1, 1, 17, f) == 0
    assert api.workspace_bytes(1, 16, 121, 3600, 128, f | api.FUSED_PROLOGUE) > n


def test_argument_errors_without_gpu(lib):
    null = None
    rc = lib.gdn_frame_scan_fwd(null, null, null, null, null, null, null, null,
                                1, 1, 4, 16, 17, api.BF16, null)
    assert rc == api.GDN_ERR_UNSUPPORTED
    rc = lib.gdn_frame_scan_fwd(null, null, null, null, null, null, null, null,
                                1, 1, 0, 16, 16, 0, null)
    assert rc == api.GDN_ERR_INVALID
    p = api.GdnParams()
    p.B, p.H, p.T, p.S, p.D = 1, 1, 2, 4, 16
    assert lib.gdn_frame_scan_fwd_ex(ctypes.byref(p), null) == api.GDN_ERR_INVALID
    assert b"null" in lib.gdn_last_error()
    assert lib.gdn_frame_scan_fwd_ex(None, null) == api.GDN_ERR_INVALID
    rc = lib.gdn_frame_scan_fwd(null, null, null, null, null, null, null, null,
                                1, 1, 4, 16, 16, api.FUSED_PROLOGUE, null)
    assert rc == api.GDN_ERR_INVALID


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "frame_wise_gated_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in txt and "from oracle" not in txt, f


def test_kernel_loads_never_multicast():
    """Every TMA or bulk load in the kernels writes only the issuing CTA's own
    shared memory: the only PTX that multicasts across a cluster is the MMA
    completion (tcgen05.commit) that releases a CTA pair's barriers."""
    needle = "multicast" + "::" + "cluster"  # split so this file names no such load
    csrc = os.path.join(ROOT, "frame_wise_gated_b200", "csrc")
    found = 0
    for f in sorted(os.listdir(csrc)):
        txt = open(os.path.join(csrc, f), encoding="utf-8").read()
        for line in re.findall(r'"([^"\n]*)"', txt):  # string literals: the inline PTX
            if needle in line:
                found += 1
                assert line.lstrip().startswith("tcgen05.commit"), (f, line)
    assert found >= 1  # the pair kernels' commits


def test_fault_injection_fails_before_any_launch(lib):
    """The armed injection turns the next scan call, once its arguments pass
    the checks, into GDN_ERR_CUDA without a launch (no GPU needed: the
    pointers are never dereferenced)."""
    fake = lambda i: ctypes.c_void_p(0x10000000 + 0x100000 * i)
    p = api.GdnParams()
    p.q, p.k, p.v, p.beta, p.gamma, p.out = (fake(i) for i in range(6))
    p.B, p.H, p.T, p.S, p.D = 1, 2, 3, 64, 128
    p.flags = api.BF16
    p.workspace = 0x40000000
    p.workspace_bytes = api.workspace_bytes(1, 2, 3, 64, 128, api.BF16)
    assert lib.gdn_fault_inject(1) == 0
    before = lib.gdn_launch_count(0)
    assert lib.gdn_frame_scan_fwd_ex(ctypes.byref(p), None) == api.GDN_ERR_CUDA
    assert b"injected" in lib.gdn_last_error()
    assert lib.gdn_launch_count(0) == before
    assert lib.gdn_fault_inject(0) == 0  # consumed by that one call
    # argument errors still come first: an invalid call does not consume it
    assert lib.gdn_fault_inject(1) == 0
    p.out = p.q
    assert lib.gdn_frame_scan_fwd_ex(ctypes.byref(p), None) == api.GDN_ERR_INVALID
    assert lib.gdn_fault_inject(0) == 1
