"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/dig_gla.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dig_gla.h")

OK, INVALID, UNSUPPORTED, ALIGN, CUDA = 0, -1, -2, -3, -4


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__._cuda_builder().build()  # by path: the package loads the library on import
    import gated_linear_attention_chunkwise_b200 as pkg
    return pkg.lib()


def test_header_declares_the_boundary():
    fns = declared_functions()
    for name in ("gla_fwd", "gla_fwd_f32", "srem_reorient", "dwconv3x3", "dig_gla_device_status",
                 "dig_gla_status_string", "dig_gla_release"):
        assert name in fns, name


def test_every_declared_symbol_is_exported(lib):
    so = lib._name
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [f for f in declared_functions() if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for f in declared_functions():
        assert hasattr(lib, f)


def test_status_strings(lib):
    import gated_linear_attention_chunkwise_b200 as pkg
    assert pkg.status_string(0) == "GLA_OK"
    for code, name in [(-1, "INVALID_ARG"), (-2, "UNSUPPORTED"), (-3, "ALIGNMENT"), (-4, "CUDA"),
                       (-5, "TIMEOUT"), (-6, "NOMEM"), (-7, "RANGE")]:
        assert pkg.status_string(code) == "GLA_ERR_" + name
    assert pkg.status_string(12345) == "GLA_ERR_UNKNOWN"


# Fake but well-aligned, non-overlapping device addresses: validation runs on the
# host before any CUDA call, so these are never dereferenced.
Q, K, V, LA, OUT = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000


def gla(lib, *, q=Q, k=K, v=V, la=LA, out=OUT, B=1, H=1, Hg=4, Wg=4, dk=64, dv=64, d=0, fn="gla_fwd"):
    return getattr(lib, fn)(q, k, v, la, B, H, Hg, Wg, dk, dv, d, out, None)


@pytest.mark.parametrize("fn", ["gla_fwd", "gla_fwd_f32"])
def test_gla_argument_validation(lib, fn):
    assert gla(lib, q=None, fn=fn) == INVALID
    assert gla(lib, out=None, fn=fn) == INVALID
    assert gla(lib, B=0, fn=fn) == INVALID
    assert gla(lib, Hg=-1, fn=fn) == INVALID
    assert gla(lib, d=12, fn=fn) == INVALID     # codes 0..3 SREM orders, 4..11 zigzag
    assert gla(lib, d=-1, fn=fn) == INVALID
    assert gla(lib, dk=60, fn=fn) == UNSUPPORTED       # not a multiple of 8
    assert gla(lib, dv=136, fn=fn) == UNSUPPORTED      # above 128
    assert gla(lib, B=300, H=300, fn=fn) == UNSUPPORTED
    assert gla(lib, q=Q + 8, fn=fn) == ALIGN
    assert gla(lib, out=OUT + 4, fn=fn) == ALIGN
    assert gla(lib, out=Q, fn=fn) == INVALID            # output aliases an input
    assert gla(lib, out=LA + 16, fn=fn) == INVALID      # partial overlap


def test_gla_valid_arguments_reach_the_device_check(lib):
    """Well-formed arguments pass validation and then fail only for want of an
    sm_100 device (no CPU fallback exists)."""
    import torch
    rc = gla(lib)
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the GPU tests")
    assert rc in (CUDA, UNSUPPORTED)


def test_grid_op_validation(lib):
    X, Y, W = 0x100000, 0x900000, 0x1100000
    assert lib.srem_reorient(None, 0, 0, 1, 4, 4, 64, 0, Y, None) == INVALID
    assert lib.srem_reorient(X, 12, 0, 1, 4, 4, 64, 0, Y, None) == INVALID
    assert lib.srem_reorient(X, 0, 2, 1, 4, 4, 64, 0, Y, None) == INVALID
    assert lib.srem_reorient(X, 0, 0, 1, 4, 4, 64, 7, Y, None) == INVALID
    assert lib.srem_reorient(X, 0, 0, 1, 4, 4, 12, 0, Y, None) == ALIGN     # 24-byte rows
    assert lib.srem_reorient(X, 0, 0, 1, 4, 4, 64, 0, X + 16, None) == INVALID
    assert lib.dwconv3x3(X, None, 1, 4, 4, 64, 0, Y, None) == INVALID
    assert lib.dwconv3x3(X, W + 4, 1, 4, 4, 64, 0, Y, None) == ALIGN
    assert lib.dwconv3x3(X, W, 0, 4, 4, 64, 0, Y, None) == INVALID
    assert lib.dwconv3x3(X, W, 1, 4, 4, 6, 1, Y, None) == ALIGN              # 24-byte rows (fp32)


def test_product_path_imports_no_oracle():
    """The binding and the CUDA sources never reference the oracle."""
    pkg_dir = os.path.join(ROOT, "gated_linear_attention_chunkwise_b200")
    for dirpath, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in text.lower(), f"{f} mentions the oracle"
