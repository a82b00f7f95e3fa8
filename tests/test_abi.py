"""The C-ABI library builds, loads without a GPU, exports every function that
include/fourtune.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from diffusion_dit_b200 import build as ftbuild
from diffusion_dit_b200 import fourtune as ft

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fourtune.h")


@pytest.fixture(scope="module")
def lib():
    ftbuild.build()
    return ft.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fourtune_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_three_layer_entry_points():
    names = declared_functions()
    for must in ("fourtune_linear_fwd", "fourtune_linear_bwd", "fourtune_quantize_block16"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in ft.EXPORTS, f"binding lacks {name}"


def test_status_strings(lib):
    assert lib.fourtune_status_string(0) == b"ok"
    assert lib.fourtune_status_string(2) == b"unsupported shape"
    assert lib.fourtune_status_string(99) == b"unknown status"


def _fp4(rows, cols, base=0x10000, sf=True):
    return ft.FtFp4(base, base + 0x1000, base + 0x2000 if sf else None, base + 0x3000, rows, cols)


def test_quantize_rejects_bad_arguments_on_host(lib):
    out = _fp4(32, 32, sf=False)
    q = lib.fourtune_quantize_block16
    # null input
    assert q(None, 0, 32, 32, 32, None, None, 0, None, ctypes.byref(out), None, None, 0, None) == 1
    # bad dtype
    assert q(0x10000, 7, 32, 32, 32, None, None, 0, None, ctypes.byref(out), None, None, 0, None) == 1
    # rows not a multiple of 16
    assert q(0x10000, 0, 24, 32, 32, None, None, 0, None, ctypes.byref(out), None, None, 0, None) == 2
    # shape of the output struct does not match
    bad = _fp4(16, 32, sf=False)
    assert q(0x10000, 0, 32, 32, 32, None, None, 0, None, ctypes.byref(bad), None, None, 0, None) == 2
    # misaligned input pointer
    assert q(0x10008, 0, 32, 32, 32, None, None, 0, None, ctypes.byref(out), None, None, 0, None) == 3
    # no workspace
    assert q(0x10000, 0, 32, 32, 32, None, None, 0, None, ctypes.byref(out), None, None, 0, None) == 4
    # the tensor-core scale layout needs 128-row bands
    with_sf = _fp4(32, 32, sf=True)
    assert q(0x10000, 0, 32, 32, 32, None, None, 0, None, ctypes.byref(with_sf), None, None, 0, None) == 2


def _layer(N=256, K=256, r_s=8, r=8):
    return ft.FtLinear(N, K, r_s, r, 1.0, _fp4(N, K, 0x100000), _fp4(K, N, 0x200000),
                       0x300000, 0x310000, 0x320000, 0x330000)


def test_linear_rejects_bad_arguments_on_host(lib):
    L = _layer()
    nws = lib.fourtune_linear_workspace_bytes(ctypes.byref(L), 128)
    assert nws > 0
    fwd = lib.fourtune_linear_fwd
    ws = 0x1000000
    # M not a multiple of 128
    assert fwd(ctypes.byref(L), 0x400000, 96, None, 0x500000, 0x600000, ws, nws, None) == 2
    # workspace too small
    assert fwd(ctypes.byref(L), 0x400000, 128, None, 0x500000, 0x600000, ws, nws - 1, None) == 4
    # N not a multiple of 256
    L2 = _layer(N=384)
    assert fwd(ctypes.byref(L2), 0x400000, 128, None, 0x500000, 0x600000, ws, 1 << 30, None) == 2
    # adapter rank above the supported 64
    L3 = _layer(r=80)
    assert fwd(ctypes.byref(L3), 0x400000, 128, None, 0x500000, 0x600000, ws, 1 << 30, None) == 2
    # missing stabilizer factor
    L4 = _layer()
    L4.ls_down = None
    assert fwd(ctypes.byref(L4), 0x400000, 128, None, 0x500000, 0x600000, ws, 1 << 30, None) == 1
    bwd = lib.fourtune_linear_bwd
    assert bwd(ctypes.byref(L), 0x400000, 0x600000, None, 128, None, 0x700000, 0x800000, 0x900000, ws,
               nws, None) == 1


def test_transposed_codes_may_be_absent_but_not_their_scale_layout(lib):
    # Q(R)^T transposed on the fly in the dX GEMM: qr_t.codes (and scales) NULL is valid;
    # qr_t's tensor-core scale layout and g stay required, with their shape and alignment.
    # Every call returns before any device work: an accepted layer stops at the misaligned
    # x pointer (3), or at M = 96 (2) where the case itself is an alignment error.
    bwd = lib.fourtune_linear_bwd
    ws = 0x1000000

    def call(L, M=128, x=0x400008):
        return bwd(ctypes.byref(L), x, 0x600000, 0x650000, M, None, 0x700000, 0x800000, 0x900000, ws,
                   1 << 30, None)

    def onfly():
        L = _layer()
        L.qr_t.codes = None
        L.qr_t.scales = None
        return L

    assert call(onfly()) == 3                 # accepted: the layer check passes
    L = onfly()
    L.qr_t.sf_mma = None
    assert call(L) == 1
    L = onfly()
    L.qr_t.g = None
    assert call(L) == 1
    L = onfly()
    L.qr_t.rows = 128                         # Q(R)^T must be K x N
    assert call(L) == 2
    L = onfly()
    L.qr_t.sf_mma = 0x200008                  # misaligned scale layout (accepted would give 2)
    assert call(L, M=96, x=0x400000) == 3
    L = onfly()
    L.qr.codes = None                         # Q(R)'s codes are the transposition's source
    assert call(L) == 1


def test_workspace_grows_with_tokens(lib):
    L = _layer(N=512, K=512, r_s=16, r=8)
    a = lib.fourtune_linear_workspace_bytes(ctypes.byref(L), 128)
    b = lib.fourtune_linear_workspace_bytes(ctypes.byref(L), 256)
    assert b > a > 0 and a % 256 == 0 and b % 256 == 0
