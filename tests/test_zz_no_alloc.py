"""The quantizer entry point that allocates nothing (fourtune_quantize_block16_noalloc).

It is for callers that cannot allocate device memory, e.g. a plugin interface that only
hands over its input and output buffers, or a host whose device memory is budgeted and
owned by another runtime.  Its scratch lives in a fixed array inside the library.  This
test calls it through the C ABI and checks that it gives exactly what the workspace entry
point gives on the same inputs, on two calls in a row (the second with other data, so
nothing left in the shared array from the first call can leak into the second), and that
a problem too large for the array is refused.  The array's status word, where a kernel
would report a bounded wait that gave up, reads back FT_OK through fourtune_device_status
with a NULL workspace.  This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _noalloc(ft, x, down):
    rows, cols = x.shape
    r = down.shape[0]
    q = ft.QuantizedMatrix.empty(rows, cols, x.device, with_sf=True)
    t = torch.empty(rows, r, dtype=torch.float32, device=x.device)
    qs = q.c_struct()
    st = ft.lib().fourtune_quantize_block16_noalloc(
        ctypes.c_void_p(x.data_ptr()), ft.FT_DTYPE_BF16, rows, cols, cols, None, ctypes.c_void_p(down.data_ptr()),
        r, ctypes.c_void_p(t.data_ptr()), ctypes.byref(qs), None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, ft.STATUS.get(st, st)
    return q, t


def _noalloc_status(ft):
    v = ctypes.c_int32(-1)
    st = ft.lib().fourtune_device_status(None, ctypes.byref(v),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, ft.STATUS.get(st, st)
    return int(v.value)


def test_noalloc_matches_the_workspace_entry_point_on_two_calls():
    ft = _ft()
    for seed, (rows, cols) in ((0, (1024, 3072)), (1, (512, 1536))):
        x, down = wl.make_quant_input(wl.QuantSpec("t", rows, cols, 32, 0.01, 10.0), seed=seed)
        xg, dg = x.cuda(), down.cuda()
        q_ref, _, t_ref = ft.quantize_block16(xg, with_sf=True, down=dg)
        q, t = _noalloc(ft, xg, dg)
        torch.cuda.synchronize()
        assert q.g.item() == q_ref.g.item()
        assert torch.equal(q.codes, q_ref.codes)
        assert torch.equal(q.scales, q_ref.scales)
        assert torch.equal(q.sf_mma, q_ref.sf_mma)
        # the down-projection within the tolerance the other tests use against fp64
        assert ora.rel_frobenius(t.double().cpu().numpy(), t_ref.double().cpu().numpy()) < 1e-5
        # the fixed array's status word (read and cleared with a NULL workspace): no timeout
        assert _noalloc_status(ft) == 0


def test_noalloc_refuses_problems_beyond_its_scratch():
    ft = _ft()
    rows, cols, r = 65536, 8192, 64          # needs far more scratch than the fixed array
    assert ft.lib().fourtune_quantize_workspace_bytes(rows, cols, r) > ft.NOALLOC_SCRATCH_BYTES
    fake = ft.FtFp4(0x100000, 0x200000, 0x300000, 0x400000, rows, cols)
    st = ft.lib().fourtune_quantize_block16_noalloc(
        ctypes.c_void_p(0x10000), ft.FT_DTYPE_BF16, rows, cols, cols, None, ctypes.c_void_p(0x20000), r,
        ctypes.c_void_p(0x30000), ctypes.byref(fake), None, None)
    assert st == 4  # FT_ERR_WORKSPACE, before any launch
