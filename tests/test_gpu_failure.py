"""Failure detection on the GPU without a fault: a kernel's bounded wait runs out on a
barrier that nothing completes, the kernel reports FT_ERR_TIMEOUT through the status
word and returns, and the context keeps working."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    from diffusion_dit_b200 import fourtune as ft
    from diffusion_dit_b200 import workloads as wl
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert ft.lib().fourtune_selftest_bounded_wait(2_000_000, ctypes.c_void_p(ws.data_ptr()), stream) == 0
    torch.cuda.synchronize()
    st = ctypes.c_int32(-1)
    assert ft.lib().fourtune_device_status(ctypes.c_void_p(ws.data_ptr()), ctypes.byref(st), stream) == 0
    assert st.value == 7  # FT_ERR_TIMEOUT
    # reading cleared it
    assert ft.lib().fourtune_device_status(ctypes.c_void_p(ws.data_ptr()), ctypes.byref(st), stream) == 0
    assert st.value == 0
    # the context still runs the real kernels
    x = wl.make_gaussian_bf16((128, 256), 1.0, 3).cuda()
    q, _, _ = ft.quantize_block16(x, with_sf=True)
    torch.cuda.synchronize()
    assert q.g.item() > 0


def test_selftest_rejects_bad_limits():
    from diffusion_dit_b200 import fourtune as ft
    assert ft.lib().fourtune_selftest_bounded_wait(0, ctypes.c_void_p(0x1000), None) == 1
    assert ft.lib().fourtune_selftest_bounded_wait(5_000_000_000, ctypes.c_void_p(0x1000), None) == 1
