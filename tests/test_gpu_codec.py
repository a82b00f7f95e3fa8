"""Exhaustive check of the GPU's E2M1 and UE4M3 conversions (the ones the quantizer
uses) against the oracle, over every fp32 bit pattern.

Both conversions are monotone in the input, so the oracle's answer over all 2^31
non-negative patterns is fixed by where it changes: the boundaries are found by
binary search over bit patterns with the oracle's brute-force nearest-value encoder,
and expanded on the device with searchsorted to the expected code of every pattern.
"""
import numpy as np
import pytest
import torch

from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu

POS_LIMIT = 0x7F800000  # +inf; patterns above are NaN (not inputs of the quantizer)


def _f32(bits: int) -> np.float32:
    return np.array([bits], dtype=np.uint32).view(np.float32)[0]


def _boundaries(encode, ncodes, lo=0, hi=POS_LIMIT):
    """For each code c >= 1: the smallest pattern p in [lo, hi] whose oracle code >= c."""
    out = []
    for c in range(1, ncodes):
        a, b = lo, hi + 1
        while a < b:
            mid = (a + b) // 2
            if encode(np.array([_f32(mid)]))[0] & 0x7F >= c:
                b = mid
            else:
                a = mid + 1
        out.append(a)
    return out


def _sweep(enc_gpu, bounds, sign_bit, mask, chunk=1 << 28):
    dev = torch.device("cuda")
    bt = torch.tensor(bounds, dtype=torch.int64, device=dev)
    mism = 0
    for start in range(0, POS_LIMIT + 1, chunk):
        stop = min(start + chunk, POS_LIMIT + 1)
        pat = torch.arange(start, stop, dtype=torch.int64, device=dev)
        want = torch.searchsorted(bt, pat, right=True).to(torch.uint8)
        if sign_bit:
            want = want | 8
            pat = pat | 0x80000000
        vals = pat.to(torch.int64).to(torch.int32).view(torch.float32) if not sign_bit else \
            (pat - (1 << 32)).to(torch.int32).view(torch.float32)
        got = enc_gpu(vals) & mask
        mism += int((got != want).sum())
        del pat, want, vals, got
    return mism


def test_e2m1_all_nonnegative_patterns():
    from diffusion_dit_b200 import fourtune as ft
    bounds = _boundaries(ora.e2m1_encode, 8)
    # sanity: the boundaries sit at the RNE tie points of {0,.5,1,1.5,2,3,4,6}
    assert _f32(bounds[0] - 1) == np.float32(0.25) and _f32(bounds[1]) == np.float32(0.75)
    assert _sweep(ft.encode_e2m1, bounds, sign_bit=False, mask=0xF) == 0


def test_e2m1_all_negative_patterns():
    from diffusion_dit_b200 import fourtune as ft
    bounds = _boundaries(ora.e2m1_encode, 8)
    assert _sweep(ft.encode_e2m1, bounds, sign_bit=True, mask=0xF) == 0


def test_ue4m3_all_nonnegative_patterns():
    from diffusion_dit_b200 import fourtune as ft
    bounds = _boundaries(ora.ue4m3_encode, 127)
    assert _sweep(ft.encode_ue4m3, bounds, sign_bit=False, mask=0xFF) == 0
