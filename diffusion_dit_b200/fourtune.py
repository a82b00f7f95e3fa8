"""Python binding of the C ABI in include/fourtune.h (argument marshalling only).

Every step of the layer runs in the CUDA library ``_lib/libfourtune.so``; this module
allocates device tensors with PyTorch, passes raw pointers and the current stream,
and raises on any non-OK status.  There is no fallback: if the library is missing or
the device is not sm_100 the calls fail loudly.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libfourtune.so")

FT_DTYPE_BF16 = 0
FT_DTYPE_F32 = 1
# size of the fixed scratch array behind fourtune_quantize_block16_noalloc
NOALLOC_SCRATCH_BYTES = 8 << 20

STATUS = {0: "FT_OK", 1: "FT_ERR_INVALID_ARG", 2: "FT_ERR_SHAPE", 3: "FT_ERR_ALIGN",
          4: "FT_ERR_WORKSPACE", 5: "FT_ERR_CUDA", 6: "FT_ERR_UNSUPPORTED", 7: "FT_ERR_TIMEOUT"}


class FourTuneError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class FtFp4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("sf_mma", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class FtLinear(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64), ("r_s", ctypes.c_int32),
                ("r", ctypes.c_int32), ("lora_scale", ctypes.c_float), ("qr", FtFp4),
                ("qr_t", FtFp4), ("ls_down", ctypes.c_void_p), ("ls_up", ctypes.c_void_p),
                ("lora_a", ctypes.c_void_p), ("lora_b", ctypes.c_void_p)]


EXPORTS = {
    # name: (argtypes, restype)
    "fourtune_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "fourtune_quantize_workspace_bytes": ([ctypes.c_int64, ctypes.c_int64, ctypes.c_int32], ctypes.c_size_t),
    "fourtune_quantize_block16": ([ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64,
                                   ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                   ctypes.c_void_p, ctypes.POINTER(FtFp4), ctypes.POINTER(FtFp4),
                                   ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "fourtune_linear_workspace_bytes": ([ctypes.POINTER(FtLinear), ctypes.c_int64], ctypes.c_size_t),
    "fourtune_linear_fwd": ([ctypes.POINTER(FtLinear), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                             ctypes.c_void_p], ctypes.c_int),
    "fourtune_quantize_1x16": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                ctypes.POINTER(FtFp4), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
                               ctypes.c_int),
    "fourtune_linear_fwd_1x16": ([ctypes.POINTER(FtLinear), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                  ctypes.c_void_p], ctypes.c_int),
    "fourtune_linear_fwd_gelu": ([ctypes.POINTER(FtLinear), ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p], ctypes.c_int),
    "fourtune_linear_bwd": ([ctypes.POINTER(FtLinear), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                             ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
                            ctypes.c_int),
    "fourtune_linear_bwd_gelu": ([ctypes.POINTER(FtLinear), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                  ctypes.c_void_p], ctypes.c_int),
    "fourtune_device_status": ([ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.c_void_p], ctypes.c_int),
    "fourtune_gelu_tanh_fwd": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p], ctypes.c_int),
    "fourtune_gelu_tanh_bwd": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                ctypes.c_void_p], ctypes.c_int),
    "fourtune_encode_e2m1": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "fourtune_encode_ue4m3": ([ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "fourtune_quantize_block16_noalloc": ([ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.POINTER(FtFp4), ctypes.POINTER(FtFp4),
                                           ctypes.c_void_p], ctypes.c_int),
    "fourtune_launch_count": ([], ctypes.c_uint64),
    "fourtune_selftest_bounded_wait": ([ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "fourtune_time_next_launch": ([ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
}

FT_KERNEL_GEMM, FT_KERNEL_QUANT, FT_KERNEL_AMAX, FT_KERNEL_LOWRANK, FT_KERNEL_LORA_DB, FT_KERNEL_LORA_DA = range(6)

_lib = None


def lib():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run diffusion_dit_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (argt, rest) in EXPORTS.items():
            fn = getattr(L, name)
            fn.argtypes = argt
            fn.restype = rest
        _lib = L
    return _lib


def _check(name: str, status: int):
    if status != 0:
        raise FourTuneError(name, status)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


# ---------------------------------------------------------------------------
@dataclasses.dataclass
class QuantizedMatrix:
    """Device tensors of one 16x16-block quantized matrix (see ft_fp4)."""

    codes: Optional[torch.Tensor]   # uint8 [rows, cols/2] (None: see drop_transposed_codes)
    scales: Optional[torch.Tensor]  # uint8 [rows/16, cols/16]
    sf_mma: Optional[torch.Tensor]  # uint8 [rows * cols / 16] or None
    g: torch.Tensor                # float32 [1]
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device, with_sf: bool = True, block_rows: int = 16) -> "QuantizedMatrix":
        return QuantizedMatrix(
            codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=device),
            scales=torch.empty(rows // block_rows, cols // 16, dtype=torch.uint8, device=device),
            sf_mma=torch.empty(rows * cols // 16, dtype=torch.uint8, device=device) if with_sf else None,
            g=torch.empty(1, dtype=torch.float32, device=device), rows=rows, cols=cols)

    def c_struct(self) -> FtFp4:
        def ptr(t):
            return t.data_ptr() if t is not None else None
        return FtFp4(ptr(self.codes), ptr(self.scales), ptr(self.sf_mma), self.g.data_ptr(), self.rows, self.cols)


def quantize_block16(x: torch.Tensor, amax: Optional[torch.Tensor] = None, with_sf: bool = False,
                     transposed: bool = False, down: Optional[torch.Tensor] = None,
                     stream=None):
    """Q(x) in 16x16 blocks on the GPU.  Returns (q, q_t or None, down_out or None)."""
    _require_cuda(x, amax, down)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a row-major 2-D tensor")
    rows, cols = x.shape
    dt = {torch.bfloat16: FT_DTYPE_BF16, torch.float32: FT_DTYPE_F32}[x.dtype]
    q = QuantizedMatrix.empty(rows, cols, x.device, with_sf=with_sf or transposed)
    qt = QuantizedMatrix.empty(cols, rows, x.device, with_sf=True) if transposed else None
    r_down = 0 if down is None else down.shape[0]
    down_out = torch.empty(rows, r_down, dtype=torch.float32, device=x.device) if r_down else None
    nws = lib().fourtune_quantize_workspace_bytes(rows, cols, r_down)
    ws = torch.zeros(nws, dtype=torch.uint8, device=x.device)
    qs = q.c_struct()
    qts = qt.c_struct() if qt is not None else None
    st = lib().fourtune_quantize_block16(_p(x), dt, rows, cols, x.stride(0), _p(amax), _p(down), r_down,
                                         _p(down_out), ctypes.byref(qs),
                                         ctypes.byref(qts) if qts is not None else None,
                                         _p(ws), nws, _stream(stream))
    _check("fourtune_quantize_block16", st)
    return q, qt, down_out


def quantize_block16_into(x: torch.Tensor, q: QuantizedMatrix, ws: torch.Tensor, amax: Optional[torch.Tensor] = None,
                          down: Optional[torch.Tensor] = None, down_out: Optional[torch.Tensor] = None,
                          q_t: Optional[QuantizedMatrix] = None, stream=None):
    """Q(x) in 16x16 blocks into preallocated outputs with a caller workspace ``ws`` (uint8,
    at least fourtune_quantize_workspace_bytes): allocates nothing, so it can be captured
    in a CUDA graph.  ``down`` [r, cols] bf16 with ``down_out`` [rows, r] fp32: the fused
    down-projection x down^T."""
    _require_cuda(x, amax, down, down_out, ws)
    rows, cols = x.shape
    dt = {torch.bfloat16: FT_DTYPE_BF16, torch.float32: FT_DTYPE_F32}[x.dtype]
    r_down = 0 if down is None else down.shape[0]
    qs = q.c_struct()
    qts = q_t.c_struct() if q_t is not None else None
    st = lib().fourtune_quantize_block16(_p(x), dt, rows, cols, x.stride(0), _p(amax), _p(down), r_down,
                                         _p(down_out), ctypes.byref(qs),
                                         ctypes.byref(qts) if qts is not None else None,
                                         _p(ws), ws.numel(), _stream(stream))
    _check("fourtune_quantize_block16", st)


def quantize_1x16(x: torch.Tensor, amax: Optional[torch.Tensor] = None, with_sf: bool = True, stream=None):
    """Q(x) in group-wise 1x16 blocks (scales [rows, cols/16]) on the GPU; bf16 x."""
    _require_cuda(x, amax)
    if x.dim() != 2 or x.stride(1) != 1 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a row-major 2-D bf16 tensor")
    rows, cols = x.shape
    q = QuantizedMatrix.empty(rows, cols, x.device, with_sf=with_sf, block_rows=1)
    nws = lib().fourtune_quantize_workspace_bytes(rows, cols, 0)
    ws = torch.zeros(nws, dtype=torch.uint8, device=x.device)
    qs = q.c_struct()
    st = lib().fourtune_quantize_1x16(_p(x), rows, cols, x.stride(0), _p(amax), ctypes.byref(qs), _p(ws), nws,
                                      _stream(stream))
    _check("fourtune_quantize_1x16", st)
    return q


@dataclasses.dataclass
class LinearWeights:
    """Frozen backbone + adapter of one layer, on the device."""

    qr: QuantizedMatrix
    qr_t: QuantizedMatrix
    ls_down: torch.Tensor   # bf16 [r_s, K]
    ls_up: torch.Tensor     # bf16 [N, r_s]
    lora_a: torch.Tensor    # bf16 [r, K]
    lora_b: torch.Tensor    # bf16 [N, r]
    lora_scale: float

    @property
    def N(self):
        return self.qr.rows

    @property
    def K(self):
        return self.qr.cols

    @property
    def r_s(self):
        return self.ls_down.shape[0]

    @property
    def r(self):
        return self.lora_a.shape[0]

    def c_struct(self) -> FtLinear:
        return FtLinear(self.N, self.K, self.r_s, self.r, self.lora_scale, self.qr.c_struct(),
                        self.qr_t.c_struct(), self.ls_down.data_ptr() if self.r_s else None,
                        self.ls_up.data_ptr() if self.r_s else None,
                        self.lora_a.data_ptr() if self.r else None,
                        self.lora_b.data_ptr() if self.r else None)


def prepare_weights(residual: torch.Tensor, ls_up: torch.Tensor, ls_down: torch.Tensor,
                    lora_a: torch.Tensor, lora_b: torch.Tensor, lora_scale: float,
                    transpose_on_the_fly: bool = False) -> LinearWeights:
    """Q(R) offline (section 3.1) with its transposed copy (section 3.2), on the GPU.
    ``residual`` is the fp32 (or bf16) R [N, K] on the device.  With
    ``transpose_on_the_fly`` the transposed codes are not kept (drop_transposed_codes)."""
    qr, qr_t, _ = quantize_block16(residual.contiguous(), with_sf=True, transposed=True)
    w = LinearWeights(qr, qr_t, ls_down.contiguous(), ls_up.contiguous(), lora_a.contiguous(),
                      lora_b.contiguous(), float(lora_scale))
    return drop_transposed_codes(w) if transpose_on_the_fly else w


def drop_transposed_codes(w: LinearWeights) -> LinearWeights:
    """The same layer without Q(R)^T's codes and scale grid (N*K/2 + N*K/256 bytes): the
    backward's dX GEMM then transposes Q(R)'s codes tile by tile in shared memory (section
    3.2).  Q(R)^T's tensor-core scale layout and g are kept.  Shares every other tensor."""
    return dataclasses.replace(w, qr_t=dataclasses.replace(w.qr_t, codes=None, scales=None))


class Workspace:
    """Caller-owned scratch for the layer calls, sized by the library's query."""

    def __init__(self, weights: LinearWeights, M: int, device):
        s = weights.c_struct()
        self.nbytes = int(lib().fourtune_linear_workspace_bytes(ctypes.byref(s), M))
        self.buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)
        self.M = M

    def device_status(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        _check("fourtune_device_status",
               lib().fourtune_device_status(_p(self.buf), ctypes.byref(v), _stream(stream)))
        return int(v.value)


def linear_fwd(w: LinearWeights, x: torch.Tensor, ws: Workspace, y: Optional[torch.Tensor] = None,
               t_saved: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None, stream=None):
    """Eq. (2).  Returns (Y bf16 [M, N], T fp32 [M, r_s + r])."""
    _require_cuda(x)
    M = x.shape[0]
    if y is None:
        y = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    R = w.r_s + w.r
    if t_saved is None:
        t_saved = torch.empty(M, max(R, 1), dtype=torch.float32, device=x.device)
    s = w.c_struct()
    st = lib().fourtune_linear_fwd(ctypes.byref(s), _p(x), M, _p(amax), _p(y), _p(t_saved), _p(ws.buf),
                                   ws.nbytes, _stream(stream))
    _check("fourtune_linear_fwd", st)
    return y, t_saved


def linear_fwd_1x16(w: LinearWeights, x: torch.Tensor, ws: Workspace, y: Optional[torch.Tensor] = None,
                    t_saved: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None, stream=None):
    """Eq. (2) with X quantized group-wise 1x16 (forward only).  Returns (Y, T)."""
    _require_cuda(x)
    M = x.shape[0]
    if y is None:
        y = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    R = w.r_s + w.r
    if t_saved is None:
        t_saved = torch.empty(M, max(R, 1), dtype=torch.float32, device=x.device)
    s = w.c_struct()
    st = lib().fourtune_linear_fwd_1x16(ctypes.byref(s), _p(x), M, _p(amax), _p(y), _p(t_saved), _p(ws.buf),
                                        ws.nbytes, _stream(stream))
    _check("fourtune_linear_fwd_1x16", st)
    return y, t_saved


def linear_fwd_gelu(w: LinearWeights, x: torch.Tensor, ws: Workspace, p: Optional[torch.Tensor] = None,
                    h: Optional[torch.Tensor] = None, h_amax: Optional[torch.Tensor] = None,
                    t_saved: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None, stream=None):
    """Eq. (2) with GELU fused into the GEMM epilogue (an MLP's first linear).
    Returns (P bf16 [M, N], H = bf16(gelu_tanh(P)) [M, N], max|H| fp32 [1], T fp32 [M, r_s + r])."""
    _require_cuda(x)
    M = x.shape[0]
    if p is None:
        p = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    if h is None:
        h = torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    if h_amax is None:
        h_amax = torch.empty(1, dtype=torch.float32, device=x.device)
    R = w.r_s + w.r
    if t_saved is None:
        t_saved = torch.empty(M, max(R, 1), dtype=torch.float32, device=x.device)
    s = w.c_struct()
    st = lib().fourtune_linear_fwd_gelu(ctypes.byref(s), _p(x), M, _p(amax), _p(p), _p(h), _p(h_amax),
                                        _p(t_saved), _p(ws.buf), ws.nbytes, _stream(stream))
    _check("fourtune_linear_fwd_gelu", st)
    return p, h, h_amax, t_saved


def linear_bwd(w: LinearWeights, x: torch.Tensor, t_saved: torch.Tensor, dy: torch.Tensor, ws: Workspace,
               dx: Optional[torch.Tensor] = None, da: Optional[torch.Tensor] = None,
               db: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None, stream=None):
    """Eq. (3) and the adapter gradients.  Returns (dX bf16 [M, K], dA fp32 [r, K], dB fp32 [N, r])."""
    _require_cuda(x, t_saved, dy)
    M = x.shape[0]
    if dx is None:
        dx = torch.empty(M, w.K, dtype=torch.bfloat16, device=x.device)
    if da is None:
        da = torch.empty(max(w.r, 1), w.K, dtype=torch.float32, device=x.device)
    if db is None:
        db = torch.empty(w.N, max(w.r, 1), dtype=torch.float32, device=x.device)
    s = w.c_struct()
    st = lib().fourtune_linear_bwd(ctypes.byref(s), _p(x), _p(t_saved), _p(dy), M, _p(amax), _p(dx), _p(da),
                                   _p(db), _p(ws.buf), ws.nbytes, _stream(stream))
    _check("fourtune_linear_bwd", st)
    return dx, da, db


def linear_bwd_gelu(w: LinearWeights, x: torch.Tensor, t_saved: torch.Tensor, dy: torch.Tensor, p: torch.Tensor,
                    ws: Workspace, dp: Optional[torch.Tensor] = None, da: Optional[torch.Tensor] = None,
                    db: Optional[torch.Tensor] = None, amax: Optional[torch.Tensor] = None, stream=None):
    """Backward of an MLP's second linear with gelu' fused into the dX GEMM's epilogue.
    Returns (dP = bf16(dX * gelu'(p)) bf16 [M, K], dA fp32 [r, K], dB fp32 [N, r])."""
    _require_cuda(x, t_saved, dy, p)
    M = x.shape[0]
    if dp is None:
        dp = torch.empty(M, w.K, dtype=torch.bfloat16, device=x.device)
    if da is None:
        da = torch.empty(max(w.r, 1), w.K, dtype=torch.float32, device=x.device)
    if db is None:
        db = torch.empty(w.N, max(w.r, 1), dtype=torch.float32, device=x.device)
    s = w.c_struct()
    st = lib().fourtune_linear_bwd_gelu(ctypes.byref(s), _p(x), _p(t_saved), _p(dy), M, _p(amax), _p(p), _p(dp),
                                        _p(da), _p(db), _p(ws.buf), ws.nbytes, _stream(stream))
    _check("fourtune_linear_bwd_gelu", st)
    return dp, da, db


def gelu_tanh_fwd(p: torch.Tensor, h: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _require_cuda(p)
    h = torch.empty_like(p) if h is None else h
    _check("fourtune_gelu_tanh_fwd", lib().fourtune_gelu_tanh_fwd(_p(p), _p(h), p.numel(), _stream(stream)))
    return h


def gelu_tanh_bwd(p: torch.Tensor, dh: torch.Tensor, dp: Optional[torch.Tensor] = None, stream=None):
    _require_cuda(p, dh)
    dp = torch.empty_like(p) if dp is None else dp
    _check("fourtune_gelu_tanh_bwd",
           lib().fourtune_gelu_tanh_bwd(_p(p), _p(dh), _p(dp), p.numel(), _stream(stream)))
    return dp


def encode_e2m1(v: torch.Tensor, stream=None) -> torch.Tensor:
    _require_cuda(v)
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check("fourtune_encode_e2m1", lib().fourtune_encode_e2m1(_p(v), v.numel(), _p(out), _stream(stream)))
    return out


def encode_ue4m3(v: torch.Tensor, stream=None) -> torch.Tensor:
    _require_cuda(v)
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    _check("fourtune_encode_ue4m3", lib().fourtune_encode_ue4m3(_p(v), v.numel(), _p(out), _stream(stream)))
    return out


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(lib().fourtune_launch_count())


def time_next_launch(kind: int, before: Optional[torch.cuda.Event], after: Optional[torch.cuda.Event]):
    """Have the library record ``before``/``after`` (timing events) around its next
    launch of kernel ``kind`` (FT_KERNEL_*), on that launch's stream.  The events must
    already exist (torch creates a CUDA event at its first record())."""
    for e in (before, after):
        if e is not None and not e.cuda_event:
            raise ValueError("record the event once before handing it to the library")
    b = ctypes.c_void_p(before.cuda_event) if before is not None else None
    a = ctypes.c_void_p(after.cuda_event) if after is not None else None
    _check("fourtune_time_next_launch", lib().fourtune_time_next_launch(kind, b, a))


class FourTuneLinearFunction(torch.autograd.Function):
    """autograd wrapper: forward Eq. (2), backward Eq. (3) + adapter gradients.

    ``lora_a`` [r, K] and ``lora_b`` [N, r] are the adapter parameters this call uses (any
    float dtype; the layer computes with their bf16 values), so a caller that replaces or
    updates them is always seen; ``weights`` supplies the frozen Q(R), Q(R)^T and
    stabilizer factors (its own lora_a / lora_b are ignored).  Gradients flow to X,
    lora_a and lora_b only (R and the stabilizer are frozen), each in its input's dtype."""

    @staticmethod
    def forward(ctx, x, lora_a, lora_b, weights: LinearWeights, ws: Workspace):
        if lora_a.shape != weights.lora_a.shape or lora_b.shape != weights.lora_b.shape:
            raise ValueError("lora_a / lora_b do not match the layer's adapter shapes")
        w = dataclasses.replace(weights, lora_a=lora_a.detach().to(torch.bfloat16).contiguous(),
                                lora_b=lora_b.detach().to(torch.bfloat16).contiguous())
        x = x.contiguous()
        y, t = linear_fwd(w, x, ws)
        ctx.save_for_backward(x, t)
        ctx.weights, ctx.ws = w, ws
        ctx.dtypes = (lora_a.dtype, lora_b.dtype)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, t = ctx.saved_tensors
        dx, da, db = linear_bwd(ctx.weights, x, t, dy.to(torch.bfloat16).contiguous(), ctx.ws)
        return dx, da.to(ctx.dtypes[0]), db.to(ctx.dtypes[1]), None, None
