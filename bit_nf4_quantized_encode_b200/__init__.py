"""Python binding of libqlora: NF4 + double-quant frozen linear layer with LoRA on B200.

A thin ctypes layer over the C ABI in ``include/qlora.h``.  It only marshals
arguments -- device pointers of torch tensors, sizes, the current CUDA stream --
and allocates the output tensors and work buffers with torch.  Every step of the
computation runs in the library's sm_100a kernels; there is no CPU fallback:
if ``libqlora.so`` is missing or fails to load, importing this module raises.

Entry points (same names as the C ABI):
    qlora_quantize_nf4_dq(W)                          -> NF4Tensor
    qlora_dequantize(qt)                              -> bf16 [rows, cols]
    qlora_linear_fwd(qt, X, A, B, s, save_xa=True)    -> (Y bf16, XA fp32 or None)
    qlora_linear_bwd(qt, X, dY, A, B, s, XA=None, need_dx=True) -> (dX bf16 or None, dA fp32, dB fp32)
    qlora_get_codebook()                              -> 16 float levels
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

BLOCKSIZE = 64
BLOCKSIZE2 = 256

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libqlora.so not built at {LIB_PATH}; run "
                      "`python bit_nf4_quantized_encode_b200/build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)


class _Nf4TensorC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p),
                ("absmax_c2", ctypes.c_void_p), ("absmax_mean", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("blocksize", ctypes.c_int32), ("blocksize2", ctypes.c_int32)]


_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_szp = ctypes.POINTER(ctypes.c_size_t)
_T = ctypes.POINTER(_Nf4TensorC)

_lib.qlora_status_string.argtypes = [ctypes.c_int]
_lib.qlora_status_string.restype = ctypes.c_char_p
_lib.qlora_get_codebook.argtypes = [ctypes.POINTER(ctypes.c_float)]
_lib.qlora_get_codebook.restype = None
_lib.qlora_nf4_sizes.argtypes = [_i64, _i64, _i32, _i32, _szp, _szp, _szp, _szp]
_lib.qlora_nf4_sizes.restype = ctypes.c_int
_lib.qlora_quantize_nf4_dq.argtypes = [_vp, _T, _vp, _sz, _vp]
_lib.qlora_quantize_nf4_dq.restype = ctypes.c_int
_lib.qlora_dequantize.argtypes = [_T, _vp, _vp]
_lib.qlora_dequantize.restype = ctypes.c_int
_lib.qlora_linear_workspace_size.argtypes = [_i64, _i64, _i64, _i32, _szp, _szp]
_lib.qlora_linear_workspace_size.restype = ctypes.c_int
_lib.qlora_linear_fwd.argtypes = [_T, _vp, _i64, _vp, _vp, _i32, ctypes.c_float, _vp, _vp, _vp,
                                  _sz, _vp]
_lib.qlora_linear_fwd.restype = ctypes.c_int
_lib.qlora_linear_bwd.argtypes = [_T, _vp, _vp, _i64, _vp, _vp, _i32, ctypes.c_float, _vp, _vp,
                                  _vp, _vp, _vp, _sz, _vp]
_lib.qlora_linear_bwd.restype = ctypes.c_int
_lib.qlora_read_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
_lib.qlora_read_device_errors.restype = ctypes.c_int
_lib.qlora_quantize_nf4_dq_noalloc.argtypes = [_vp, _T, _vp]
_lib.qlora_quantize_nf4_dq_noalloc.restype = ctypes.c_int
_lib.qlora_kernel_launches.argtypes = []
_lib.qlora_kernel_launches.restype = ctypes.c_uint64
_lib.qlora_time_next_gemm.argtypes = [_vp, _vp]
_lib.qlora_time_next_gemm.restype = ctypes.c_int
_lib.qlora_selftest_bounded_wait.argtypes = [_i64, _vp, _vp]
_lib.qlora_selftest_bounded_wait.restype = ctypes.c_int

EXPORTED = ["qlora_status_string", "qlora_get_codebook", "qlora_nf4_sizes", "qlora_quantize_nf4_dq",
            "qlora_dequantize", "qlora_linear_workspace_size", "qlora_linear_fwd",
            "qlora_linear_bwd", "qlora_read_device_errors", "qlora_kernel_launches",
            "qlora_time_next_gemm", "qlora_quantize_nf4_dq_noalloc", "qlora_selftest_bounded_wait"]

# Largest weight the allocation-free quantize variant accepts.
NOALLOC_MAX_ELEMENTS = 134217728


class QloraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.qlora_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


def _check(status: int, where: str):
    if status != 0:
        raise QloraError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_bf16_cuda(name: str, t: torch.Tensor):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


@dataclass
class NF4Tensor:
    """A quantized weight: packed codes, E4M3 block constants, c2 per group, mean."""
    codes: torch.Tensor        # uint8 [ceil(rows*cols/2)]
    absmax_q: torch.Tensor     # uint8 [ceil(rows*cols/64)]
    absmax_c2: torch.Tensor    # float32 [ceil(nblocks/256)]
    absmax_mean: torch.Tensor  # float32 [1]
    rows: int
    cols: int

    def c_struct(self) -> _Nf4TensorC:
        return _Nf4TensorC(self.codes.data_ptr(), self.absmax_q.data_ptr(),
                           self.absmax_c2.data_ptr(), self.absmax_mean.data_ptr(),
                           self.rows, self.cols, BLOCKSIZE, BLOCKSIZE2)

    @property
    def device(self):
        return self.codes.device

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.codes, self.absmax_q, self.absmax_c2, self.absmax_mean))


def qlora_status_string(status: int) -> str:
    return _lib.qlora_status_string(int(status)).decode()


def qlora_get_codebook() -> list:
    out = (ctypes.c_float * 16)()
    _lib.qlora_get_codebook(out)
    return list(out)


def qlora_nf4_sizes(rows: int, cols: int) -> dict:
    v = [ctypes.c_size_t() for _ in range(4)]
    _check(_lib.qlora_nf4_sizes(rows, cols, BLOCKSIZE, BLOCKSIZE2, *[ctypes.byref(x) for x in v]),
           "qlora_nf4_sizes")
    return dict(codes=v[0].value, absmax_q=v[1].value, absmax_c2=v[2].value, workspace=v[3].value)


def empty_nf4(rows: int, cols: int, device) -> NF4Tensor:
    sz = qlora_nf4_sizes(rows, cols)
    # round each buffer up to 16 bytes so every pointer the library sees is aligned
    def buf(n, dtype, esize):
        return torch.empty(max(1, (n + 15) // 16 * 16 // esize), dtype=dtype, device=device)
    return NF4Tensor(codes=buf(sz["codes"], torch.uint8, 1), absmax_q=buf(sz["absmax_q"], torch.uint8, 1),
                     absmax_c2=buf(sz["absmax_c2"], torch.float32, 4),
                     absmax_mean=torch.empty(4, dtype=torch.float32, device=device),
                     rows=rows, cols=cols)


def _check_out_matches(W: torch.Tensor, out: NF4Tensor):
    """The C entry points take the shape from `out` alone and read that many
    weights from W: refuse a destination that describes another tensor."""
    if out.rows * out.cols != W.numel():
        raise ValueError(f"out describes {out.rows}x{out.cols} weights, W has {W.numel()}")
    for name, t in (("codes", out.codes), ("absmax_q", out.absmax_q), ("absmax_c2", out.absmax_c2),
                    ("absmax_mean", out.absmax_mean)):
        if t.device != W.device:
            raise ValueError(f"out.{name} is on {t.device}, W on {W.device}")


def qlora_quantize_nf4_dq(W: torch.Tensor, out: NF4Tensor | None = None,
                          workspace: torch.Tensor | None = None) -> NF4Tensor:
    """Blockwise NF4 encode + double quantization of a bf16 [rows, cols] weight."""
    _need_bf16_cuda("W", W)
    rows, cols = (W.shape[0], W.shape[1]) if W.dim() == 2 else (1, W.numel())
    if out is None:
        out = empty_nf4(rows, cols, W.device)
    _check_out_matches(W, out)
    need = qlora_nf4_sizes(rows, cols)["workspace"]
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    c = out.c_struct()
    _check(_lib.qlora_quantize_nf4_dq(_ptr(W), ctypes.byref(c), _ptr(workspace),
                                      workspace.numel(), _stream(W.device)), "qlora_quantize_nf4_dq")
    return out


def qlora_quantize_nf4_dq_noalloc(W: torch.Tensor, out: NF4Tensor) -> NF4Tensor:
    """Same result as qlora_quantize_nf4_dq, with the library's built-in scratch
    instead of a work buffer (for callers that cannot allocate; see qlora.h)."""
    _need_bf16_cuda("W", W)
    _check_out_matches(W, out)
    c = out.c_struct()
    _check(_lib.qlora_quantize_nf4_dq_noalloc(_ptr(W), ctypes.byref(c), _stream(W.device)),
           "qlora_quantize_nf4_dq_noalloc")
    return out


def qlora_dequantize(qt: NF4Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """Two-level dequantization to a bf16 [rows, cols] tensor."""
    if out is None:
        out = torch.empty(qt.rows, qt.cols, dtype=torch.bfloat16, device=qt.device)
    c = qt.c_struct()
    _check(_lib.qlora_dequantize(ctypes.byref(c), _ptr(out), _stream(qt.device)), "qlora_dequantize")
    return out


def qlora_linear_workspace_size(rows: int, cols: int, m: int, r: int) -> tuple:
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib.qlora_linear_workspace_size(rows, cols, m, r, ctypes.byref(f), ctypes.byref(b)),
           "qlora_linear_workspace_size")
    return f.value, b.value


def qlora_linear_fwd(qt: NF4Tensor, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                     save_xa: bool = True, Y: torch.Tensor | None = None,
                     XA: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Y = X deq(W)^T + s (X A^T) B^T.  Returns (Y bf16, XA) with XA = X A^T in fp32 (or None)."""
    for n, t in (("X", X), ("A", A), ("B", B)):
        _need_bf16_cuda(n, t)
    m, r = X.shape[0], A.shape[0]
    if Y is None:
        Y = torch.empty(m, qt.rows, dtype=torch.bfloat16, device=X.device)
    if save_xa and XA is None:
        XA = torch.empty(m, r, dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(qlora_linear_workspace_size(qt.rows, qt.cols, m, r)[0],
                                dtype=torch.uint8, device=X.device)
    c = qt.c_struct()
    _check(_lib.qlora_linear_fwd(ctypes.byref(c), _ptr(X), m, _ptr(A), _ptr(B), r, float(s), _ptr(Y),
                                 _ptr(XA if save_xa else None), _ptr(workspace), workspace.numel(),
                                 _stream(X.device)), "qlora_linear_fwd")
    return Y, (XA if save_xa else None)


def qlora_linear_bwd(qt: NF4Tensor, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor,
                     B: torch.Tensor, s: float, XA: torch.Tensor | None = None, need_dx: bool = True,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                     dB: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Returns (dX bf16 or None, dA fp32, dB fp32) of the frozen-NF4 LoRA linear layer."""
    for n, t in (("X", X), ("dY", dY), ("A", A), ("B", B)):
        _need_bf16_cuda(n, t)
    m, r = X.shape[0], A.shape[0]
    dev = X.device
    if need_dx and dX is None:
        dX = torch.empty(m, qt.cols, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(r, qt.cols, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(qt.rows, r, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(qlora_linear_workspace_size(qt.rows, qt.cols, m, r)[1],
                                dtype=torch.uint8, device=dev)
    c = qt.c_struct()
    _check(_lib.qlora_linear_bwd(ctypes.byref(c), _ptr(X), _ptr(dY), m, _ptr(A), _ptr(B), r,
                                 float(s), _ptr(XA), _ptr(dX if need_dx else None), _ptr(dA),
                                 _ptr(dB), _ptr(workspace), workspace.numel(), _stream(dev)),
           "qlora_linear_bwd")
    return (dX if need_dx else None), dA, dB


def qlora_read_device_errors(clear: bool = True) -> int:
    """Error flags set by kernels whose internal waits timed out (0 = none)."""
    v = ctypes.c_uint32()
    _check(_lib.qlora_read_device_errors(ctypes.byref(v), 1 if clear else 0),
           "qlora_read_device_errors")
    return v.value


def qlora_selftest_bounded_wait(limit_cycles: int, outcome: torch.Tensor | None = None) -> None:
    """Launch the failure-path self-test: one CTA whose bounded mbarrier wait
    must give up after `limit_cycles` SM cycles (see qlora.h)."""
    _check(_lib.qlora_selftest_bounded_wait(int(limit_cycles), _ptr(outcome),
                                            _stream(outcome.device if outcome is not None else None)),
           "qlora_selftest_bounded_wait")


def qlora_kernel_launches() -> int:
    """Kernels launched by the library in this process so far."""
    return int(_lib.qlora_kernel_launches())


def qlora_time_next_gemm(start: torch.cuda.Event, stop: torch.cuda.Event) -> None:
    """Bracket the calling thread's next fused dequant-GEMM launch with two CUDA events."""
    _check(_lib.qlora_time_next_gemm(ctypes.c_void_p(start.cuda_event), ctypes.c_void_p(stop.cuda_event)),
           "qlora_time_next_gemm")
