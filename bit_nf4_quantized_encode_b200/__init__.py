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
    qlora_linear_fwd_multi(qt, X, A_stack, B_stack, adapter_idx, s) -> (Y, XA): one adapter per token
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
                ("blocksize", ctypes.c_int32), ("blocksize2", ctypes.c_int32),
                ("absmax", ctypes.c_void_p), ("quant_type", ctypes.c_int32), ("reserved", ctypes.c_int32)]


# The 4-bit data types (qlora_quant_type): NF4 and the two it is compared with.
QUANT_TYPES = {"nf4": 0, "fp4": 1, "int4": 2}


_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_szp = ctypes.POINTER(ctypes.c_size_t)
_T = ctypes.POINTER(_Nf4TensorC)

_lib.qlora_status_string.argtypes = [ctypes.c_int]
_lib.qlora_status_string.restype = ctypes.c_char_p
_lib.qlora_get_codebook.argtypes = [ctypes.POINTER(ctypes.c_float)]
_lib.qlora_get_codebook.restype = None
_lib.qlora_get_levels.argtypes = [_i32, ctypes.POINTER(ctypes.c_float)]
_lib.qlora_get_levels.restype = ctypes.c_int
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
_lib.qlora_linear_fwd_multi.argtypes = [_T, _vp, _i64, _vp, _vp, _i32, _vp, _i32, ctypes.c_float, _vp, _vp,
                                        _vp, _sz, _vp]
_lib.qlora_linear_fwd_multi.restype = ctypes.c_int
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

EXPORTED = ["qlora_status_string", "qlora_get_codebook", "qlora_get_levels", "qlora_nf4_sizes", "qlora_quantize_nf4_dq",
            "qlora_dequantize", "qlora_linear_workspace_size", "qlora_linear_fwd", "qlora_linear_fwd_multi",
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
    """A quantized weight: packed 4-bit codes and its block constants, stored
    either double-quantized (E4M3 codes, c2 per group, mean) or as fp32 absmax
    per block (`absmax`, no double quantization)."""
    codes: torch.Tensor                     # uint8 [ceil(rows*cols/2)]
    absmax_q: torch.Tensor | None           # uint8 [ceil(rows*cols/64)] (double quantization)
    absmax_c2: torch.Tensor | None          # float32 [ceil(nblocks/256)] (double quantization)
    absmax_mean: torch.Tensor | None        # float32 [1] (double quantization)
    rows: int
    cols: int
    absmax: torch.Tensor | None = None      # float32 [nblocks] (no double quantization)
    quant_type: str = "nf4"                 # "nf4", "fp4" or "int4"

    @property
    def double_quant(self) -> bool:
        return self.absmax is None

    def c_struct(self) -> _Nf4TensorC:
        p = lambda t: 0 if t is None else t.data_ptr()
        return _Nf4TensorC(self.codes.data_ptr(), p(self.absmax_q), p(self.absmax_c2), p(self.absmax_mean),
                           self.rows, self.cols, BLOCKSIZE, BLOCKSIZE2 if self.double_quant else 0,
                           p(self.absmax), QUANT_TYPES[self.quant_type], 0)

    def buffers(self) -> dict:
        return {n: t for n, t in (("codes", self.codes), ("absmax_q", self.absmax_q),
                                  ("absmax_c2", self.absmax_c2), ("absmax_mean", self.absmax_mean),
                                  ("absmax", self.absmax)) if t is not None}

    @property
    def device(self):
        return self.codes.device

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.buffers().values())


def qlora_status_string(status: int) -> str:
    return _lib.qlora_status_string(int(status)).decode()


def qlora_get_codebook() -> list:
    out = (ctypes.c_float * 16)()
    _lib.qlora_get_codebook(out)
    return list(out)


def qlora_get_levels(quant_type: str = "nf4") -> list:
    """The 16 levels of a 4-bit type ("nf4", "fp4" or "int4")."""
    out = (ctypes.c_float * 16)()
    _check(_lib.qlora_get_levels(QUANT_TYPES[quant_type], out), "qlora_get_levels")
    return list(out)


def qlora_nf4_sizes(rows: int, cols: int, double_quant: bool = True) -> dict:
    """Buffer sizes in bytes; without double quantization 'absmax_q' is the
    size of the fp32 absmax array and 'absmax_c2' is 0."""
    v = [ctypes.c_size_t() for _ in range(4)]
    _check(_lib.qlora_nf4_sizes(rows, cols, BLOCKSIZE, BLOCKSIZE2 if double_quant else 0,
                                *[ctypes.byref(x) for x in v]), "qlora_nf4_sizes")
    return dict(codes=v[0].value, absmax_q=v[1].value, absmax_c2=v[2].value, workspace=v[3].value)


def empty_nf4(rows: int, cols: int, device, quant_type: str = "nf4", double_quant: bool = True) -> NF4Tensor:
    if quant_type not in QUANT_TYPES:
        raise ValueError(f"quant_type must be one of {sorted(QUANT_TYPES)}")
    sz = qlora_nf4_sizes(rows, cols, double_quant)
    # round each buffer up to 16 bytes so every pointer the library sees is aligned
    def buf(n, dtype, esize):
        return torch.empty(max(1, (n + 15) // 16 * 16 // esize), dtype=dtype, device=device)
    codes = buf(sz["codes"], torch.uint8, 1)
    if not double_quant:
        return NF4Tensor(codes=codes, absmax_q=None, absmax_c2=None, absmax_mean=None, rows=rows, cols=cols,
                         absmax=buf(sz["absmax_q"], torch.float32, 4), quant_type=quant_type)
    return NF4Tensor(codes=codes, absmax_q=buf(sz["absmax_q"], torch.uint8, 1),
                     absmax_c2=buf(sz["absmax_c2"], torch.float32, 4),
                     absmax_mean=torch.empty(4, dtype=torch.float32, device=device),
                     rows=rows, cols=cols, quant_type=quant_type)


def _check_out_matches(W: torch.Tensor, out: NF4Tensor):
    """The C entry points take the shape from `out` alone and read that many
    weights from W: refuse a destination that describes another tensor."""
    if out.rows * out.cols != W.numel():
        raise ValueError(f"out describes {out.rows}x{out.cols} weights, W has {W.numel()}")
    for name, t in out.buffers().items():
        if t.device != W.device:
            raise ValueError(f"out.{name} is on {t.device}, W on {W.device}")


def qlora_quantize_nf4_dq(W: torch.Tensor, out: NF4Tensor | None = None,
                          workspace: torch.Tensor | None = None, quant_type: str = "nf4",
                          double_quant: bool = True) -> NF4Tensor:
    """Blockwise 4-bit encode (NF4 by default) + double quantization of a bf16
    [rows, cols] weight; `out`, when given, fixes the type and the form."""
    _need_bf16_cuda("W", W)
    rows, cols = (W.shape[0], W.shape[1]) if W.dim() == 2 else (1, W.numel())
    if out is None:
        out = empty_nf4(rows, cols, W.device, quant_type, double_quant)
    _check_out_matches(W, out)
    need = qlora_nf4_sizes(out.rows, out.cols, out.double_quant)["workspace"]
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


def qlora_linear_fwd_multi(qt: NF4Tensor, X: torch.Tensor, A_stack: torch.Tensor, B_stack: torch.Tensor,
                           adapter_idx: torch.Tensor, s: float, save_xa: bool = True,
                           Y: torch.Tensor | None = None, XA: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None):
    """Decode-shaped forward (M <= 16) with one adapter per token:
    Y[t] = X[t] deq(W)^T + s (X[t] A_a^T) B_a^T with a = adapter_idx[t]
    (int32 on the device; negative = no adapter).  A_stack [n, r, cols] and
    B_stack [n, rows, r] bf16.  Returns (Y bf16, XA fp32 or None)."""
    for n, t in (("X", X), ("A_stack", A_stack), ("B_stack", B_stack)):
        _need_bf16_cuda(n, t)
    if not (adapter_idx.is_cuda and adapter_idx.dtype == torch.int32 and adapter_idx.is_contiguous()
            and adapter_idx.numel() == X.shape[0]):
        raise ValueError("adapter_idx must be a contiguous int32 CUDA tensor with one entry per token")
    if A_stack.dim() != 3 or B_stack.dim() != 3 or A_stack.shape[0] != B_stack.shape[0]:
        raise ValueError("A_stack [n, r, cols] and B_stack [n, rows, r] must hold the same adapters")
    m, n_ad, r = X.shape[0], A_stack.shape[0], A_stack.shape[1]
    if Y is None:
        Y = torch.empty(m, qt.rows, dtype=torch.bfloat16, device=X.device)
    if save_xa and XA is None:
        XA = torch.empty(m, r, dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = torch.empty(qlora_linear_workspace_size(qt.rows, qt.cols, m, r)[0],
                                dtype=torch.uint8, device=X.device)
    c = qt.c_struct()
    _check(_lib.qlora_linear_fwd_multi(ctypes.byref(c), _ptr(X), m, _ptr(A_stack), _ptr(B_stack), n_ad,
                                       _ptr(adapter_idx), r, float(s), _ptr(Y), _ptr(XA if save_xa else None),
                                       _ptr(workspace), workspace.numel(), _stream(X.device)),
           "qlora_linear_fwd_multi")
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
