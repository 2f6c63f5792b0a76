"""CPU oracle for the NF4 + double-quantization frozen linear layer with LoRA.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library never loads it, and it shares no code, table or constant
generator with the CUDA path.

Two halves:

* ``nf4_oracle.c`` (plain C, built here with gcc, loaded through ctypes) holds
  the codec -- codebook, blockwise absmax encode, double quantization,
  dequantization -- where every float operation must round exactly once, as
  written.
* The linear-algebra definitions of the forward and backward passes are
  written below with numpy float64 matrix products as the library primitive:
  they are exact definitions, so the oracle is the formula itself.

Citations are to the pages on QLoRA (Dettmers et al., arXiv:2305.14314):
automatone "QLoRA paper explained" (sections "How it works", "4-bit NormalFloat
(NF4)", "Double Quantization (DQ)"), creativeworksofknowledge "QLoRA: Fine-Tune
70B on One GPU" (sections "1. NF4", "2. Double quantization", "Code"), aiwiki
"QLoRA" (section "Key Concepts and Technology").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libnf4_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCKSIZE = 64      # weights per absmax block
BLOCKSIZE2 = 256    # absmax constants per double-quantization group


def build(force: bool = False) -> str:
    """Compile nf4_oracle.c with gcc (no FP contraction, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden", _SRC,
           "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64 = ctypes.c_int64
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.nf4o_bf16_to_float.argtypes = [ctypes.c_uint16]
        lib.nf4o_bf16_to_float.restype = ctypes.c_float
        lib.nf4o_bf16_rne.argtypes = [ctypes.c_float]
        lib.nf4o_bf16_rne.restype = ctypes.c_uint16
        lib.nf4o_e4m3_to_float.argtypes = [ctypes.c_uint8]
        lib.nf4o_e4m3_to_float.restype = ctypes.c_float
        lib.nf4o_e4m3_rne.argtypes = [ctypes.c_float]
        lib.nf4o_e4m3_rne.restype = ctypes.c_uint8
        lib.nf4o_normal_quantile.argtypes = [ctypes.c_double]
        lib.nf4o_normal_quantile.restype = ctypes.c_double
        lib.nf4o_default_delta.argtypes = []
        lib.nf4o_default_delta.restype = ctypes.c_double
        lib.nf4o_codebook.argtypes = [ctypes.c_double, f32p]
        lib.nf4o_codebook.restype = None
        lib.nf4o_nearest.argtypes = [ctypes.c_float, f32p]
        lib.nf4o_nearest.restype = ctypes.c_int
        lib.nf4o_storage_bytes.argtypes = [i64, ctypes.c_int, ctypes.c_int, i64p, i64p, i64p, i64p]
        lib.nf4o_storage_bytes.restype = None
        lib.nf4o_encode.argtypes = [u16p, i64, ctypes.c_int, f32p, u8p, f32p]
        lib.nf4o_encode.restype = None
        lib.nf4o_mean.argtypes = [f32p, i64]
        lib.nf4o_mean.restype = ctypes.c_float
        lib.nf4o_double_quant.argtypes = [f32p, i64, ctypes.c_int, u8p, f32p, f32p]
        lib.nf4o_double_quant.restype = None
        lib.nf4o_block_constant.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        lib.nf4o_block_constant.restype = ctypes.c_float
        lib.nf4o_dequant.argtypes = [u8p, u8p, f32p, ctypes.c_float, i64, ctypes.c_int,
                                     ctypes.c_int, f32p, u16p]
        lib.nf4o_dequant.restype = None
        lib.nf4o_bf16_rne_n.argtypes = [f32p, i64, u16p]
        lib.nf4o_bf16_rne_n.restype = None
        lib.nf4o_e4m3_rne_n.argtypes = [f32p, i64, u8p]
        lib.nf4o_e4m3_rne_n.restype = None
        lib.nf4o_levels.argtypes = [ctypes.c_int, f32p]
        lib.nf4o_levels.restype = ctypes.c_int
        lib.nf4o_dequant_f32.argtypes = [u8p, f32p, i64, ctypes.c_int, f32p, u16p]
        lib.nf4o_dequant_f32.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ---------------------------------------------------------------------------
# Scalar formats
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32, exactly (bf16 is a float's top half)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_rne(x) -> int:
    """Round one float to bf16 (nearest, ties to even); returns the bit pattern."""
    return int(_load().nf4o_bf16_rne(float(np.float32(x))))


def e4m3_rne(x) -> int:
    """Round one float to OCP E4M3 (nearest, ties to even); returns the byte."""
    return int(_load().nf4o_e4m3_rne(float(np.float32(x))))


def bf16_rne_array(x: np.ndarray) -> np.ndarray:
    """Vector form of bf16_rne: float32 array -> uint16 bit patterns."""
    a = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.zeros(max(a.size, 1), dtype=np.uint16)
    _load().nf4o_bf16_rne_n(_ptr(a, ctypes.c_float), a.size, _ptr(out, ctypes.c_uint16))
    return out[:a.size]


def e4m3_rne_array(x: np.ndarray) -> np.ndarray:
    """Vector form of e4m3_rne: float32 array -> E4M3 bytes."""
    a = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    out = np.zeros(max(a.size, 1), dtype=np.uint8)
    _load().nf4o_e4m3_rne_n(_ptr(a, ctypes.c_float), a.size, _ptr(out, ctypes.c_uint8))
    return out[:a.size]


def e4m3_to_float(b: int) -> float:
    return float(_load().nf4o_e4m3_to_float(int(b)))


# ---------------------------------------------------------------------------
# Codebook (reading R1)
# ---------------------------------------------------------------------------

def default_delta() -> float:
    return float(_load().nf4o_default_delta())


def normal_quantile(p: float) -> float:
    return float(_load().nf4o_normal_quantile(float(p)))


def codebook(delta: float | None = None) -> np.ndarray:
    """The 16 NF4 levels as float32, ascending, L[7] == 0, L[0] == -1, L[15] == 1."""
    lib = _load()
    if delta is None:
        delta = lib.nf4o_default_delta()
    out = np.zeros(16, dtype=np.float32)
    lib.nf4o_codebook(float(delta), _ptr(out, ctypes.c_float))
    return out


# The 4-bit data types (reading R7): NF4, and the two the pages compare it with
# (automatone "QLoRA paper explained", "4-bit NormalFloat (NF4)": evenly spaced
# 4-bit integers, exponent-spaced 4-bit floats).
QUANT_TYPES = {"nf4": 0, "fp4": 1, "int4": 2}


def levels(quant_type: str = "nf4") -> np.ndarray:
    """The 16 levels of a 4-bit data type as float32, ascending, in [-1, 1]:
    NF4 (the codebook above), INT4 ((2i - 15) / 15) or FP4 (the 15 distinct
    E2M1 values / 6, then +1 repeated; code 15 is never chosen)."""
    out = np.zeros(16, dtype=np.float32)
    if _load().nf4o_levels(QUANT_TYPES[quant_type], _ptr(out, ctypes.c_float)) != 0:
        raise ValueError(quant_type)
    return out


def nearest(n: float, L: np.ndarray | None = None) -> int:
    if L is None:
        L = codebook()
    L = np.ascontiguousarray(L, dtype=np.float32)
    return int(_load().nf4o_nearest(float(np.float32(n)), _ptr(L, ctypes.c_float)))


# ---------------------------------------------------------------------------
# Storage
# ---------------------------------------------------------------------------

def storage_bytes(numel: int, bs: int = BLOCKSIZE, bs2: int = BLOCKSIZE2) -> dict:
    """Bytes of each buffer of a quantized tensor with `numel` weights.  With
    bs2 = 0 (no double quantization) 'absmax_q' is the fp32 absmax array and
    there is no c2 or mean."""
    out = [ctypes.c_int64() for _ in range(4)]
    _load().nf4o_storage_bytes(int(numel), int(bs), int(bs2), *[ctypes.byref(o) for o in out])
    return dict(codes=out[0].value, absmax_q=out[1].value, absmax_c2=out[2].value,
                mean=out[3].value)


# ---------------------------------------------------------------------------
# Encode / double-quant / dequant
# ---------------------------------------------------------------------------

def encode(w_bits: np.ndarray, bs: int = BLOCKSIZE, L: np.ndarray | None = None):
    """Blockwise absmax NF4 encode of bf16 weights (given as uint16 bit patterns).

    Returns (packed codes uint8 [(numel+1)//2], c1 float32 [ceil(numel/bs)]).
    """
    if L is None:
        L = codebook()
    w = np.ascontiguousarray(w_bits, dtype=np.uint16).reshape(-1)
    numel = w.size
    nblocks = (numel + bs - 1) // bs
    packed = np.zeros((numel + 1) // 2, dtype=np.uint8)
    c1 = np.zeros(max(nblocks, 1), dtype=np.float32)
    Lc = np.ascontiguousarray(L, dtype=np.float32)
    if numel:
        _load().nf4o_encode(_ptr(w, ctypes.c_uint16), numel, bs, _ptr(Lc, ctypes.c_float),
                            _ptr(packed, ctypes.c_uint8), _ptr(c1, ctypes.c_float))
    return packed, c1[:nblocks]


def block_mean(c1: np.ndarray) -> np.float32:
    c = np.ascontiguousarray(c1, dtype=np.float32)
    return np.float32(_load().nf4o_mean(_ptr(c, ctypes.c_float), c.size))


def double_quant_fn(c1: np.ndarray, bs2: int = BLOCKSIZE2):
    """Returns (q uint8 [nblocks] E4M3 codes, c2 float32 [ngroups], mean float32)."""
    c = np.ascontiguousarray(c1, dtype=np.float32)
    nb = c.size
    ng = (nb + bs2 - 1) // bs2
    q = np.zeros(max(nb, 1), dtype=np.uint8)
    c2 = np.zeros(max(ng, 1), dtype=np.float32)
    mu = np.zeros(1, dtype=np.float32)
    if nb:
        _load().nf4o_double_quant(_ptr(c, ctypes.c_float), nb, bs2, _ptr(q, ctypes.c_uint8),
                                  _ptr(c2, ctypes.c_float), _ptr(mu, ctypes.c_float))
    return q[:nb], c2[:ng], mu[0]


double_quant = double_quant_fn


def block_constant(q: int, c2: float, mu: float) -> np.float32:
    return np.float32(_load().nf4o_block_constant(int(q), float(np.float32(c2)),
                                                  float(np.float32(mu))))


def dequant(packed, q, c2, mu, numel: int, bs: int = BLOCKSIZE, bs2: int = BLOCKSIZE2,
            L: np.ndarray | None = None) -> np.ndarray:
    """Two-level dequantization to bf16; returns uint16 bit patterns [numel]."""
    if L is None:
        L = codebook()
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    qq = np.ascontiguousarray(q, dtype=np.uint8)
    cc = np.ascontiguousarray(c2, dtype=np.float32)
    Lc = np.ascontiguousarray(L, dtype=np.float32)
    out = np.zeros(max(int(numel), 1), dtype=np.uint16)
    if numel:
        _load().nf4o_dequant(_ptr(p, ctypes.c_uint8), _ptr(qq, ctypes.c_uint8),
                             _ptr(cc, ctypes.c_float), float(np.float32(mu)), int(numel), bs, bs2,
                             _ptr(Lc, ctypes.c_float), _ptr(out, ctypes.c_uint16))
    return out[:numel]


def dequant_f32(packed, c1, numel: int, bs: int = BLOCKSIZE, L: np.ndarray | None = None) -> np.ndarray:
    """Dequantization without double quantization: w' = bf16_RNE(L[code] * c1)
    with the block's fp32 absmax c1; returns uint16 bit patterns [numel]."""
    if L is None:
        L = codebook()
    p = np.ascontiguousarray(packed, dtype=np.uint8)
    cc = np.ascontiguousarray(c1, dtype=np.float32)
    Lc = np.ascontiguousarray(L, dtype=np.float32)
    out = np.zeros(max(int(numel), 1), dtype=np.uint16)
    if numel:
        _load().nf4o_dequant_f32(_ptr(p, ctypes.c_uint8), _ptr(cc, ctypes.c_float), int(numel), bs,
                                 _ptr(Lc, ctypes.c_float), _ptr(out, ctypes.c_uint16))
    return out[:numel]


def quantize(w_bits: np.ndarray, bs: int = BLOCKSIZE, bs2: int = BLOCKSIZE2, quant_type: str = "nf4",
             double_quant: bool = True) -> dict:
    """Encode (with the levels of `quant_type`), then double-quantize the block
    constants -- or, with double_quant=False, keep them as fp32 (the variant
    without double quantization).  The full stored form of one weight tensor."""
    L = levels(quant_type)
    packed, c1 = encode(w_bits, bs, L)
    qt = dict(codes=packed, c1=c1, quant_type=quant_type, double_quant=double_quant, levels=L,
              numel=int(np.asarray(w_bits).size), shape=tuple(np.asarray(w_bits).shape))
    if double_quant:
        q, c2, mu = double_quant_fn(c1, bs2)
        qt.update(absmax_q=q, absmax_c2=c2, mean=mu)
    else:
        qt.update(absmax=c1.copy())
    return qt


def dequant_tensor(qt: dict, bs: int = BLOCKSIZE, bs2: int = BLOCKSIZE2) -> np.ndarray:
    """deq(W) as float32 values (bf16-exact), reshaped like the original weight."""
    bits = dequant_bits(qt, bs, bs2)
    return bf16_bits_to_f32(bits).reshape(qt["shape"])


def dequant_bits(qt: dict, bs: int = BLOCKSIZE, bs2: int = BLOCKSIZE2) -> np.ndarray:
    """deq(W) as bf16 bit patterns [numel], for either stored form."""
    L = qt.get("levels")
    if L is None:
        L = codebook()
    if qt.get("double_quant", True):
        return dequant(qt["codes"], qt["absmax_q"], qt["absmax_c2"], qt["mean"], qt["numel"], bs, bs2, L)
    return dequant_f32(qt["codes"], qt["absmax"], qt["numel"], bs, L)


# ---------------------------------------------------------------------------
# LoRA linear forward / backward: the formulas themselves, in float64.
# Y = X W'^T + s (X A^T) B^T;  G = dY B;  dX = dY W' + s G A;
# dB = s dY^T (X A^T);  dA = s G^T X.  (W frozen: no dW; no bias; no dropout.)
# ---------------------------------------------------------------------------

def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def linear_fwd(Wd, X, A, B, s: float):
    """Returns (Y, XA) in float64.  Wd [N,K], X [M,K], A [r,K], B [N,r]."""
    Wd, X, A, B = _f64(Wd), _f64(X), _f64(A), _f64(B)
    XA = X @ A.T
    Y = X @ Wd.T + s * (XA @ B.T)
    return Y, XA


def linear_bwd(Wd, X, dY, A, B, s: float):
    """Returns (dX, dA, dB) in float64."""
    Wd, X, dY, A, B = _f64(Wd), _f64(X), _f64(dY), _f64(A), _f64(B)
    XA = X @ A.T
    G = dY @ B
    dX = dY @ Wd + s * (G @ A)
    dB = s * (dY.T @ XA)
    dA = s * (G.T @ X)
    return dX, dA, dB


def lora_grads(X, dY, A, B, s: float):
    """The LoRA branch's own quantities, in float64 (they do not involve W):
    XA = X A^T [M, r], G = dY B [M, r], dA = s G^T X [r, K], dB = s dY^T XA [N, r].
    Same formulas as linear_fwd / linear_bwd (automatone "QLoRA paper explained",
    "How it works": the gradients land only on the LoRA adapters)."""
    X, dY, A, B = _f64(X), _f64(dY), _f64(A), _f64(B)
    XA = X @ A.T
    G = dY @ B
    dA = s * (G.T @ X)
    dB = s * (dY.T @ XA)
    return XA, G, dA, dB


def linear_fwd_multi(Wd, X, A_stack, B_stack, adapter_idx, s: float):
    """Forward with a LoRA adapter per token (batched decode of several adapters
    over one frozen weight; automatone "QLoRA paper explained", "Results": the
    4-bit base is also what gets deployed).  Token t uses adapter
    a = adapter_idx[t]:  Y[t] = X[t] W'^T + s (X[t] A_a^T) B_a^T  and
    XA[t] = X[t] A_a^T; a token whose index is negative (or not in the stack)
    gets no LoRA term and XA[t] = 0.  A_stack [n, r, K], B_stack [n, N, r].
    Returns (Y, XA) in float64."""
    Wd, X = _f64(Wd), _f64(X)
    A_stack, B_stack = _f64(A_stack), _f64(B_stack)
    n_ad, r = A_stack.shape[0], A_stack.shape[1]
    Y = X @ Wd.T
    XA = np.zeros((X.shape[0], r))
    for t, a in enumerate(np.asarray(adapter_idx).reshape(-1)):
        if 0 <= a < n_ad:
            XA[t] = X[t] @ A_stack[a].T
            Y[t] += s * (XA[t] @ B_stack[a].T)
    return Y, XA


def linear_fwd_rows(Wd, X, A, B, s: float, rows):
    """Forward restricted to selected token rows (exactly the same formula)."""
    return linear_fwd(Wd, np.asarray(X)[rows], A, B, s)[0]


def linear_bwd_dx_rows(Wd, dY, A, B, s: float, rows):
    """dX restricted to selected token rows (dX row m depends only on dY row m)."""
    Wd, dYr, A, B = _f64(Wd), _f64(np.asarray(dY)[rows]), _f64(A), _f64(B)
    return dYr @ Wd + s * ((dYr @ B) @ A)
