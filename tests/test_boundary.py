"""The C-ABI boundary on CPU: the library loads, exports every declared entry
point, its host-side tables agree with the oracle, and argument validation
rejects bad calls before anything reaches a GPU.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")

qb = pytest.importorskip("bit_nf4_quantized_encode_b200")
lib = qb._lib

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUP, ERR_CUDA, ERR_WS = 0, -1, -2, -3, -4, -5, -6


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"QLORA_EXPORT[^;(]*?\b(qlora_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), f"{n} declared in qlora.h but not exported"
    assert set(names) == set(qb.EXPORTED)


def test_codebook_matches_oracle_bit_for_bit():
    ours = np.array(qb.qlora_get_codebook(), dtype=np.float32)
    ref = oracle.codebook()
    assert ours.view(np.uint32).tolist() == ref.view(np.uint32).tolist()


@pytest.mark.parametrize("rows,cols", [(256, 256), (4096, 4096), (11008, 4096), (3, 100), (1, 1),
                                       (0, 5), (22016, 8192)])
def test_nf4_sizes_match_oracle(rows, cols):
    sz = qb.qlora_nf4_sizes(rows, cols)
    ref = oracle.storage_bytes(rows * cols)
    assert sz["codes"] == ref["codes"]
    assert sz["absmax_q"] == ref["absmax_q"]
    assert sz["absmax_c2"] == ref["absmax_c2"]


def _tensor(rows=64, cols=64, base=0x10000):
    return qb._Nf4TensorC(base, base + 0x1000, base + 0x2000, base + 0x3000, rows, cols, 64, 256)


def test_sizes_reject_bad_block_sizes_and_shapes():
    z = ctypes.c_size_t()
    assert lib.qlora_nf4_sizes(4, 64, 128, 256, None, None, None, ctypes.byref(z)) == ERR_UNSUP
    assert lib.qlora_nf4_sizes(4, 64, 64, 512, None, None, None, None) == ERR_UNSUP
    assert lib.qlora_nf4_sizes(-1, 64, 64, 256, None, None, None, None) == ERR_SHAPE


def test_quantize_validation_before_launch():
    t = _tensor()
    w, ws = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    assert lib.qlora_quantize_nf4_dq(None, ctypes.byref(t), ws, 1 << 20, None) == ERR_NULL
    assert lib.qlora_quantize_nf4_dq(w, None, ws, 1 << 20, None) == ERR_NULL
    assert lib.qlora_quantize_nf4_dq(ctypes.c_void_p(0x20008), ctypes.byref(t), ws, 1 << 20, None) == ERR_ALIGN
    assert lib.qlora_quantize_nf4_dq(w, ctypes.byref(t), ws, 8, None) == ERR_WS
    bad = _tensor()
    bad.blocksize = 32
    assert lib.qlora_quantize_nf4_dq(w, ctypes.byref(bad), ws, 1 << 20, None) == ERR_UNSUP
    mis = _tensor()
    mis.absmax_c2 = mis.absmax_c2 + 4
    assert lib.qlora_quantize_nf4_dq(w, ctypes.byref(mis), ws, 1 << 20, None) == ERR_ALIGN
    nul = _tensor()
    nul.codes = None
    assert lib.qlora_quantize_nf4_dq(w, ctypes.byref(nul), ws, 1 << 20, None) == ERR_NULL
    empty = _tensor(rows=0)
    assert lib.qlora_quantize_nf4_dq(None, ctypes.byref(empty), None, 0, None) == OK   # no-op


def test_dequantize_validation_before_launch():
    t = _tensor()
    assert lib.qlora_dequantize(ctypes.byref(t), None, None) == ERR_NULL
    assert lib.qlora_dequantize(ctypes.byref(t), ctypes.c_void_p(0x20002), None) == ERR_ALIGN


def test_workspace_sizes():
    f, b = qb.qlora_linear_workspace_size(4096, 4096, 8192, 64)
    assert f >= 8192 * 64 * 6 and b >= (4096 + 4096) * 64 * 4
    # decode shapes (M <= 16): per-warp tile counters, partial slots of at most
    # 256 CTAs x 2 x 8 warps x 32 lanes x 16 fp32, and 16 K-slices of X A^T
    f16, b16 = qb.qlora_linear_workspace_size(22016, 8192, 16, 64)
    tiles, steps = (22016 + 255) // 256, 8192 // 256
    slots = min(tiles * steps, 256) * 2 * 8 * 32 * 16 * 4
    assert f16 >= tiles * 8 * 4 + slots + 16 * 16 * 64 * 4
    # a one-unit weight needs the slots of one CTA only
    f_tiny, _ = qb.qlora_linear_workspace_size(256, 256, 16, 8)
    assert 2 * 8 * 32 * 16 * 4 <= f_tiny < 2 * 2 * 8 * 32 * 16 * 4 + 16 * 16 * 64 * 4 + 1024
    with pytest.raises(qb.QloraError):
        qb.qlora_linear_workspace_size(4096, 100, 16, 64)     # cols % 64 != 0
    with pytest.raises(qb.QloraError):
        qb.qlora_linear_workspace_size(4096, 4096, 16, 12)    # r % 8 != 0


@pytest.mark.parametrize("rows,cols,m,r,expect", [
    (4096, 4096, 0, 64, ERR_SHAPE),       # no tokens
    (4096, 4100, 16, 64, ERR_SHAPE),      # cols not a multiple of 64 (tensor shape)
    (4100, 4096, 16, 64, ERR_SHAPE),      # rows not a multiple of 8
    (4096, 4096, 16, 4, ERR_SHAPE),       # rank below 8
    (4096, 4096, 16, 264, ERR_SHAPE),     # rank above 256
])
def test_linear_shape_validation(rows, cols, m, r, expect):
    t = _tensor(rows, cols)
    p = ctypes.c_void_p(0x40000)
    st = lib.qlora_linear_fwd(ctypes.byref(t), p, m, p, p, r, ctypes.c_float(0.25), p, None, p,
                              1 << 40, None)
    assert st == expect
    st = lib.qlora_linear_bwd(ctypes.byref(t), p, p, m, p, p, r, ctypes.c_float(0.25), None, p, p, p,
                              p, 1 << 40, None)
    assert st == expect


def test_linear_pointer_validation():
    t = _tensor(256, 256)
    p = ctypes.c_void_p(0x40000)
    odd = ctypes.c_void_p(0x40002)
    s = ctypes.c_float(2.0)
    assert lib.qlora_linear_fwd(ctypes.byref(t), None, 16, p, p, 8, s, p, None, p, 1 << 40, None) == ERR_NULL
    assert lib.qlora_linear_fwd(ctypes.byref(t), odd, 16, p, p, 8, s, p, None, p, 1 << 40, None) == ERR_ALIGN
    assert lib.qlora_linear_fwd(ctypes.byref(t), p, 16, p, p, 8, s, p, odd, p, 1 << 40, None) == ERR_ALIGN
    assert lib.qlora_linear_fwd(ctypes.byref(t), p, 16, p, p, 8, s, p, None, p, 16, None) == ERR_WS
    assert lib.qlora_linear_fwd(ctypes.byref(t), p, 16, p, p, 8, ctypes.c_float(float("nan")), p, None,
                                p, 1 << 40, None) == ERR_SHAPE
    assert lib.qlora_linear_bwd(ctypes.byref(t), p, p, 16, p, p, 8, s, None, None, None, p, p,
                                1 << 40, None) == ERR_NULL          # dA is required
    assert lib.qlora_linear_bwd(ctypes.byref(t), p, p, 16, p, p, 8, s, odd, None, p, p, p,
                                1 << 40, None) == ERR_ALIGN
    assert lib.qlora_linear_bwd(ctypes.byref(t), p, p, 16, p, p, 8, s, None, None, p, p, p,
                                64, None) == ERR_WS


def test_status_strings():
    for st in (OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUP, ERR_CUDA, ERR_WS, 12345):
        assert isinstance(qb.qlora_status_string(st), str) and qb.qlora_status_string(st)


def test_noalloc_validates_like_the_workspace_entry_point():
    """The allocation-free quantize runs the same descriptor checks in the same
    order as qlora_quantize_nf4_dq, so a bad call gets the same status from
    both; only its size limit replaces the work-buffer check."""
    w, ws = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    huge_cols = _tensor(rows=0, cols=(1 << 31) + 64)          # empty, but cols out of range
    bad_bs = _tensor()
    bad_bs.blocksize2 = 128
    mis = _tensor()
    mis.absmax_mean = mis.absmax_mean + 8
    nul = _tensor()
    nul.absmax_q = None
    cases = [(w, huge_cols, ERR_SHAPE), (w, bad_bs, ERR_UNSUP), (w, mis, ERR_ALIGN), (w, nul, ERR_NULL),
             (None, _tensor(), ERR_NULL), (ctypes.c_void_p(0x20004), _tensor(), ERR_ALIGN)]
    for wp, t, expect in cases:
        a = lib.qlora_quantize_nf4_dq(wp, ctypes.byref(t), ws, 1 << 40, None)
        b = lib.qlora_quantize_nf4_dq_noalloc(wp, ctypes.byref(t), None)
        assert a == b == expect, (a, b, expect)
    assert lib.qlora_quantize_nf4_dq_noalloc(w, None, None) == ERR_NULL
    big = _tensor(rows=2, cols=qb.NOALLOC_MAX_ELEMENTS // 2 + 64)
    assert lib.qlora_quantize_nf4_dq_noalloc(w, ctypes.byref(big), None) == ERR_WS


def test_python_wrapper_refuses_a_destination_of_another_shape():
    """The C entry points read out.rows * out.cols weights from W; the binding
    refuses a destination that describes more (or fewer) weights than W holds,
    or that lives on another device, before calling the library."""
    import torch
    w = torch.zeros(64, 128, dtype=torch.bfloat16)
    cpu = torch.device("cpu")
    good = qb.NF4Tensor(codes=torch.zeros(4096, dtype=torch.uint8), absmax_q=torch.zeros(128, dtype=torch.uint8),
                        absmax_c2=torch.zeros(4), absmax_mean=torch.zeros(4), rows=64, cols=128)
    qb._check_out_matches(w, good)
    bigger = qb.NF4Tensor(codes=good.codes, absmax_q=good.absmax_q, absmax_c2=good.absmax_c2,
                          absmax_mean=good.absmax_mean, rows=128, cols=128)
    with pytest.raises(ValueError, match="describes"):
        qb._check_out_matches(w, bigger)
    meta = qb.NF4Tensor(codes=torch.empty(4096, dtype=torch.uint8, device="meta"), absmax_q=good.absmax_q,
                        absmax_c2=good.absmax_c2, absmax_mean=good.absmax_mean, rows=64, cols=128)
    assert meta.codes.device != cpu
    with pytest.raises(ValueError, match="codes"):
        qb._check_out_matches(w, meta)


def test_selftest_rejects_limits_out_of_range():
    assert lib.qlora_selftest_bounded_wait(-1, None, None) == ERR_SHAPE
    assert lib.qlora_selftest_bounded_wait(100000001, None, None) == ERR_SHAPE
    assert lib.qlora_selftest_bounded_wait(1000, ctypes.c_void_p(0x40002), None) == ERR_ALIGN


@pytest.mark.parametrize("quant_type", ["nf4", "fp4", "int4"])
def test_levels_match_oracle_bit_for_bit(quant_type):
    """The library builds each 4-bit type's table itself; it must equal the
    oracle's, bit for bit (+0 included)."""
    ours = np.array(qb.qlora_get_levels(quant_type), dtype=np.float32)
    assert ours.view(np.uint32).tolist() == oracle.levels(quant_type).view(np.uint32).tolist()
    out = (ctypes.c_float * 16)()
    assert lib.qlora_get_levels(3, out) == ERR_UNSUP
    assert lib.qlora_get_levels(0, None) == ERR_NULL


@pytest.mark.parametrize("rows,cols", [(4096, 4096), (3, 100), (22016, 8192), (1, 1)])
def test_sizes_without_double_quant_match_oracle(rows, cols):
    sz = qb.qlora_nf4_sizes(rows, cols, double_quant=False)
    ref = oracle.storage_bytes(rows * cols, 64, 0)
    assert (sz["codes"], sz["absmax_q"], sz["absmax_c2"]) == (ref["codes"], ref["absmax_q"], ref["absmax_c2"])
    assert sz["workspace"] >= 8 * 148                  # the encoder's per-CTA partial sums only


def test_variant_descriptor_validation():
    w, ws = ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    bad_type = _tensor()
    bad_type.quant_type = 3
    assert lib.qlora_quantize_nf4_dq(w, ctypes.byref(bad_type), ws, 1 << 40, None) == ERR_UNSUP
    assert lib.qlora_dequantize(ctypes.byref(bad_type), w, None) == ERR_UNSUP
    rsv = _tensor()
    rsv.reserved = 1
    assert lib.qlora_dequantize(ctypes.byref(rsv), w, None) == ERR_UNSUP
    plain = _tensor()
    plain.blocksize2 = 0                        # fp32 constants: `absmax` is required, the rest ignored
    assert lib.qlora_dequantize(ctypes.byref(plain), w, None) == ERR_NULL
    plain.absmax = 0x50008
    assert lib.qlora_dequantize(ctypes.byref(plain), w, None) == ERR_ALIGN
    plain.absmax = 0x50000
    plain.absmax_q = plain.absmax_c2 = plain.absmax_mean = None
    # passes validation; without a GPU it can only fail at the device query
    assert lib.qlora_dequantize(ctypes.byref(plain), w, None) not in (ERR_NULL, ERR_ALIGN, ERR_UNSUP, ERR_SHAPE)
    small_ws = lib.qlora_quantize_nf4_dq(w, ctypes.byref(plain), ws, 8 * 2048 - 8, None)
    assert small_ws == ERR_WS


def test_multi_adapter_validation_before_launch():
    t = _tensor(256, 256)
    p = ctypes.c_void_p(0x40000)
    s = ctypes.c_float(2.0)
    idx = ctypes.c_void_p(0x60000)
    f = lib.qlora_linear_fwd_multi
    assert f(ctypes.byref(t), p, 17, p, p, 2, idx, 8, s, p, None, p, 1 << 40, None) == ERR_SHAPE   # M > 16
    assert f(ctypes.byref(t), p, 4, p, p, 0, idx, 8, s, p, None, p, 1 << 40, None) == ERR_SHAPE    # no adapter
    assert f(ctypes.byref(t), p, 4, p, p, 2, None, 8, s, p, None, p, 1 << 40, None) == ERR_NULL
    assert f(ctypes.byref(t), p, 4, p, p, 2, ctypes.c_void_p(0x60002), 8, s, p, None, p, 1 << 40,
             None) == ERR_ALIGN
    assert f(ctypes.byref(t), p, 4, p, ctypes.c_void_p(0x40008), 2, idx, 8, s, p, None, p, 1 << 40,
             None) == ERR_ALIGN
    assert f(ctypes.byref(t), p, 4, p, p, 2, idx, 8, s, p, None, p, 16, None) == ERR_WS
