"""Pins for the oracle's variants: the FP4 and INT4 level tables and the stored
form without double quantization.

Pages: automatone "QLoRA paper explained", paragraph "4-bit NormalFloat (NF4)"
(standard 4-bit integers space their 16 levels evenly, 4-bit floats space them
by exponent, and NF4 beats both on quantization precision; "Results": FP4
trails NF4); creativeworksofknowledge "QLoRA: Fine-Tune 70B on One GPU",
section "2. Double quantization" (constants FP32 -> FP8, about 0.37 bits per
parameter saved).  The FP4 values are pinned against ml_dtypes' E2M1 decode,
the encode against exact-rational brute force, the fp32-constant dequant
against torch's float32 product and bf16 cast, and the storage against the
closed form.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads


def _unpack(packed, numel):
    out = []
    for byte in packed:
        out += [int(byte) >> 4, int(byte) & 15]
    return out[:numel]


def _brute_codes(bits, L, bs=64):
    """Nearest level by exact rationals over all 16 entries; tie -> lower index;
    a block whose absmax is 0 gets code 7."""
    x = oracle.bf16_bits_to_f32(bits)
    Lf = [Fraction(float(v)) for v in L]
    codes = []
    for b0 in range(0, len(x), bs):
        blk = x[b0:b0 + bs]
        c1 = np.max(np.abs(blk))
        for v in blk:
            if c1 == 0:
                codes.append(7)
                continue
            n = Fraction(float(np.float32(v) / np.float32(c1)))
            d = [abs(n - lv) for lv in Lf]
            codes.append(min(range(16), key=lambda i: (d[i], i)))
    return codes


def test_fp4_levels_are_the_e2m1_values():
    """All 16 E2M1 bit patterns decoded by ml_dtypes: 15 distinct values (+0 and
    -0 coincide), divided by the largest, 6; the 16th entry repeats +1."""
    vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    distinct = np.unique(vals)
    assert distinct.size == 15 and distinct.max() == 6.0
    L = oracle.levels("fp4")
    assert np.array_equal(L[:15], (distinct / 6.0).astype(np.float32))
    assert L[15] == L[14] == 1.0 and L[0] == -1.0
    assert L.view(np.uint32)[7] == 0                           # the zero level is +0 (bf16 0x0000 out)
    assert np.all(np.diff(L[:15]) > 0)


def test_int4_levels_are_sixteen_even_steps():
    L = oracle.levels("int4").astype(np.float64)
    assert L[0] == -1.0 and L[15] == 1.0
    steps = np.diff(L)
    assert np.all(steps > 0)
    assert np.max(np.abs(steps - 2.0 / 15.0)) < 2e-7          # one float rounding per level
    assert np.array_equal(L, -L[::-1])                         # symmetric about zero
    assert np.all(L != 0.0)                                    # an even 16-step grid has no zero


@pytest.mark.parametrize("quant_type", ["fp4", "int4"])
def test_variant_encode_matches_brute_force(quant_type):
    L = oracle.levels(quant_type)
    rng = np.random.Generator(np.random.PCG64(21))
    x = rng.standard_normal(6 * 64).astype(np.float32) * np.float32(0.02)
    # values at and next to every decision midpoint, in blocks with absmax 1
    mids = []
    for i in range(15):
        m = np.float32((float(L[i]) + float(L[i + 1])) / 2)
        mids += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    mids = oracle.bf16_bits_to_f32(oracle.bf16_rne_array(np.array(mids, np.float32)))
    blocks = []
    for b0 in range(0, mids.size, 62):
        chunk = list(mids[b0:b0 + 62]) + [1.0, -1.0]
        blocks += chunk + [0.0] * (64 - len(chunk))
    allx = np.concatenate([x, np.array(blocks, np.float32), np.zeros(64, np.float32)])
    bits = oracle.bf16_rne_array(allx)
    qt = oracle.quantize(bits, quant_type=quant_type)
    codes = _unpack(qt["codes"], bits.size)
    assert codes == _brute_codes(bits, L)
    if quant_type == "fp4":
        assert 15 not in codes                                 # the repeated +1 is never chosen


@pytest.mark.parametrize("quant_type", ["nf4", "fp4", "int4"])
def test_no_double_quant_keeps_fp32_absmax_and_dequant_is_one_product(quant_type):
    w = workloads.weight((96, 320), proj=2)
    bits = workloads.bf16_bits(w)
    qt = oracle.quantize(bits, quant_type=quant_type, double_quant=False)
    x = oracle.bf16_bits_to_f32(bits).reshape(-1, 64)
    assert np.array_equal(qt["absmax"], np.max(np.abs(x), axis=1))
    assert "absmax_q" not in qt
    codes = np.array(_unpack(qt["codes"], bits.size))
    L = torch.from_numpy(oracle.levels(quant_type))
    prod = L[torch.from_numpy(codes)] * torch.from_numpy(np.repeat(qt["absmax"], 64))   # float32 product
    want = prod.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.dequant_bits(qt), want)
    # the codes do not depend on how the constants are stored
    assert np.array_equal(oracle.quantize(bits, quant_type=quant_type)["codes"], qt["codes"])


@pytest.mark.parametrize("shape", [(4096, 4096), (22016, 8192), (256, 256)])
def test_storage_without_double_quant_is_half_a_bit(shape):
    """fp32 constants per 64 weights cost 32/64 = 0.5 bits per parameter;
    double quantization brings that to 8/64 + 32/(64*256) (+ one mean): the
    saving of about 0.37 bits the pages report."""
    nk = shape[0] * shape[1]
    plain = oracle.storage_bytes(nk, 64, 0)
    dq = oracle.storage_bytes(nk, 64, 256)
    assert plain["codes"] == dq["codes"] == nk // 2
    bits_plain = Fraction(8 * (plain["absmax_q"] + plain["absmax_c2"] + plain["mean"]), nk)
    bits_dq = Fraction(8 * (dq["absmax_q"] + dq["absmax_c2"] + dq["mean"]), nk)
    assert bits_plain == Fraction(1, 2)
    assert bits_plain - bits_dq == Fraction(373046875, 10 ** 9) - Fraction(32, nk)


def test_nf4_beats_fp4_and_int4_on_normal_weights():
    """The pages' ranking on zero-centred normal weights: NF4's quantization
    error is below both INT4's and FP4's (double quantization on or off)."""
    w = workloads.weight((512, 1024), proj=3)
    bits = workloads.bf16_bits(w)
    x = oracle.bf16_bits_to_f32(bits).astype(np.float64).reshape(-1)
    for dq in (True, False):
        err = {}
        for t in ("nf4", "fp4", "int4"):
            d = oracle.dequant_bits(oracle.quantize(bits, quant_type=t, double_quant=dq))
            err[t] = float(np.mean((oracle.bf16_bits_to_f32(d).astype(np.float64) - x) ** 2))
        assert err["nf4"] < err["int4"] and err["nf4"] < err["fp4"], err
