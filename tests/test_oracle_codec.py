"""Pins for the oracle's blockwise NF4 encode, double quantization and dequant.

Pages: automatone "QLoRA paper explained", paragraphs "4-bit NormalFloat (NF4)"
and "Double Quantization (DQ)" (one scaling constant per block; the constants
are quantized again); creativeworksofknowledge "QLoRA: Fine-Tune 70B on One
GPU", section "2. Double quantization" (FP32 -> FP8).  Every check here is
independent of the oracle's own arithmetic: exact rational brute force,
round trips the method must reproduce exactly, hand-built byte layouts, and
error bounds that follow from the format definitions.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads


def _bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits):
    return oracle.bf16_bits_to_f32(bits)


def _brute_codes(bits, L, bs=64):
    """Nearest level by exact rational arithmetic over all 16 levels; tie -> lower index."""
    x = _f32(bits)
    Lf = [Fraction(float(v)) for v in L]
    codes = []
    for b0 in range(0, len(x), bs):
        blk = x[b0:b0 + bs]
        c1 = np.max(np.abs(blk)) if blk.size else np.float32(0)
        for v in blk:
            if c1 == 0:
                codes.append(7)
                continue
            n = Fraction(float(np.float32(v) / np.float32(c1)))     # the float quotient
            d = [abs(n - l) for l in Lf]
            codes.append(min(range(16), key=lambda i: (d[i], i)))
    return codes


def _unpack(packed, numel):
    out = []
    for byte in packed:
        out += [int(byte) >> 4, int(byte) & 15]
    return out[:numel]


def test_brute_force_nearest_random_blocks(L):
    rng = np.random.Generator(np.random.PCG64(11))
    x = rng.standard_normal(4 * 64).astype(np.float32) * np.float32(0.02)
    bits = _bits(x)
    packed, c1 = oracle.encode(bits)
    assert _unpack(packed, bits.size) == _brute_codes(bits, L)
    assert np.array_equal(c1, np.max(np.abs(_f32(bits).reshape(4, 64)), axis=1))


def test_brute_force_at_midpoints_and_extremes(L):
    # blocks with c1 = 1 so that n == x exactly: put x at and around every midpoint
    vals = []
    for i in range(15):
        mid = (float(L[i]) + float(L[i + 1])) / 2.0
        m32 = np.float32(mid)
        vals += [m32, np.nextafter(m32, np.float32(2)), np.nextafter(m32, np.float32(-2))]
    vals = np.array(vals, dtype=np.float32)
    bits = oracle.bf16_rne_array(vals)           # the inputs are bf16 weights
    # put +-1 in every block so c1 == 1, and pad to whole blocks
    blocks = []
    for b0 in range(0, bits.size, 62):
        chunk = list(bits[b0:b0 + 62]) + list(_bits([1.0, -1.0]))
        chunk += list(_bits([0.0] * (64 - len(chunk))))
        blocks += chunk
    bits = np.array(blocks, dtype=np.uint16)
    packed, c1 = oracle.encode(bits)
    assert np.all(c1 == 1.0)
    assert _unpack(packed, bits.size) == _brute_codes(bits, L)


def test_tie_goes_to_lower_index(L):
    # find a level pair whose midpoint is an exact bf16 value (with c1 == 1 the quotient is exact)
    found = 0
    for i in range(15):
        mid = (Fraction(float(L[i])) + Fraction(float(L[i + 1]))) / 2
        b = oracle.bf16_rne(float(mid))
        if Fraction(float(_f32(np.array([b], np.uint16))[0])) == mid:
            assert oracle.nearest(float(mid), L) == i
            found += 1
    # the zero level gives one: midpoint of L[7] = 0 and L[8] need not be bf16, so also
    # check the float tie directly through nearest() on every float midpoint
    for i in range(15):
        mid = (Fraction(float(L[i])) + Fraction(float(L[i + 1]))) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            assert oracle.nearest(f, L) == i
            found += 1
    assert found > 0


def test_zero_block_and_ragged_tail(L):
    bits = np.concatenate([_bits([0.0] * 64), _bits([0.01, -0.02, 0.03])])
    packed, c1 = oracle.encode(bits)
    assert c1.tolist()[0] == 0.0
    codes = _unpack(packed, 64 + 3)
    assert codes[:64] == [7] * 64
    assert codes[64:] == _brute_codes(bits[64:], L)
    assert packed.size == (67 + 1) // 2
    assert int(packed[-1]) & 15 == 7          # odd count: padding nibble is the zero code


def test_packing_high_nibble_first(L):
    # c1 = 1 block holding exactly the levels 3 and 12 first
    vals = [float(L[3]), float(L[12]), 1.0] + [0.0] * 61
    packed, _ = oracle.encode(_bits(vals))
    assert int(packed[0]) == (3 << 4) | 12
    assert int(packed[1]) == (15 << 4) | 7


def test_codebook_round_trip_exact(L):
    """Blocks whose absmax is exactly 1: mu = 1, c2 = 0, q = 0, c1' = 1, and a weight
    equal to bf16(L[i]) encodes to i and decodes to bf16(L[i]) exactly, for all i."""
    lv = oracle.bf16_rne_array(L)
    block = np.tile(lv, 4)                       # 64 weights, contains -1 and +1
    bits = np.tile(block, 8)                     # 8 blocks, all c1 == 1
    qt = oracle.quantize(bits)
    assert np.all(qt["c1"] == 1.0)
    assert qt["mean"] == np.float32(1.0)
    assert np.all(qt["absmax_c2"] == 0.0) and np.all(qt["absmax_q"] == 0)
    assert _unpack(qt["codes"], bits.size) == list(range(16)) * 32
    out = oracle.dequant(qt["codes"], qt["absmax_q"], qt["absmax_c2"], qt["mean"], bits.size)
    assert np.array_equal(out, bits)


def test_double_quant_structure():
    rng = np.random.Generator(np.random.PCG64(5))
    c1 = np.abs(rng.standard_normal(1000)).astype(np.float32) * np.float32(0.05) + np.float32(0.01)
    c1 = _f32(oracle.bf16_rne_array(c1))         # block maxima of bf16 weights are bf16 values
    q, c2, mu = oracle.double_quant(c1, 256)
    assert q.size == 1000 and c2.size == 4
    assert mu == np.float32(np.sum(c1.astype(np.float64)) / 1000)
    # the mean is order independent (the double sum of bf16 values is exact here)
    perm = rng.permutation(1000)
    assert oracle.block_mean(c1[perm]) == mu
    for g in range(4):
        grp = c1[g * 256:(g + 1) * 256]
        dev = np.abs(grp - mu)                  # float subtraction
        assert c2[g] == np.max(dev)
        # the group's largest deviation maps to the end of the FP8 range
        j = int(np.argmax(dev))
        assert abs(oracle.e4m3_to_float(int(q[g * 256 + j]))) == 448.0


def test_double_quant_error_bound():
    """c1' is within half an E4M3 step (scaled by c2/448) of c1, plus float rounding."""
    rng = np.random.Generator(np.random.PCG64(6))
    c1 = _f32(oracle.bf16_rne_array(np.abs(rng.standard_normal(4096)).astype(np.float32) * np.float32(0.03)))
    q, c2, mu = oracle.double_quant(c1, 256)
    for b in range(4096):
        t448 = (c1[b] - mu) / c2[b // 256] * 448.0
        e = max(int(np.floor(np.log2(max(abs(t448), 2.0 ** -6)))), -6)
        half_step = 2.0 ** (e - 3) / 2               # half an E4M3 ulp at t*448
        bound = c2[b // 256] / 448.0 * (half_step + 1e-3) + 4 * np.finfo(np.float32).eps * max(abs(mu), abs(c1[b]))
        c1p = oracle.block_constant(int(q[b]), float(c2[b // 256]), float(mu))
        assert abs(float(c1p) - float(c1[b])) <= bound


def test_dequant_error_bound(L):
    w = workloads.weight((64, 256), proj=3, outliers=True)
    bits = workloads.bf16_bits(w)
    qt = oracle.quantize(bits)
    wd = oracle.dequant_tensor(qt).reshape(-1).astype(np.float64)
    x = _f32(bits).reshape(-1).astype(np.float64)
    half_gap = np.max(np.diff(L.astype(np.float64))) / 2
    nb = x.size // 64
    for b in range(nb):
        c1 = float(qt["c1"][b])
        c1p = float(oracle.block_constant(int(qt["absmax_q"][b]), float(qt["absmax_c2"][b // 256]), float(qt["mean"])))
        blk = slice(b * 64, (b + 1) * 64)
        # |x - w'| <= c1 * half_gap (code choice) + |c1 - c1'| (constant) + 2^-8 |w'| (bf16)
        bound = c1 * half_gap + abs(c1 - c1p) + 2.0 ** -8 * np.abs(wd[blk]) + 1e-12
        assert np.all(np.abs(x[blk] - wd[blk]) <= bound)


def test_dequant_reads_each_level_and_constant(L):
    # hand-built stored tensor: 2 blocks, known codes, q and c2 -> expected values by formula
    packed = np.array([(0 << 4) | 15] + [(7 << 4) | 8] * 31 + [(15 << 4) | 0] * 32, dtype=np.uint8)
    q = np.array([0x38, 0xB8], dtype=np.uint8)      # +1.0 and -1.0 in E4M3
    c2 = np.array([448.0], dtype=np.float32)
    mu = np.float32(2.0)
    out = _f32(oracle.dequant(packed, q, c2, mu, 128))
    # c1' = fma(+-1, 448/448, 2) = 3 and 1
    assert out[0] == np.float32(-3.0) and out[1] == np.float32(3.0)
    assert out[2] == 0.0 and out[3] == _f32(oracle.bf16_rne_array(np.float32(L[8] * 3.0)))[0]
    assert out[64] == np.float32(1.0) and out[65] == np.float32(-1.0)


@pytest.mark.parametrize("shape", [(256, 256), (4096, 4096), (11008, 4096), (22016, 8192)])
def test_storage_closed_form(shape):
    """Actual byte counts reproduce 8/64 + 32/(64*256) bits of constants per weight."""
    numel = shape[0] * shape[1]
    sb = oracle.storage_bytes(numel)
    assert sb["codes"] * 2 == numel                     # 4 bits per weight
    const_bits = 8 * (sb["absmax_q"] + sb["absmax_c2"] + sb["mean"]) / numel
    closed = 8 / 64 + 32 / (64 * 256) + 32 / numel
    assert const_bits == closed
    no_dq_bits = 32 * (numel // 64) / numel
    assert no_dq_bits == 0.5
    saved = no_dq_bits - (8 / 64 + 32 / (64 * 256))
    assert saved == 0.373046875


def test_storage_golden_matches_pages():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "storage_closed_form.txt")
    g = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            g[k] = float(v)
    assert 8 / 64 + 32 / (64 * 256) == g["bits_with_dq_asymptotic"]
    assert g["bits_without_dq"] - g["bits_with_dq_asymptotic"] == g["bits_saved_asymptotic"]
    assert round(g["bits_saved_asymptotic"], 2) == g["bits_saved_pages_approx"]
    gb = g["params_65b"] * g["bits_saved_asymptotic"] / 8 / 1e9
    assert round(gb) == g["gb_saved_65b_pages_approx"]        # the pages' approximate figure for 65B
    # count the real bytes for a 65B-parameter tensor (a multiple of 64*256)
    numel = int(g["params_65b"]) // 16384 * 16384
    sb = oracle.storage_bytes(numel)
    saved_bytes = 4 * (numel // 64) - (sb["absmax_q"] + sb["absmax_c2"] + sb["mean"])
    assert abs(saved_bytes / 1e9 - gb) < 1e-3
