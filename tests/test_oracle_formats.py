"""Pins for the oracle's scalar roundings (bf16 RNE, OCP E4M3) against torch's casts.

torch's CPU casts are an independent implementation of the same IEEE / OCP
rounding rules, so agreement on a dense sweep plus the edge cases pins them.
"""
import numpy as np
import torch

import oracle


def _edge_floats():
    vals = [0.0, -0.0, 1.0, -1.0, 448.0, -448.0, 1e-40, -1e-40, 3.4e38, -3.4e38,
            np.float32(np.finfo(np.float32).tiny), 2.0 ** -133, 2.0 ** -134, 2.0 ** -149]
    # exact bf16 ties: 1 + 2^-8 (tie, even -> 1), 1 + 3*2^-8 (tie, even -> up)
    vals += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.5 + 2.0 ** -9]
    return np.array(vals, dtype=np.float32)


def test_bf16_rne_matches_torch_sweep():
    rng = np.random.Generator(np.random.PCG64(123))
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e-38).astype(np.float32),      # subnormal range
        (rng.standard_normal(50_000) * 1e30).astype(np.float32),
        rng.integers(0, 2**32, 100_000, dtype=np.uint64).astype(np.uint32).view(np.float32),
        _edge_floats(),
    ])
    x = x[np.isfinite(x)]
    ours = oracle.bf16_rne_array(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[0]]!r} ours={ours[bad[0]]:#06x} ref={ref[bad[0]]:#06x}"


def test_bf16_rne_every_tie_pattern():
    # every bf16 value plus exactly half an ulp: a tie that must go to the even neighbour
    b = np.arange(0, 0x7F80, dtype=np.uint32)            # positive finite bf16 patterns
    f = (b << 16).view(np.float32)
    tie = ((b << 16) | 0x8000).view(np.float32)
    for arr in (f, tie, -tie):
        ours = oracle.bf16_rne_array(arr)
        ref = torch.from_numpy(np.ascontiguousarray(arr)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(ours, ref)


def test_e4m3_decode_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    ours = np.array([oracle.e4m3_to_float(int(c)) for c in codes], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.max(ours[~nan]) == 448.0


def test_e4m3_rne_matches_torch():
    rng = np.random.Generator(np.random.PCG64(7))
    t = rng.uniform(-1.0, 1.0, 300_000).astype(np.float32)
    x = np.concatenate([t * np.float32(448.0), (t * np.float32(1e-2)).astype(np.float32),
                        (t * np.float32(2.0 ** -8)).astype(np.float32)])
    # exact ties between adjacent E4M3 values, both normal and subnormal
    vals = np.array([oracle.e4m3_to_float(c) for c in range(0, 0x7E)], dtype=np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.array([0.0, -0.0, 448.0, -448.0], np.float32)])
    ours = oracle.e4m3_rne_array(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[0]]!r} ours={ours[bad[0]]:#04x} ref={ref[bad[0]]:#04x}"
