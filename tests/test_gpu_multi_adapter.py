"""GPU parity of the batched decode with one LoRA adapter per token over one
frozen 4-bit weight (qlora_linear_fwd_multi), against the oracle's per-token
formula: Y[t] = X[t] deq(W)^T + s (X[t] A_a^T) B_a^T with a = adapter_idx[t],
no LoRA term for a negative index.  Bar: max|err| <= 2e-2 * rms(oracle) for Y
and X A^T; an out-of-range index must set bit 3 of the device error flag.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def qb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_nf4_quantized_encode_b200 as m
    return m


@functools.lru_cache(maxsize=2)
def _oracle_weight(n, k, proj):
    qt = oracle.quantize(workloads.bf16_bits(workloads.weight((n, k), proj=proj)))
    return qt, oracle.dequant_tensor(qt)


def _upload(qb, qt, n, k):
    t = qb.empty_nf4(n, k, torch.device("cuda"))
    t.codes[: qt["codes"].size].copy_(torch.from_numpy(qt["codes"]))
    t.absmax_q[: qt["absmax_q"].size].copy_(torch.from_numpy(qt["absmax_q"]))
    t.absmax_c2[: qt["absmax_c2"].size].copy_(torch.from_numpy(qt["absmax_c2"]))
    t.absmax_mean[:1].copy_(torch.tensor([float(qt["mean"])], dtype=torch.float32))
    return t


def _close(name, got, ref, tag):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got)), name
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    if rms == 0.0:                          # e.g. X A^T when no token has an adapter: exactly zero
        print(f"PARITY {tag} {name}: reference all zero, max|got| = {err:.3e}")
        assert err == 0.0, f"{name} [{tag}]: expected exact zeros, max|got| {err:.4g}"
        return
    print(f"PARITY {tag} {name}: max|err|/rms = {err / rms:.3e} (bar {TOL:.0e})")
    assert err <= TOL * rms, f"{name} [{tag}]: max|err| {err:.4g} > {TOL} * rms {rms:.4g}"


def _multi_case(qb, n, k, idx, n_ad, r=64, proj=7):
    qt, Wd = _oracle_weight(n, k, proj)
    m = len(idx)
    X = workloads.activations(m, k, proj)
    A_st = torch.stack([workloads.lora_a(r, k, 40 + a) for a in range(n_ad)])
    B_st = torch.stack([workloads.lora_b(n, r, 40 + a) for a in range(n_ad)])
    s = 16.0 / r
    up = _upload(qb, qt, n, k)
    idx_t = torch.tensor(idx, dtype=torch.int32, device="cuda")
    Y, XA = qb.qlora_linear_fwd_multi(up, X.cuda(), A_st.cuda(), B_st.cuda(), idx_t, s)
    torch.cuda.synchronize()
    flags = qb.qlora_read_device_errors()
    Y_ref, XA_ref = oracle.linear_fwd_multi(Wd, X.float().numpy(), A_st.float().numpy(), B_st.float().numpy(),
                                            np.array(idx), s)
    tag = f"{n}x{k} m={m} adapters={n_ad}"
    _close("Y", Y.float().cpu().numpy(), Y_ref, tag)
    _close("XA", XA.cpu().numpy(), XA_ref, tag)
    return flags


@pytest.mark.parametrize("idx,n_ad", [
    ([0], 1),
    ([2, 0, 1, 2], 3),
    ([3, 3, 0, -1, 1, 2, 3, 0, 1], 4),
    (list(range(16)), 16),
    ([5] * 16, 8),
    ([-1] * 4, 2),
])
def test_multi_adapter_decode(qb, idx, n_ad):
    assert _multi_case(qb, 392, 640, idx, n_ad) == 0


def test_multi_adapter_wide_rank(qb):
    """Rank 136: three 64-column groups of the rank per adapter pass."""
    assert _multi_case(qb, 392, 640, [1, 0, 1, 2, 0], 3, r=136) == 0


def test_multi_adapter_matches_single_adapter_call(qb):
    """Every token on adapter a gives the single-adapter forward with (A_a, B_a)."""
    n, k, m, r = 392, 640, 7, 64
    qt, _ = _oracle_weight(n, k, 7)
    up = _upload(qb, qt, n, k)
    X = workloads.activations(m, k, 7).cuda()
    A_st = torch.stack([workloads.lora_a(r, k, 50 + a) for a in range(3)]).cuda()
    B_st = torch.stack([workloads.lora_b(n, r, 50 + a) for a in range(3)]).cuda()
    Ym, XAm = qb.qlora_linear_fwd_multi(up, X, A_st, B_st, torch.full((m,), 2, dtype=torch.int32, device="cuda"),
                                        0.25)
    Ys, XAs = qb.qlora_linear_fwd(up, X, A_st[2].contiguous(), B_st[2].contiguous(), 0.25)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    ref = Ys.float().cpu().numpy().astype(np.float64)
    err = np.max(np.abs(Ym.float().cpu().numpy() - ref)) / np.sqrt(np.mean(ref ** 2))
    assert err <= 1e-2, err
    assert np.allclose(XAm.cpu().numpy(), XAs.cpu().numpy(), rtol=1e-5, atol=1e-6)


def test_multi_adapter_65b_ffn_sixteen_adapters(qb):
    """16 tokens on 16 different adapters over the 65B FFN weight 22016 x 8192."""
    assert _multi_case(qb, 22016, 8192, list(range(15, -1, -1)), 16, proj=5) == 0


def test_out_of_range_adapter_index_is_flagged(qb):
    """An index beyond the stack cannot be checked on the host: the token gets no
    LoRA term (like a negative index) and bit 3 of the error flag is set."""
    flags = _multi_case(qb, 392, 640, [0, 7, 1], 2)
    assert flags & 8, f"flags {flags:#x}"
    assert qb.qlora_read_device_errors() == 0          # the read above cleared it
