"""Pins for the oracle's LoRA linear forward/backward formulas.

Pages: automatone "QLoRA paper explained", section "How it works" (dequantize
to bf16 on the fly, run the math; gradients flow through the frozen 4-bit base
and land only on the 16-bit LoRA adapters); the Deep Analysis methodology on
the gptget.net page (backward dequantizes to 16-bit for the matmul).  The
formulas Y = X W'^T + s (X A^T) B^T, dX, dA, dB are the hot path's statement.

The gradients are pinned against torch float64 autograd, which derives them
independently of the hand-written backward formulas; B = 0 or s = 0 reduce the
layer to a plain matmul against the dequantized weight.
"""
import numpy as np
import torch

import oracle
import workloads


def _case(m=16, n=48, k=64, r=8, proj=0):
    w = workloads.weight((n, k), proj)
    qt = oracle.quantize(workloads.bf16_bits(w))
    Wd = oracle.dequant_tensor(qt)
    X = workloads.activations(m, k, proj).float().numpy()
    A = workloads.lora_a(r, k, proj).float().numpy()
    B = workloads.lora_b(n, r, proj).float().numpy()
    dY = workloads.grad_output(m, n, proj).float().numpy()
    return Wd, X, A, B, dY


def test_forward_and_backward_match_autograd():
    Wd, X, A, B, dY = _case()
    s = 2.0
    Y, XA = oracle.linear_fwd(Wd, X, A, B, s)
    dX, dA, dB = oracle.linear_bwd(Wd, X, dY, A, B, s)

    Xt = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    At = torch.tensor(A, dtype=torch.float64, requires_grad=True)
    Bt = torch.tensor(B, dtype=torch.float64, requires_grad=True)
    Wt = torch.tensor(Wd, dtype=torch.float64)                   # frozen
    Yt = torch.nn.functional.linear(Xt, Wt) + s * torch.nn.functional.linear(
        torch.nn.functional.linear(Xt, At), Bt)
    Yt.backward(torch.tensor(dY, dtype=torch.float64))
    rms = lambda a: float(np.sqrt(np.mean(np.square(a))))
    assert np.max(np.abs(Y - Yt.detach().numpy())) <= 1e-12 * rms(Y)
    assert np.max(np.abs(XA - (X.astype(np.float64) @ A.T.astype(np.float64)))) <= 1e-12 * rms(XA)
    assert np.max(np.abs(dX - Xt.grad.numpy())) <= 1e-12 * rms(dX)
    assert np.max(np.abs(dA - At.grad.numpy())) <= 1e-12 * rms(dA)
    assert np.max(np.abs(dB - Bt.grad.numpy())) <= 1e-12 * rms(dB)


def test_lora_grads_match_autograd():
    """oracle.lora_grads (X A^T, dY B, dA, dB: what the GPU parity tests compare
    against at full size) against torch float64 autograd of the LoRA branch
    alone, and its intermediates against the hidden activations autograd saw."""
    _, X, A, B, dY = _case(m=24, n=40, k=128, r=16, proj=4)
    s = 0.25
    XA, G, dA, dB = oracle.lora_grads(X, dY, A, B, s)
    Xt = torch.tensor(X, dtype=torch.float64)
    At = torch.tensor(A, dtype=torch.float64, requires_grad=True)
    Bt = torch.tensor(B, dtype=torch.float64, requires_grad=True)
    H = torch.nn.functional.linear(Xt, At)            # X A^T
    H.retain_grad()
    Yl = s * torch.nn.functional.linear(H, Bt)
    Yl.backward(torch.tensor(dY, dtype=torch.float64))
    rms = lambda a: float(np.sqrt(np.mean(np.square(a))))
    assert np.max(np.abs(XA - H.detach().numpy())) <= 1e-12 * rms(XA)
    # dL/dH = s dY B = s G
    assert np.max(np.abs(s * G - H.grad.numpy())) <= 1e-12 * rms(G)
    assert np.max(np.abs(dA - At.grad.numpy())) <= 1e-12 * rms(dA)
    assert np.max(np.abs(dB - Bt.grad.numpy())) <= 1e-12 * rms(dB)
    # the same quantities as the full layer's backward (W only adds to dX)
    Wd = np.zeros((40, 128), np.float32)
    _, dA2, dB2 = oracle.linear_bwd(Wd, X, dY, A, B, s)
    assert np.array_equal(dA, dA2) and np.array_equal(dB, dB2)


def test_zero_lora_reduces_to_plain_matmul():
    Wd, X, A, B, dY = _case(m=8, n=32, k=128, r=4, proj=1)
    Y0, _ = oracle.linear_fwd(Wd, X, A, np.zeros_like(B), 2.0)
    Ys, _ = oracle.linear_fwd(Wd, X, A, B, 0.0)
    plain = torch.nn.functional.linear(torch.tensor(X, dtype=torch.float64),
                                       torch.tensor(Wd, dtype=torch.float64)).numpy()
    assert np.array_equal(Y0, plain) or np.max(np.abs(Y0 - plain)) < 1e-12
    assert np.max(np.abs(Ys - plain)) < 1e-12
    dX, dA, dB = oracle.linear_bwd(Wd, X, dY, A, B, 0.0)
    assert np.max(np.abs(dX - dY.astype(np.float64) @ Wd.astype(np.float64))) < 1e-12
    assert np.all(dA == 0) and np.all(dB == 0)


def test_row_restricted_forms_equal_full():
    Wd, X, A, B, dY = _case(m=32, n=40, k=64, r=8, proj=2)
    rows = np.array([0, 5, 31, 7])
    Y, _ = oracle.linear_fwd(Wd, X, A, B, 0.25)
    dX, _, _ = oracle.linear_bwd(Wd, X, dY, A, B, 0.25)
    assert np.allclose(oracle.linear_fwd_rows(Wd, X, A, B, 0.25, rows), Y[rows], rtol=0, atol=1e-12)
    assert np.allclose(oracle.linear_bwd_dx_rows(Wd, dY, A, B, 0.25, rows), dX[rows], rtol=0, atol=1e-12)


def test_gradients_are_lora_only_and_scale_linearly():
    Wd, X, A, B, dY = _case(proj=3)
    dX1, dA1, dB1 = oracle.linear_bwd(Wd, X, dY, A, B, 1.0)
    dX2, dA2, dB2 = oracle.linear_bwd(Wd, X, dY, A, B, 2.0)
    assert np.allclose(dA2, 2 * dA1, rtol=1e-13, atol=0) and np.allclose(dB2, 2 * dB1, rtol=1e-13, atol=0)
    assert dA1.shape == A.shape and dB1.shape == B.shape and dX1.shape == X.shape


def test_multi_adapter_forward_properties():
    """Per-token adapters: one adapter for every token reduces to the single-
    adapter forward; a negative index means the base weight alone; permuting
    the tokens together with their indices permutes the rows; an adapter no
    token uses changes nothing; zero B_a removes exactly adapter a's term."""
    Wd, X, A, B, dY = _case(m=12, n=40, k=128, r=8, proj=5)
    rng = np.random.Generator(np.random.PCG64(7))
    A_st = np.stack([A, 0.5 * A[::-1], rng.standard_normal(A.shape).astype(np.float32) * 0.02])
    B_st = np.stack([B, -B, rng.standard_normal(B.shape).astype(np.float32) * 0.02])
    s = 2.0
    for a in range(3):
        Y1, XA1 = oracle.linear_fwd_multi(Wd, X, A_st, B_st, np.full(12, a), s)
        Y2, XA2 = oracle.linear_fwd(Wd, X, A_st[a], B_st[a], s)
        assert np.max(np.abs(Y1 - Y2)) <= 1e-12 * np.sqrt(np.mean(Y2 ** 2))
        assert np.max(np.abs(XA1 - XA2)) <= 1e-12 * np.sqrt(np.mean(XA2 ** 2))
    base = X.astype(np.float64) @ Wd.T.astype(np.float64)
    Yn, XAn = oracle.linear_fwd_multi(Wd, X, A_st, B_st, np.full(12, -1), s)
    assert np.array_equal(Yn, base) and np.all(XAn == 0)
    idx = np.array([0, 1, 2, -1, 2, 2, 0, 1, 1, 0, 2, 1])
    Y, XA = oracle.linear_fwd_multi(Wd, X, A_st, B_st, idx, s)
    perm = rng.permutation(12)
    Yp, XAp = oracle.linear_fwd_multi(Wd, X[perm], A_st, B_st, idx[perm], s)
    assert np.max(np.abs(Yp - Y[perm])) < 1e-12 and np.max(np.abs(XAp - XA[perm])) < 1e-12
    A4 = np.concatenate([A_st, A_st[:1] * 3])
    B4 = np.concatenate([B_st, B_st[:1] * 3])
    Y4, _ = oracle.linear_fwd_multi(Wd, X, A4, B4, idx, s)
    assert np.max(np.abs(Y4 - Y)) < 1e-12
    Bz = B_st.copy()
    Bz[1] = 0
    Yz, _ = oracle.linear_fwd_multi(Wd, X, A_st, Bz, idx, s)
    assert np.max(np.abs(Yz[idx == 1] - base[idx == 1])) < 1e-12
    assert np.max(np.abs(Yz[idx != 1] - Y[idx != 1])) < 1e-12
