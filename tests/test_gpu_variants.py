"""GPU parity of the variants: the FP4 and INT4 level tables the pages compare
NF4 with (automatone "QLoRA paper explained", "4-bit NormalFloat (NF4)"), and
the stored form without double quantization (fp32 constants, 0.5 bits per
weight: creativeworksofknowledge "QLoRA: Fine-Tune 70B on One GPU", "2. Double
quantization"), through the same kernels as NF4 with double quantization.

Bar: bit-exact codes, constants and dequantized bf16 weights; max|err| <=
2e-2 * rms(oracle) per tensor for Y, X A^T, dX, dA, dB.  Every expected value
comes from the oracle on the CPU.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-2
VARIANTS = [(t, dq) for t in ("nf4", "fp4", "int4") for dq in (True, False) if (t, dq) != ("nf4", True)]


@pytest.fixture(scope="module")
def qb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_nf4_quantized_encode_b200 as m
    return m


def _upload(qb, qt, rows, cols):
    """The oracle's stored tensor in the library's descriptor."""
    t = qb.empty_nf4(rows, cols, torch.device("cuda"), qt["quant_type"], qt["double_quant"])
    t.codes[: qt["codes"].size].copy_(torch.from_numpy(qt["codes"]))
    if qt["double_quant"]:
        t.absmax_q[: qt["absmax_q"].size].copy_(torch.from_numpy(qt["absmax_q"]))
        t.absmax_c2[: qt["absmax_c2"].size].copy_(torch.from_numpy(qt["absmax_c2"]))
        t.absmax_mean[:1].copy_(torch.tensor([float(qt["mean"])], dtype=torch.float32))
    else:
        t.absmax[: qt["absmax"].size].copy_(torch.from_numpy(qt["absmax"]))
    return t


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def _codec_case(qb, w, quant_type, dq):
    rows, cols = w.shape
    ref = oracle.quantize(workloads.bf16_bits(w), quant_type=quant_type, double_quant=dq)
    got = qb.qlora_quantize_nf4_dq(w.cuda(), quant_type=quant_type, double_quant=dq)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    n = ref["codes"].size
    codes = got.codes[:n].cpu().numpy()
    bad = np.nonzero(codes != ref["codes"])[0]
    assert bad.size == 0, f"{bad.size} code bytes differ; first at {bad[0]}"
    if dq:
        nb = ref["absmax_q"].size
        assert np.array_equal(got.absmax_q[:nb].cpu().numpy(), ref["absmax_q"])
        assert np.array_equal(got.absmax_c2[: ref["absmax_c2"].size].cpu().numpy().view(np.uint32),
                              ref["absmax_c2"].view(np.uint32))
        assert got.absmax_mean[:1].cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
    else:
        assert np.array_equal(got.absmax[: ref["absmax"].size].cpu().numpy().view(np.uint32),
                              ref["absmax"].view(np.uint32))
    deq = qb.qlora_dequantize(_upload(qb, ref, rows, cols))
    torch.cuda.synchronize()
    want = oracle.dequant_bits(ref)
    bad = np.nonzero(_bits(deq)[: ref["numel"]] != want)[0]
    assert bad.size == 0, f"{bad.size} dequantized weights differ; first {bad[0]}"


@pytest.mark.parametrize("quant_type,dq", VARIANTS)
@pytest.mark.parametrize("shape", [(256, 256), (300, 4160), (5, 13), (1, 64 * 256 + 8)])
def test_codec_variants_small_and_ragged(qb, quant_type, dq, shape):
    _codec_case(qb, workloads.weight(shape, proj=shape[0] % 5), quant_type, dq)


@pytest.mark.parametrize("quant_type,dq", VARIANTS)
def test_codec_variants_4096_outliers(qb, quant_type, dq):
    _codec_case(qb, workloads.weight((4096, 4096), proj=0, outliers=True), quant_type, dq)


@pytest.mark.parametrize("quant_type", ["fp4", "int4"])
def test_codec_variant_thresholds_and_levels(qb, quant_type):
    """Weights at, above and below every decision midpoint of the type's table
    and at every level, in blocks with absmax 1 (so n == x), and scaled copies."""
    L = oracle.levels(quant_type)
    vals = []
    for i in range(15):
        m = np.float32((float(L[i]) + float(L[i + 1])) / 2)
        vals += [m, np.nextafter(m, np.float32(2)), np.nextafter(m, np.float32(-2))]
    vals += list(L)
    vals = oracle.bf16_bits_to_f32(oracle.bf16_rne_array(np.array(vals, np.float32)))
    blocks = []
    for i in range(0, len(vals), 62):
        chunk = list(vals[i:i + 62]) + [1.0, -1.0]
        blocks += chunk + [0.0] * (64 - len(chunk))
    base = np.array(blocks, np.float32)
    allw = np.concatenate([base * np.float32(s) for s in (1.0, 0.5, 0.0078125, 3.0)])
    w = torch.from_numpy(allw).to(torch.bfloat16).reshape(4, -1)
    for dq in (True, False):
        _codec_case(qb, w, quant_type, dq)


@functools.lru_cache(maxsize=4)
def _oracle_weight(n, k, proj, quant_type, dq):
    qt = oracle.quantize(workloads.bf16_bits(workloads.weight((n, k), proj=proj)), quant_type=quant_type,
                         double_quant=dq)
    return qt, oracle.dequant_tensor(qt)


def _close(name, got, ref, tag):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got)), name
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    print(f"PARITY {tag} {name}: max|err|/rms = {err / rms:.3e} (bar {TOL:.0e})")
    assert err <= TOL * rms, f"{name} [{tag}]: max|err| {err:.4g} > {TOL} * rms {rms:.4g}"


def _linear_variant(qb, quant_type, dq, n, k, m, r, proj, rows_sample=None, check_bwd=True):
    qt, Wd = _oracle_weight(n, k, proj, quant_type, dq)
    X, A = workloads.activations(m, k, proj), workloads.lora_a(r, k, proj)
    B, dY = workloads.lora_b(n, r, proj), workloads.grad_output(m, n, proj)
    s = 16.0 / r
    up = _upload(qb, qt, n, k)
    Y, XA = qb.qlora_linear_fwd(up, X.cuda(), A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    rows = np.arange(m) if rows_sample is None else rows_sample
    Xf, Af, Bf, dYf = (t.float().numpy() for t in (X, A, B, dY))
    tag = f"{quant_type}{'+dq' if dq else ''} {n}x{k} m={m}"
    _close("Y", Y.float().cpu().numpy()[rows], oracle.linear_fwd_rows(Wd, Xf, Af, Bf, s, rows), tag)
    XA_ref, _, dA_ref, dB_ref = oracle.lora_grads(Xf, dYf, Af, Bf, s)
    _close("XA", XA.cpu().numpy()[rows], XA_ref[rows], tag)
    if not check_bwd:
        return
    dX, dA, dB = qb.qlora_linear_bwd(up, X.cuda(), dY.cuda(), A.cuda(), B.cuda(), s, XA=XA)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    _close("dX", dX.float().cpu().numpy()[rows], oracle.linear_bwd_dx_rows(Wd, dYf, Af, Bf, s, rows), tag)
    _close("dA", dA.cpu().numpy(), dA_ref, tag)
    _close("dB", dB.cpu().numpy(), dB_ref, tag)


@pytest.mark.parametrize("quant_type,dq", VARIANTS)
@pytest.mark.parametrize("m", [1, 16, 257])
def test_linear_variants(qb, quant_type, dq, m):
    """Decode-shaped (1 and 16 tokens: the weight stream) and prefill-shaped
    (257 tokens: the fused dequant-GEMM both ways) calls on a 392 x 640 layer."""
    _linear_variant(qb, quant_type, dq, 392, 640, m, 64, proj=3)


@pytest.mark.parametrize("quant_type,dq", [("nf4", False), ("fp4", True), ("int4", True)])
def test_linear_variants_full_size(qb, quant_type, dq):
    """A 65B attention projection (8192 x 8192) at 8192 tokens with each
    variant: Y and dX on 64 sampled token rows, dA and dB in full; and the
    decode forward at 4 tokens on the same weight."""
    rng = np.random.Generator(np.random.PCG64(94))
    rows = np.sort(rng.choice(8192, 64, replace=False))
    _linear_variant(qb, quant_type, dq, 8192, 8192, 8192, 64, proj=1, rows_sample=rows)
    _linear_variant(qb, quant_type, dq, 8192, 8192, 4, 64, proj=1, check_bwd=False)
