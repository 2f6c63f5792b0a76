"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bar: bit-exact for NF4 codes, E4M3 constants, c2, the mean and dequantized bf16
weights; max |err| <= 2e-2 * rms(oracle) per tensor for Y, dX, dA, dB.
The GEMM cases take the oracle's quantized weight as their input (uploaded),
so they do not depend on the GPU encoder; every expected value comes from the
oracle on the CPU.
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


def _no_device_errors(qb):
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0


def _upload_oracle_quant(qb, qt):
    dev = torch.device("cuda")
    t = qb.empty_nf4(qt["shape"][0] if len(qt["shape"]) == 2 else 1,
                     qt["shape"][1] if len(qt["shape"]) == 2 else qt["numel"], dev)
    t.codes[: qt["codes"].size].copy_(torch.from_numpy(qt["codes"]))
    t.absmax_q[: qt["absmax_q"].size].copy_(torch.from_numpy(qt["absmax_q"]))
    t.absmax_c2[: qt["absmax_c2"].size].copy_(torch.from_numpy(qt["absmax_c2"]))
    t.absmax_mean[:1].copy_(torch.tensor([float(qt["mean"])], dtype=torch.float32))
    return t


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def _assert_codec_equal(qb, w_cpu: torch.Tensor):
    bits = workloads.bf16_bits(w_cpu)
    ref = oracle.quantize(bits)
    got = qb.qlora_quantize_nf4_dq(w_cpu.cuda())
    _no_device_errors(qb)
    n = ref["codes"].size
    codes = got.codes[:n].cpu().numpy()
    bad = np.nonzero(codes != ref["codes"])[0]
    assert bad.size == 0, f"{bad.size} code bytes differ; first at byte {bad[0]}: {codes[bad[0]]:#x} vs {ref['codes'][bad[0]]:#x}"
    nb = ref["absmax_q"].size
    assert np.array_equal(got.absmax_mean[:1].cpu().numpy().view(np.uint32),
                          np.array([ref["mean"]], np.float32).view(np.uint32))
    assert np.array_equal(got.absmax_c2[: ref["absmax_c2"].size].cpu().numpy().view(np.uint32),
                          ref["absmax_c2"].view(np.uint32))
    assert np.array_equal(got.absmax_q[:nb].cpu().numpy(), ref["absmax_q"])
    # dequantize the ORACLE's stored tensor on the GPU and compare with the oracle's dequant
    up = _upload_oracle_quant(qb, ref)
    deq = qb.qlora_dequantize(up)
    _no_device_errors(qb)
    ref_deq = oracle.dequant(ref["codes"], ref["absmax_q"], ref["absmax_c2"], ref["mean"], ref["numel"])
    got_deq = _bits(deq)[: ref["numel"]]
    bad = np.nonzero(got_deq != ref_deq)[0]
    assert bad.size == 0, f"{bad.size} dequantized weights differ; first {bad[0]}"


@pytest.mark.parametrize("shape", [(256, 256), (64, 64), (128, 192), (3, 100), (1, 1), (1, 7),
                                   (5, 13), (1, 64 * 256 + 8), (300, 4160)])
def test_codec_small_and_ragged(qb, shape):
    w = workloads.weight(shape, proj=shape[0] % 7)
    _assert_codec_equal(qb, w)


def test_codec_4096_outliers(qb):
    w = workloads.weight((4096, 4096), proj=0, outliers=True)
    _assert_codec_equal(qb, w)


@pytest.mark.parametrize("shape", [(11008, 4096), (22016, 8192)])
def test_codec_llama_shapes(qb, shape):
    _assert_codec_equal(qb, workloads.weight(shape, proj=4))


def test_codec_thresholds_and_levels(qb):
    """Weights placed at, just above and just below every decision midpoint, and
    at every level, with block absmax 1 so the quotient is the value itself."""
    L = oracle.codebook()
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
    # scaled copies exercise other absmax values with the same quotients
    base = np.array(blocks, np.float32)
    allw = np.concatenate([base * np.float32(s) for s in (1.0, 0.5, 0.0078125, 3.0)])
    w = torch.from_numpy(allw).to(torch.bfloat16).reshape(1, -1)
    _assert_codec_equal(qb, w)


def _near_threshold_pairs(band=2.0 ** -18):
    """(c1, x) bf16 pairs whose IEEE quotient x / c1 lies within `band` of a
    decision midpoint, found by search over c1 (CPU, float32 arithmetic)."""
    L = oracle.codebook().astype(np.float64)
    mids = [(L[i] + L[i + 1]) / 2 for i in range(15)]
    # positive bf16 values with exponents 2^-6 .. 2^6
    c1 = oracle.bf16_bits_to_f32(np.arange(0x3C80, 0x4300, dtype=np.uint16))
    pairs = []
    for mid in mids:
        t = oracle.bf16_rne_array((c1 * np.float32(mid)).astype(np.float32))
        for delta in (-1, 0, 1):
            xb = (t.astype(np.int32) + (delta if mid >= 0 else -delta)).astype(np.uint16)
            x = oracle.bf16_bits_to_f32(xb)
            q = (x / c1).astype(np.float32)                 # IEEE float division
            hit = np.abs(q.astype(np.float64) - mid) <= band
            hit &= np.abs(x) <= c1
            pairs += list(zip(c1[hit], x[hit]))
    return pairs


def test_codec_quotients_next_to_thresholds(qb):
    """Blocks whose element quotient falls within 2^-18 of a decision midpoint:
    the encoder's reciprocal path must hand these to the IEEE-division path."""
    pairs = _near_threshold_pairs()
    assert len(pairs) >= 20, len(pairs)
    blocks = []
    for c1, x in pairs:
        blk = np.zeros(64, np.float32)
        blk[0], blk[17], blk[38], blk[63] = c1, x, -x, np.float32(0.5) * x
        blocks.append(blk)
    w = torch.from_numpy(np.concatenate(blocks)).to(torch.bfloat16).reshape(len(pairs), 64)
    _assert_codec_equal(qb, w)


def test_codec_zero_and_constant_blocks(qb):
    w = torch.zeros(4, 512, dtype=torch.bfloat16)
    w[1, :] = 0.5                      # constant blocks: c2 may be zero in a group
    w[2, 64:128] = -0.25
    _assert_codec_equal(qb, w)


# ------------------------------------------------------------------ linear layer
@functools.lru_cache(maxsize=2)
def _oracle_weight(n, k, proj):
    """The oracle's stored form of the seeded [n, k] weight and its dequantized
    float32 values (cached: several token counts share one weight)."""
    w = workloads.weight((n, k), proj=proj)
    qt = oracle.quantize(workloads.bf16_bits(w))
    return qt, oracle.dequant_tensor(qt)


def _linear_case(qb, n, k, m, r, alpha, proj, rows_sample=None, check_bwd=True, with_xa=True):
    qt, Wd = _oracle_weight(n, k, proj)                 # Wd float32 [n, k], bf16-exact
    X = workloads.activations(m, k, proj)
    A = workloads.lora_a(r, k, proj)
    B = workloads.lora_b(n, r, proj)
    dY = workloads.grad_output(m, n, proj)
    s = alpha / r
    up = _upload_oracle_quant(qb, qt)
    Xg, Ag, Bg, dYg = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    Y, XA = qb.qlora_linear_fwd(up, Xg, Ag, Bg, s, save_xa=True)
    _no_device_errors(qb)
    rows = np.arange(m) if rows_sample is None else rows_sample
    Xf, Af, Bf, dYf = (t.float().numpy() for t in (X, A, B, dY))
    tag = f"{n}x{k} m={m} r={r}"
    Y_ref = oracle.linear_fwd_rows(Wd, Xf, Af, Bf, s, rows)
    _close("Y", Y.float().cpu().numpy()[rows], Y_ref, tag)
    XA_ref, _, dA_ref, dB_ref = oracle.lora_grads(Xf, dYf, Af, Bf, s)
    _close("XA", XA.float().cpu().numpy()[rows], XA_ref[rows], tag)
    if not check_bwd:
        return
    dX, dA, dB = qb.qlora_linear_bwd(up, Xg, dYg, Ag, Bg, s, XA=XA if with_xa else None)
    _no_device_errors(qb)
    dX_ref = oracle.linear_bwd_dx_rows(Wd, dYf, Af, Bf, s, rows)
    _close("dX", dX.float().cpu().numpy()[rows], dX_ref, tag)
    _close("dA", dA.float().cpu().numpy(), dA_ref, tag)
    _close("dB", dB.float().cpu().numpy(), dB_ref, tag)


def _close(name, got, ref, tag=""):
    """max|err| <= TOL * rms(oracle), per tensor.  The ratio err/rms is printed
    (visible with -s) and put in the failure message, so the margin to the bar
    can be followed from run to run."""
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name} [{tag}]: non-finite output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref)))
    ratio = err / rms if rms > 0 else float("inf") if err > 0 else 0.0
    print(f"PARITY {tag} {name}: max|err|/rms = {ratio:.3e} (bar {TOL:.0e})")
    assert err <= TOL * rms, f"{name} [{tag}]: max|err| {err:.4g} > {TOL} * rms {rms:.4g} (ratio {ratio:.4g})"


def test_linear_tiny_layer(qb):
    """The 256x256 layer, 16 tokens, r = 8, alpha = 16 (s = 2): forward and backward."""
    _linear_case(qb, 256, 256, 16, 8, 16.0, proj=0)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_linear_decode_shapes(qb, m):
    _linear_case(qb, 392, 640, m, 64, 16.0, proj=1)


@pytest.mark.parametrize("m,r", [(1, 72), (9, 256), (16, 136)])
def test_linear_decode_wide_rank(qb, m, r):
    """Decode shapes with more than one 64-column group of the rank, and a
    partial last group: the in-kernel LoRA up-projection loops over the groups."""
    _linear_case(qb, 392, 640, m, r, 16.0, proj=4)


@pytest.mark.parametrize("n,k,m,r", [(392, 320, 300, 16), (256, 512, 257, 64), (136, 192, 520, 72),
                                     (512, 256, 1024, 128)])
def test_linear_prefill_ragged(qb, n, k, m, r):
    _linear_case(qb, n, k, m, r, 16.0, proj=2)


def test_linear_bwd_recomputes_xa(qb):
    _linear_case(qb, 264, 384, 96, 64, 16.0, proj=3, with_xa=False)


def test_linear_llama7b_q_projection_full_size(qb):
    """4096 x 4096 at 8192 tokens (r = 64): Y and dX on 256 sampled token rows,
    dA and dB in full."""
    rng = np.random.Generator(np.random.PCG64(99))
    rows = np.sort(rng.choice(8192, 256, replace=False))
    _linear_case(qb, 4096, 4096, 8192, 64, 16.0, proj=0, rows_sample=rows)


def test_linear_llama65b_gate_projection_full_size(qb):
    """22016 x 8192 (the 65B FFN gate projection of the layer benchmark, same
    seeds) at 8192 tokens, r = 64: Y and dX on 128 sampled token rows, dA and
    dB in full."""
    rng = np.random.Generator(np.random.PCG64(98))
    rows = np.sort(rng.choice(8192, 128, replace=False))
    _linear_case(qb, 22016, 8192, 8192, 64, 16.0, proj=4, rows_sample=rows)


def test_linear_llama65b_down_projection_full_size(qb):
    """8192 x 22016 (the 65B FFN down projection of the layer benchmark) at
    8192 tokens, r = 64: Y and dX on 128 sampled token rows, dA and dB in full."""
    rng = np.random.Generator(np.random.PCG64(97))
    rows = np.sort(rng.choice(8192, 128, replace=False))
    _linear_case(qb, 8192, 22016, 8192, 64, 16.0, proj=6, rows_sample=rows)


def test_linear_llama65b_q_projection_full_size(qb):
    """8192 x 8192 (the 65B attention projections of the layer benchmark) at
    8192 tokens, r = 64: Y and dX on 128 sampled token rows, dA and dB in full."""
    rng = np.random.Generator(np.random.PCG64(96))
    rows = np.sort(rng.choice(8192, 128, replace=False))
    _linear_case(qb, 8192, 8192, 8192, 64, 16.0, proj=0, rows_sample=rows)


@pytest.mark.parametrize("n,k,proj", [(11008, 4096, 4), (4096, 11008, 6)])
def test_linear_llama7b_ffn_full_size(qb, n, k, proj):
    """The LLaMA-7B FFN shapes (gate/up 11008 x 4096, down 4096 x 11008) at 8192
    tokens, r = 64: Y and dX on 128 sampled token rows, dA and dB in full."""
    rng = np.random.Generator(np.random.PCG64(95 + proj))
    rows = np.sort(rng.choice(8192, 128, replace=False))
    _linear_case(qb, n, k, 8192, 64, 16.0, proj=proj, rows_sample=rows)


@pytest.mark.parametrize("n,k", [(22016, 8192), (8192, 22016)])
@pytest.mark.parametrize("m", [1, 4, 16])
def test_linear_gemv_65b_ffn(qb, n, k, m):
    """The decode-shaped forward on the 65B FFN weights (22016 x 8192 and
    8192 x 22016) at 1, 4 and 16 tokens, r = 64: every output compared."""
    _linear_case(qb, n, k, m, 64, 16.0, proj=5 if n > k else 6, check_bwd=False)


@pytest.mark.parametrize("n,k,m", [(22016, 8192, 1024), (392, 640, 300), (4096, 4096, 16)])
def test_results_are_bit_reproducible(qb, n, k, m):
    """The split contractions sum their partial tiles in a fixed order, so two
    identical calls give the same bits (outputs poisoned in between):
    Y, X A^T, dA, dB always, and dX with more than 16 tokens."""
    qt, _ = _oracle_weight(n, k, 2)
    up = _upload_oracle_quant(qb, qt)
    X, A = workloads.activations(m, k, 2).cuda(), workloads.lora_a(64, k, 2).cuda()
    B, dY = workloads.lora_b(n, 64, 2).cuda(), workloads.grad_output(m, n, 2).cuda()
    runs = []
    for _ in range(2):
        Y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        XA = torch.full((m, 64), float("nan"), dtype=torch.float32, device="cuda")
        qb.qlora_linear_fwd(up, X, A, B, 0.25, Y=Y, XA=XA)
        dX, dA, dB = qb.qlora_linear_bwd(up, X, dY, A, B, 0.25, XA=XA)
        xa_again = qb.qlora_linear_bwd(up, X, dY, A, B, 0.25, XA=None, need_dx=False)  # X A^T recomputed
        torch.cuda.synchronize()
        runs.append([t.cpu().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)
                     for t in (Y, XA, dA, dB, dX, xa_again[1], xa_again[2])])
    assert qb.qlora_read_device_errors() == 0
    names = ["Y", "XA", "dA", "dB", "dX", "dA (X A^T recomputed)", "dB (X A^T recomputed)"]
    for name, a, b in zip(names, runs[0], runs[1]):
        if name == "dX" and m <= 16:
            continue                                  # split-K fp32 atomics at 16 tokens or fewer
        assert torch.equal(a, b), f"{name} differs between two identical calls ({n}x{k}, m={m})"


@pytest.mark.parametrize("m", [64, 8])
def test_codes_at_a_16_byte_offset_give_identical_results(qb, m):
    """The fused kernel takes its code tiles by TMA straight from the code
    array; an array at a 16-byte offset (the least alignment the ABI accepts)
    gives the same bits as an aligned one, forward and backward."""
    import dataclasses
    n, k, r = 392, 640, 64
    W = workloads.weight((n, k), proj=3).cuda()
    qt = qb.qlora_quantize_nf4_dq(W)
    base = torch.empty(qt.codes.numel() + 32, dtype=torch.uint8, device="cuda")
    off = 16 - base.data_ptr() % 32 if base.data_ptr() % 32 <= 16 else 48 - base.data_ptr() % 32
    codes16 = base[off:off + qt.codes.numel()]
    assert codes16.data_ptr() % 32 == 16
    codes16.copy_(qt.codes)
    qt16 = dataclasses.replace(qt, codes=codes16)
    X = workloads.activations(m, k, 3).cuda()
    dY = workloads.grad_output(m, n, 3).cuda()
    A, B = workloads.lora_a(r, k, 3).cuda(), workloads.lora_b(n, r, 3).cuda()
    outs = []
    for t in (qt, qt16):
        Y, XA = qb.qlora_linear_fwd(t, X, A, B, 0.25)
        dX, dA, dB = qb.qlora_linear_bwd(t, X, dY, A, B, 0.25, XA=XA)
        outs.append((Y, dX, dA, dB))
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    for a, b, name in zip(outs[0], outs[1], ("Y", "dX", "dA", "dB")):
        assert torch.equal(a, b), name
