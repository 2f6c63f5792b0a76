"""The allocation-free quantize entry point, called through the C ABI.

qlora_quantize_nf4_dq_noalloc serves callers that cannot allocate device
memory at quantize time (a server that fixed its memory at start-up, code
inside another framework's allocator or out-of-memory path, a loader with no
allocator): it uses a scratch array compiled into the library instead of a
caller-supplied work buffer.  Its output must equal the ordinary entry point's
byte for byte (codes, E4M3 constants, c2, mean), call after call, with the
shared scratch left over from the previous call.

This file is collected last on purpose, and it passes both on its own in a
fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qb():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_nf4_quantized_encode_b200 as m
    return m


def _stored(t, nbytes_codes, nblocks, ngroups):
    return (t.codes[:nbytes_codes].cpu().numpy(), t.absmax_q[:nblocks].cpu().numpy(),
            t.absmax_c2[:ngroups].cpu().numpy().view(np.uint32),
            t.absmax_mean[:1].cpu().numpy().view(np.uint32))


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(qb):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # a large call, then a smaller ragged one, then the large one again: each
    # must be unaffected by what the previous call left in the shared scratch
    cases = [((4096, 4096), 0, True), ((300, 4160), 1, False), ((4096, 4096), 2, True)]
    for shape, proj, outl in cases:
        w = workloads.weight(shape, proj=proj, outliers=outl).cuda()
        rows, cols = shape
        sz = qb.qlora_nf4_sizes(rows, cols)
        ngroups = sz["absmax_c2"] // 4
        ref = qb.qlora_quantize_nf4_dq(w, out=qb.empty_nf4(rows, cols, w.device))
        got = qb.empty_nf4(rows, cols, w.device)
        for t in (got.codes, got.absmax_q):
            t.fill_(0xA5)                       # poison: every byte must be rewritten
        got.absmax_c2.fill_(float("nan"))
        c = got.c_struct()
        launches0 = qb.qlora_kernel_launches()
        st = qb._lib.qlora_quantize_nf4_dq_noalloc(ctypes.c_void_p(w.data_ptr()), ctypes.byref(c), stream)
        assert st == 0, qb.qlora_status_string(st)
        # the encoder and the double quantization, counted like every launch
        assert qb.qlora_kernel_launches() - launches0 == 2
        torch.cuda.synchronize()
        assert qb.qlora_read_device_errors() == 0
        a = _stored(ref, sz["codes"], sz["absmax_q"], ngroups)
        b = _stored(got, sz["codes"], sz["absmax_q"], ngroups)
        for name, x, y in zip(("codes", "absmax_q", "absmax_c2", "mean"), a, b):
            assert np.array_equal(x, y), f"{name} differs for shape {shape}"


def test_noalloc_rejects_weights_above_its_scratch(qb):
    limit = qb.NOALLOC_MAX_ELEMENTS
    t = qb._Nf4TensorC(0x10000, 0x20000, 0x30000, 0x40000, 2, limit // 2 + 64, 64, 256)
    st = qb._lib.qlora_quantize_nf4_dq_noalloc(ctypes.c_void_p(0x50000), ctypes.byref(t), None)
    assert qb.qlora_status_string(st) == "work buffer too small"
    ok = qb._Nf4TensorC(0x10000, 0x20000, 0x30000, 0x40000, 0, 5, 64, 256)
    assert qb._lib.qlora_quantize_nf4_dq_noalloc(None, ctypes.byref(ok), None) == 0   # empty: no-op
