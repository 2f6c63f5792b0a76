"""Failure detection on the GPU without a GPU fault.

Every mbarrier wait in the library's pipelines is bounded: a wait that runs
past its limit records "wait timed out" (bit 0) in the device error flag and
lets the kernel return, so a logic error ends in a status instead of a hang.
Here a one-CTA self-test kernel waits, with a short limit, on an mbarrier that
nothing arrives on -- no copy, MMA or other CTA is involved -- and the test
checks that the wait gave up, that the flag reports it through
qlora_read_device_errors, and that the context still runs the hot path.
"""
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


def test_bounded_wait_gives_up_and_reports(qb):
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors(clear=True) == 0
    outcome = torch.zeros(4, dtype=torch.int32, device="cuda")
    qb.qlora_selftest_bounded_wait(100000, outcome)        # about 50 us of SM cycles
    torch.cuda.synchronize()
    assert int(outcome[0].item()) == 1, "the wait on a barrier nothing arrives on must give up"
    flags = qb.qlora_read_device_errors(clear=True)
    assert flags & 1, f"the timed-out wait must set bit 0 of the device error flag (flags {flags:#x})"
    assert qb.qlora_read_device_errors(clear=False) == 0, "clearing the flag must reset it"


def test_context_usable_after_the_timed_out_wait(qb):
    qb.qlora_selftest_bounded_wait(1000)
    torch.cuda.synchronize()
    qb.qlora_read_device_errors(clear=True)
    w = workloads.weight((256, 256))
    qt = qb.qlora_quantize_nf4_dq(w.cuda())
    X, A, B = (workloads.activations(16, 256).cuda(), workloads.lora_a(8, 256).cuda(),
               workloads.lora_b(256, 8).cuda())
    Y, _ = qb.qlora_linear_fwd(qt, X, A, B, 2.0)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    assert np.all(np.isfinite(Y.float().cpu().numpy()))
