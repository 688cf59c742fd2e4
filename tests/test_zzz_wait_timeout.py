"""The device error path: a bounded wait that nothing completes gives up after its limit,
sets MLA_DEVERR_TIMEOUT in the error word the host reads, and leaves the context usable.
No fault, trap or hang: the wait is the same bounded mbarrier wait every kernel uses."""
import time

import pytest
import torch

import head_latent_attention_attn_b200 as mla
from mla_inputs import CONFIGS, make_workload
from tests.gpu_harness import GpuProblem, check_sequence

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    mla.mla_selftest_wait_timeout(err)
    status = mla.mla_get_device_status(err, reset=True)
    elapsed = time.time() - t0
    assert status == mla.MLA_ERR_DEVICE_TIMEOUT
    assert 1.0 <= elapsed < 60.0, elapsed          # the wait ran out after its 2 s limit
    assert mla.mla_get_device_status(err) == mla.MLA_OK   # the word was cleared
    # the context still works: a decode step matches the oracle
    prob = GpuProblem(make_workload(CONFIGS["tiny"]))
    prob.step()
    torch.cuda.synchronize()
    assert prob.device_status() == mla.MLA_OK
    check_sequence(prob, 0, "after the timeout self-test")
