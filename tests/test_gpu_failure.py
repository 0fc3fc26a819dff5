"""Failure detection on the GPU without a fault.

Every pipelined kernel bounds its mbarrier waits by the global timer and, when
one runs out, records MSA_ERR_TIMEOUT in the device status word instead of
hanging.  msa_check_bounded_wait runs that path alone: a wait that nothing
completes must end after about its limit with the timeout recorded, and the
context must stay usable for the next call.  No fault, trap or endless loop
is involved.
"""

import numpy as np
import pytest
import torch

import oracle
from latent_memory_routing_b200 import msa, pipeline

pytestmark = pytest.mark.gpu

TIMEOUT = -5


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from latent_memory_routing_b200 import build
    build.build()
    msa.lib()
    msa.msa_device_status(clear=True)
    yield
    torch.cuda.synchronize()
    msa.msa_device_status(clear=True)


def test_completed_wait_records_nothing():
    msa.msa_check_bounded_wait(1_000_000, True)
    assert msa.msa_device_status(clear=True) == 0


@pytest.mark.parametrize("limit_ns", [20_000, 2_000_000])
def test_expired_wait_records_timeout_and_context_stays_usable(limit_ns):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    msa.msa_check_bounded_wait(limit_ns, False)
    e1.record()
    torch.cuda.synchronize()
    assert msa.msa_device_status(clear=True) == TIMEOUT
    ms = e0.elapsed_time(e1)
    # the wait gives up only after its limit, and not much later
    assert 0.9 * limit_ns * 1e-6 <= ms < 1000.0, ms
    # the next call runs normally and records nothing
    g = torch.Generator(device="cuda").manual_seed(5)
    s = torch.rand((2, 1000), generator=g, device="cuda")
    idx, _ = pipeline.topk_docs(s, 8)
    torch.cuda.synchronize()
    assert msa.msa_device_status(clear=True) == 0
    want, _ = oracle.topk_docs(s.double().cpu().numpy(), 8)
    np.testing.assert_array_equal(idx.cpu().numpy(), want)


def test_timeout_is_kept_until_read():
    """The status word keeps the first device-detected error: later clean
    calls do not overwrite it, and reading with clear resets it."""
    msa.msa_check_bounded_wait(20_000, False)
    msa.msa_check_bounded_wait(20_000, True)
    assert msa.msa_device_status(clear=False) == TIMEOUT
    assert msa.msa_device_status(clear=True) == TIMEOUT
    assert msa.msa_device_status(clear=True) == 0
