"""The kernels' bounded waits, made to run out on purpose (on a B200).

Every mbarrier wait in the library's kernels has a bound; when it runs out the kernel records
GDR_ERR_TIMEOUT in the device error word, releases its tensor memory and returns, so the
context stays usable.  gdr_debug_wait_timeout runs one CTA that waits, with a short bound, on
an mbarrier that nothing ever arrives at (no copy or MMA in flight).  The test checks that the
kernel returns, that the error word reports the timeout and is cleared by reading it, and that
the library's kernels (which allocate tensor memory too) still run and match afterwards.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_63_b200 as G
import gdr_inputs as GI
from tests.test_gpu_parity import check_core

pytestmark = pytest.mark.gpu

GDR_ERR_TIMEOUT = 8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    G.lib()
    assert G.get_device_error() == 0


@pytest.mark.parametrize("kind,limit", [(0, 1000), (1, 200_000)], ids=["poll-bound", "clock-bound"])
def test_a_wait_that_runs_out_reports_a_timeout_and_returns(kind, limit):
    verdict = G.debug_wait_timeout(kind, limit)     # .item() synchronises: the kernel returned
    assert verdict == 0
    assert G.get_device_error() == GDR_ERR_TIMEOUT
    assert G.get_device_error() == 0                # reading clears the word
    # tensor memory was released: the prefill (which allocates it) still runs and matches
    check_core(GI.make_core_inputs(93, [70, 5], prenorm_qk=False, h0_std=0.02))
    assert G.get_device_error() == 0
