"""Failure detection on the GPU, without any GPU fault.

Every device-side wait of the library is bounded; a wait that gives up writes a timeout code
into the handle's device status word and its kernel returns. Here a wait is made to run out
on purpose (gqe_selftest_timeout: a barrier phase that nothing completes, the same bounded
wait the pipeline kernels use), and the test checks that the host sees GQE_ERR_TIMEOUT, that
reading the status clears it, and that the handle and context stay usable: a forward after
the timeout equals one before it, bit for bit.
"""
import numpy as np
import pytest
import torch

from moe_query_head_b200 import workloads as W
from tests.gqe_testlib import GpuRun

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    from moe_query_head_b200 import gqe as G
    run = GpuRun(W.generate(W.WORKLOADS["main_b8_t2048"].with_(B=1, T=300))).forward()
    before = run.out.clone()
    G.gqe_selftest_timeout(run.h, 1000)
    assert G.gqe_check_device_status(run.h) == G.GQE_ERR_TIMEOUT
    assert G.gqe_check_device_status(run.h) == G.GQE_OK  # the check cleared the word
    run.out.fill_(float("nan"))
    run.forward()  # asserts the status is OK again
    torch.cuda.synchronize()
    assert torch.equal(run.out, before)
    run.close()


def test_selftest_rejects_bad_arguments():
    from moe_query_head_b200 import gqe as G
    with pytest.raises(G.GQEError) as e:
        G.gqe_selftest_timeout(None, 10)
    assert e.value.status == G.GQE_ERR_INVALID_ARG
