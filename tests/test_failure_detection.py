"""Failure detection without a GPU fault.

The kernels bound every mbarrier wait.  The self-test launches a warp that
waits on a barrier nothing ever arrives on (the "flag that nothing sets");
the wait must run out after the given limit, report GEMM_ERR_TIMEOUT through
the sticky device error word, and leave the CUDA context usable.
"""
from __future__ import annotations

import time

import pytest
import torch

import oracle
import tiled_tensor_core_04_b200 as g
from tests.parity_util import check_close
from tiled_tensor_core_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    g.load()


def test_bounded_wait_runs_out_and_reports():
    assert g.gemm_relu_last_device_error()[0] == g.GEMM_OK       # start clean
    t0 = time.perf_counter()
    st = g.gemm_relu_selftest_timeout(20_000_000)                 # 20 ms limit
    elapsed = time.perf_counter() - t0
    assert st == g.GEMM_ERR_TIMEOUT
    assert elapsed < 5.0
    st, detail = g.gemm_relu_last_device_error()
    assert st == g.GEMM_ERR_TIMEOUT and detail == 32              # the self-test bit
    assert g.gemm_relu_last_device_error() == (g.GEMM_OK, 0)      # read clears it


def test_context_still_usable_after_a_timeout():
    assert g.gemm_relu_selftest_timeout(5_000_000) == g.GEMM_ERR_TIMEOUT
    g.gemm_relu_last_device_error()
    A, B = wl.make_inputs(300, 264, 200, torch.float16, False, "uniform", seed=1)
    C = g.matmul_relu(A.cuda(), B.cuda())
    torch.cuda.synchronize()
    assert g.gemm_relu_last_device_error()[0] == g.GEMM_OK
    check_close(C.cpu(), oracle.gemm_relu(A, B), torch.float16, True, "after timeout")


def test_selftest_rejects_bad_limits():
    assert g.gemm_relu_selftest_timeout(0) == g.GEMM_ERR_INVALID_ARG
    assert g.gemm_relu_selftest_timeout(10 ** 12) == g.GEMM_ERR_INVALID_ARG
