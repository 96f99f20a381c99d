"""The measured tile / hint choice (autotune) on the GPU: every option it may
return is a parity-tested setting; here the tuned call itself is checked
against the oracle, and the per-shape cache is checked to measure only once."""
import pytest
import torch

import oracle
import tiled_tensor_core_04_b200 as g
from tiled_tensor_core_04_b200 import autotune as at
from tiled_tensor_core_04_b200 import workloads as wl
from parity_util import check_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,trans_b", [(600, 1100, 700, False), (520, 900, 640, True),
                                           (48, 3000, 1500, False)])
def test_tuned_options_are_exact_and_cached(M, N, K, trans_b):
    A, B = wl.make_inputs(M, N, K, torch.float16, trans_b, "uniform", seed=M + N)
    Ad, Bd = A.cuda(), B.cuda()
    C = torch.empty(M, N, dtype=torch.float16, device="cuda")
    before = at.tune_calls
    opts = at.tuned_options(Ad, Bd, C, M, N, K, torch.float16, torch.float16, trans_b,
                            iters=3, warmup=1)
    measured = at.tune_calls - before
    assert measured == len(at.candidates(M, N, K, torch.float16, torch.float16, trans_b,
                                         torch.cuda.get_device_properties(0).multi_processor_count))
    again = at.tuned_options(Ad, Bd, C, M, N, K, torch.float16, torch.float16, trans_b)
    assert again == opts and at.tune_calls - before == measured      # served from the cache
    C.fill_(float("nan"))
    g.gemm_relu_ex(Ad, Bd, C, M, N, K, torch.float16, torch.float16, trans_b, True, options=opts)
    torch.cuda.synchronize()
    check_close(C.cpu(), oracle.gemm_relu(A, B, trans_b=trans_b), torch.float16, True,
                f"tuned {opts}")
