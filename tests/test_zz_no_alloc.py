"""The allocation-free split-K entry point (gemm_relu_splitk_noalloc).

Callers that cannot allocate device memory while they run (an arena that owns
all of it, a fixed footprint after start-up) use this entry point instead of
gemm_relu: its fp32 partial sums live in a static device array inside the
library.  These tests call it through the C ABI and compare it with the
existing entry point (gemm_relu) on the same inputs, within the parity
tolerance, on two calls in a row.  The file is collected last so that a run
that stops at the first failure has already run every other test.
"""
from __future__ import annotations

import pytest
import torch

import tiled_tensor_core_04_b200 as g
from tests.parity_util import check_close
from tiled_tensor_core_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu

F16, BF16, F32 = torch.float16, torch.bfloat16, torch.float32


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    g.load()


def _pair(M, N, K, din, dout, trans_b, split_k, seed):
    A, B = wl.make_inputs(M, N, K, din, trans_b, "uniform", seed)
    A, B = A.cuda(), B.cuda()
    want = torch.empty((M, N), dtype=dout, device="cuda")
    got = torch.full((M, N), float("nan"), dtype=dout, device="cuda")
    g.gemm_relu_ex(A, B, want, M, N, K, din, dout, trans_b, True,
                   options={"split_k": split_k} if split_k else None)
    g.gemm_relu_splitk_noalloc(A, B, got, M, N, K, din, dout, trans_b, True, split_k)
    torch.cuda.synchronize()
    assert g.gemm_relu_last_device_error()[0] == g.GEMM_OK
    return got, want


def test_two_calls_in_a_row_match_gemm_relu():
    # skinny split-K shapes of the benchmark set: 4 x 64 x 8192 and 2 x 16 x 16384 fp32
    # partials (8 MiB and 2 MiB) fit the 16 MiB array
    for (M, N, K, split, seed) in [(64, 8192, 8192, 0, 4), (16, 16384, 4096, 0, 5)]:
        got, want = _pair(M, N, K, F16, F16, False, split, seed)
        ref = want.double().cpu().numpy()
        check_close(got.cpu(), ref, F16, True, f"no-alloc {M}x{N}x{K}")


@pytest.mark.parametrize("trans_b", [False, True])
@pytest.mark.parametrize("dout", [F16, BF16, F32])
def test_matches_gemm_relu_across_dtypes(trans_b, dout):
    for call in range(2):
        got, want = _pair(300, 520, 1000, BF16 if dout == F32 else F16, dout, trans_b, 3,
                          seed=10 + call)
        check_close(got.cpu(), want.double().cpu().numpy(), dout, True, f"call {call}")


def test_does_not_grow_device_memory():
    A, B = wl.make_inputs(64, 8192, 8192, F16, False, "uniform", 4)
    A, B = A.cuda(), B.cuda()
    C = torch.empty((64, 8192), dtype=F16, device="cuda")
    g.gemm_relu_splitk_noalloc(A, B, C, 64, 8192, 8192, F16, F16, False, True, 4)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        g.gemm_relu_splitk_noalloc(A, B, C, 64, 8192, 8192, F16, F16, False, True, 4)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free0 - free1 < 4 * 64 * 8192 * 4  # no workspace of the partials' size appeared


def test_refuses_what_would_need_memory():
    A = torch.zeros((1024, 4096), dtype=F16, device="cuda")
    B = torch.zeros((4096, 2048), dtype=F16, device="cuda")
    C = torch.zeros((1024, 2048), dtype=F16, device="cuda")
    # 4 splits x 1024 x 2048 x 4 bytes = 32 MiB of partials > 16 MiB
    assert g.gemm_relu_splitk_noalloc(A, B, C, 1024, 2048, 4096, F16, F16, False, True, 4,
                                      check=False) == g.GEMM_ERR_INVALID_ARG
    # a 2-byte offset base would have to be re-pitched into memory
    Ab = torch.zeros(64 * 512 + 1, dtype=F16, device="cuda")
    assert g.gemm_relu_splitk_noalloc(Ab[1:], B[:512], C[:64], 64, 2048, 512, F16, F16, False,
                                      True, 2, check=False) == g.GEMM_ERR_MISALIGNED
    assert g.NOALLOC_SCRATCH_BYTES == 16 * 1024 * 1024
