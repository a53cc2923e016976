"""nvfp4_linear_noalloc, the entry point for callers that cannot allocate device memory.

Code that runs while a serving runtime or framework owns all device memory through its own pool, or
on a path where cudaMalloc / cudaFree would synchronise the device, cannot let the library allocate
its split-K scratch.  nvfp4_linear_noalloc keeps that scratch in a fixed device array instead.  These
tests call it through the C ABI on long-K shapes (K >= 32768, where the scratch is used) and check
that two calls in a row give the output of nvfp4_linear within the parity tolerance, and that a
problem too large for the array is refused before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _call(fn, aq, wq, desc, out, q=None):
    ca, cw = aq.c(), wq.c()
    cq = q.c() if q is not None else None
    return fn(ctypes.byref(ca), ctypes.byref(cw), ctypes.byref(desc), ctypes.c_void_p(out.data_ptr()),
              out.stride(0), ctypes.byref(cq) if cq is not None else None,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("kind,M,N,K", [("bias", 512, 4608, 53248), ("gated_silu", 130, 512, 32768),
                                        ("bias", 200, 256, 4608)])
def test_noalloc_matches_linear_on_two_calls(lib, kind, M, N, K):
    if kind == "bias":
        case = W.case_bias(M, N, K, seed=11, w_std=0.005, x_dist="student_t")
    else:
        case = W.case_ffn_up(M, K=K, F=N // 2, seed=12)
    aq, wq = B.quantize(case.x.cuda()), B.quantize(case.w.cuda())
    bias = case.bias.cuda() if case.bias is not None else None
    desc = B.make_epilogue(case.epilogue, bias=bias)
    ref = torch.empty(case.M, case.n_out, dtype=torch.bfloat16, device="cuda")
    assert _call(lib.nvfp4_linear, aq, wq, desc, ref) == B.OK
    B.check_device_error()
    want = ref.float().cpu().numpy()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _call(lib.nvfp4_linear_noalloc, aq, wq, desc, out) == B.OK
        B.check_device_error()
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert O.rel_err_normwise(got, want) <= TOL


def test_noalloc_refuses_problems_larger_than_its_array(lib):
    limit = int(lib.nvfp4_linear_noalloc_scratch_bytes())
    assert limit == 64 << 20
    # 8192 x 4608 output tiles of 128 x 256 need 1152 * 128 KiB of split-K scratch (> 64 MiB)
    M, N, K = 8192, 4608, 53248
    assert B.split_k(N, K, "bias") == 2
    aq, wq = B.QTensor.empty(M, K), B.QTensor.empty(N, K)
    out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    desc = B.make_epilogue("bias")
    assert _call(lib.nvfp4_linear_noalloc, aq, wq, desc, out) == B.ERR_SCRATCH_LIMIT
    assert B.status_string(B.ERR_SCRATCH_LIMIT).startswith("split-K scratch")
    assert B.get_device_error() == B.OK
