"""nvfp4_linear_noalloc, the entry point for callers that cannot allocate device memory.

Code that runs while a serving runtime or framework owns all device memory through its own pool, or
on a path where cudaMalloc / cudaFree would synchronise the device, cannot let the library allocate
its split-K scratch.  nvfp4_linear_noalloc keeps that scratch in a fixed device array instead.  These
tests call it through the C ABI on long-K shapes (K >= 32768, where the scratch is used) and check
that two calls in a row give the output of nvfp4_linear bit for bit without allocating device memory,
and that a problem too large for the array is refused before anything is launched.
"""
import ctypes

import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _call(fn, aq, wq, desc, out, q=None):
    ca, cw = aq.c(), wq.c()
    cq = q.c() if q is not None else None
    return fn(ctypes.byref(ca), ctypes.byref(cw), ctypes.byref(desc), ctypes.c_void_p(out.data_ptr()),
              out.stride(0), ctypes.byref(cq) if cq is not None else None,
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("kind,M,N,K", [("bias", 512, 4608, 53248), ("gated_silu", 130, 512, 32768),
                                        ("bias", 300, 4608 + 128, 32768), ("bias", 200, 256, 4608)])
def test_noalloc_matches_linear_on_two_calls(lib, kind, M, N, K):
    """Two calls in a row equal nvfp4_linear bit for bit (both run the same fixed-order split-K).  N = 4736
    takes 128-wide tiles on single CTAs, whose split-K exchange layout differs from the CTA pairs'."""
    if kind == "bias":
        case = W.case_bias(M, N, K, seed=11, w_std=0.005, x_dist="student_t")
    else:
        case = W.case_ffn_up(M, K=K, F=N // 2, seed=12)
    assert B.split_k(N, K, kind) == (2 if K >= 32768 else 1)
    aq, wq = B.quantize(case.x.cuda()), B.quantize(case.w.cuda())
    bias = case.bias.cuda() if case.bias is not None else None
    desc = B.make_epilogue(case.epilogue, bias=bias)
    outs = [torch.full((case.M, case.n_out), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ref = torch.empty(case.M, case.n_out, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    # the first no-alloc call comes first, on a stream the library has never seen (a per-stream scratch
    # buffer would have to be allocated here); a later one runs on a second fresh stream while the device's
    # free memory is watched: nothing may be allocated
    s0, s1 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s0):
        assert _call(lib.nvfp4_linear_noalloc, aq, wq, desc, outs[0]) == B.OK
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    with torch.cuda.stream(s1):
        assert _call(lib.nvfp4_linear_noalloc, aq, wq, desc, outs[1]) == B.OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    B.check_device_error()
    assert _call(lib.nvfp4_linear, aq, wq, desc, ref) == B.OK
    B.check_device_error()
    assert torch.all(torch.isfinite(ref.float()))
    for out in outs:
        assert torch.equal(out, ref)


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
