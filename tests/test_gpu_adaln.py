"""GPU parity of the quantiser with the fused adaLN prologue (nvfp4_adaln_quantize through the C ABI)
against the oracle's fp64 RMSNorm + modulation.

The kernel sums squares in fp32, so its rstd and its bf16 u may differ from the oracle's in the last
bit: rstd is compared within a relative 4e-6, u within the error that allows, and the codes and
scales within one step wherever an input differs.  Exact, bit for bit: the fused codes equal the
library's plain quantiser applied to the kernel's own u, and a row's result does not depend on the
rows around it.
"""
import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O
from tests.helpers import assert_quant_arrays_close, f32, gpu_qtensor_bytes

pytestmark = pytest.mark.gpu


def run_gpu(case, dynamic=True, g=None, with_shift=True, with_scale=True):
    x = case.x.cuda()
    M, C = case.x.shape
    shift = case.shift.cuda() if with_shift else None
    scale = case.scale.cuda() if with_scale else None
    if shift is not None and case.rows_per_sample == 0:
        shift = shift[0]
    if scale is not None and case.rows_per_sample == 0:
        scale = scale[0]
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    u = torch.empty((M, C), dtype=torch.bfloat16, device="cuda")
    q = B.adaln_quantize(x, shift, scale, eps=case.eps, rows_per_sample=case.rows_per_sample,
                         g=None if dynamic else g, rstd=rstd, u_out=u)
    torch.cuda.synchronize()
    return q, rstd.cpu().numpy().astype(np.float64), f32(u)


def run_oracle(case, rows=None, g=None, with_shift=True, with_scale=True):
    x = f32(case.x) if rows is None else f32(case.x[rows])
    sh = f32(case.shift) if with_shift else None
    sc = f32(case.scale) if with_scale else None
    L = case.rows_per_sample
    if rows is not None and L:
        raise ValueError("sampled rows use one sample")
    q, ub, rstd = O.adaln_quantize(x, sh, sc, case.eps, L, g)
    u64, _ = O.adaln_modulate(x, sh, sc, case.eps, L)
    # magnitude of the product term, which bounds the fp32 error of x * rstd * (1 + scale)
    mult = 1.0 + (np.zeros_like(x, dtype=np.float64) if sc is None else
                  np.asarray(sc, np.float64).reshape(-1, x.shape[1])[(np.arange(x.shape[0]) // L) if L else 0])
    prod = np.abs(np.asarray(x, np.float64) * rstd[:, None] * mult)
    return q, ub, rstd, u64, prod


def bf16_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_u(u_gpu, ub, u64, prod, max_frac=2e-3):
    """Each bf16 u within the fp32 error (rstd to 2e-6, two roundings) plus half a bf16 step of the exact
    value, and different from the oracle's rounding in at most max_frac of the elements."""
    err = 2e-6 * prod + 1.2e-7 * np.abs(u64)
    assert np.all(np.abs(u_gpu - u64) <= err + 0.5 * bf16_ulp(np.abs(u64) + err))
    assert np.mean(u_gpu != ub) <= max_frac, np.mean(u_gpu != ub)


def gpu_rows(q, M, K, rows=None):
    codes, scales, g = gpu_qtensor_bytes(q)
    c = O.unpack_codes(codes)
    s = O.scales_from_mma_layout(scales, M, K)
    if rows is not None:
        c, s = c[rows], s[rows]
    return c, s, g


def check_fused_equals_plain_quantiser(q, u_gpu_bf16, M, K):
    """The fused codes are the library's own quantiser run on the kernel's u, with the same g."""
    plain = B.quantize(u_gpu_bf16, g=q.g.clone())
    torch.cuda.synchronize()
    assert torch.equal(plain.codes, q.codes)
    assert torch.equal(plain.scales, q.scales)       # padding rows and blocks included


CASES = [
    # rows, cols, seed, samples: 1 step, ragged steps, a whole 4608-wide row in registers, a 4624-wide
    # row (a one-lane tail step past the registers), 6144 (the re-read path), per-sample vectors
    (1, 16, 0, 1), (5, 48, 1, 1), (130, 208, 2, 1), (129, 4608, 3, 1), (40, 4624, 4, 1), (33, 6144, 5, 1),
    (300, 4608, 6, 3),
]


@pytest.mark.parametrize("M,C,seed,samples", CASES)
def test_adaln_quantize_dynamic_scale(lib, M, C, seed, samples):
    case = W.case_adaln(M, C, samples=samples, seed=seed)
    if M > 3:
        case.x[2] = 0                                     # a zero row normalises to 0: u = shift
    q, rstd, u = run_gpu(case)
    (rc, rs, rg), ub, rstd_ref, u64, prod = run_oracle(case)
    np.testing.assert_allclose(rstd, rstd_ref, rtol=4e-6)
    check_u(u, ub, u64, prod)
    got = gpu_rows(q, M, C)
    if got[2] == rg:
        assert_quant_arrays_close(got, (rc, rs, rg))
    else:
        # the tensor max itself rounded the other way: g one bf16 step apart, codes checked against u
        assert abs(float(got[2]) - float(rg)) <= float(bf16_ulp(rg * 2688.0)) / 2688.0 * 1.01
        deq = O.dequantize_exact(*got)
        d = O.e4m3_decode(got[1]) * np.float64(got[2])
        assert np.all(np.abs(deq - u).reshape(M, -1, 16).max(axis=2) <= d * (1 + 1e-6) +
                      np.maximum(np.abs(u).reshape(M, -1, 16).max(axis=2) - 6 * d, 0))
    check_fused_equals_plain_quantiser(q, torch.from_numpy(u).to(torch.bfloat16).cuda(), M, C)


@pytest.mark.parametrize("with_shift,with_scale", [(True, False), (False, True), (False, False)])
def test_adaln_quantize_static_scale_optional_vectors(lib, with_shift, with_scale):
    M, C = 70, 1024
    case = W.case_adaln(M, C, seed=11)
    g = np.float32(0.002)
    q, rstd, u = run_gpu(case, dynamic=False, g=float(g), with_shift=with_shift, with_scale=with_scale)
    (rc, rs, rg), ub, rstd_ref, u64, prod = run_oracle(case, g=g, with_shift=with_shift, with_scale=with_scale)
    np.testing.assert_allclose(rstd, rstd_ref, rtol=4e-6)
    check_u(u, ub, u64, prod)
    assert_quant_arrays_close(gpu_rows(q, M, C), (rc, rs, rg))
    check_fused_equals_plain_quantiser(q, torch.from_numpy(u).to(torch.bfloat16).cuda(), M, C)


def test_adaln_rows_do_not_depend_on_their_neighbours(lib):
    """Rows [0, 100) quantised alone and inside a 300-row call give the same bytes (static g)."""
    case = W.case_adaln(300, 4608, seed=12)
    x = case.x.cuda()
    sh, sc = case.shift[0].cuda(), case.scale[0].cuda()
    full = B.adaln_quantize(x, sh, sc, g=0.003)
    part = B.adaln_quantize(x[:100], sh, sc, g=0.003)
    torch.cuda.synchronize()
    assert torch.equal(full.codes[:100], part.codes)
    a = gpu_rows(full, 300, 4608, rows=np.arange(100))
    b = gpu_rows(part, 100, 4608)
    assert np.array_equal(a[1], b[1])


def test_adaln_quantize_empty_rows(lib):
    """rows == 0: nothing is encoded and the dynamic scale is 1.  Called through the C ABI with real
    buffers (torch reports a null data pointer for a tensor with no elements)."""
    import ctypes
    x = torch.empty((1, 512), dtype=torch.bfloat16, device="cuda")
    codes = torch.empty((1, 256), dtype=torch.uint8, device="cuda")
    scales = torch.empty(512, dtype=torch.uint8, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    t = B.CTensor(codes.data_ptr(), scales.data_ptr(), g.data_ptr(), 0, 512, 256)
    d = B.CAdaln(None, None, 512, 0, 1e-6, None, None, 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.nvfp4_adaln_quantize(x.data_ptr(), 0, 512, 512, ctypes.byref(d), 1, ctypes.byref(t), stream) == B.OK
    torch.cuda.synchronize()
    assert g.item() == 1.0


def test_adaln_full_size_sampled_rows(lib):
    """The bench's tensor [16896, 4608], dynamic scale: g from the oracle's max over every row (computed in
    row chunks), then 64 sampled rows compared one by one."""
    case = W.adaln_2k()
    M, C = case.x.shape
    q, rstd, u = run_gpu(case)
    best, best_rows = -1.0, None
    for r0 in range(0, M, 2048):
        rows = np.arange(r0, min(M, r0 + 2048))
        u64, _ = O.adaln_modulate(f32(case.x[rows]), f32(case.shift), f32(case.scale), case.eps)
        m = float(np.max(np.abs(O.to_bf16_round(u64))))
        if m > best:
            best, best_rows = m, rows
    u64, _ = O.adaln_modulate(f32(case.x[best_rows]), f32(case.shift), f32(case.scale), case.eps)
    g_ref = O.tensor_scale(O.to_bf16_round(u64))
    rows = np.sort(np.random.default_rng(0).choice(M, 64, replace=False))
    (rc, rs, rg), ub, rstd_ref, u64, prod = run_oracle(case, rows=rows, g=g_ref)
    np.testing.assert_allclose(rstd[rows], rstd_ref, rtol=4e-6)
    check_u(u[rows], ub, u64, prod)
    assert_quant_arrays_close(gpu_rows(q, M, C, rows=rows), (rc, rs, rg))
