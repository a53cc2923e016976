"""GPU parity of the W8A8 INT8 path through the C ABI: the per-row quantiser must equal the oracle byte for
byte; the linear's integer products are exact, so its output differs from the oracle's fp64 value only by
the fp32 scaling and the bf16 rounding (half a bf16 step plus a few fp32 roundings), except where the
epilogue itself approximates (the fast exponential and division of the gated SiLU, the head norm's
reciprocal square root)."""
import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O
from tests.helpers import f32

pytestmark = pytest.mark.gpu

F32 = np.float32


def gpu_i8(t: B.Int8Tensor):
    torch.cuda.synchronize()
    return t.q.cpu().numpy(), t.scale[: t.rows].cpu().numpy()


def bf16_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_close(got, ref_y, scale_terms, what):
    """|got - y| <= half a bf16 step of y plus 8 fp32 roundings of the terms that formed it."""
    bound = 0.5 * bf16_ulp(ref_y) + 8 * 2.0 ** -24 * scale_terms + 1e-30
    bad = np.argwhere(np.abs(got - ref_y) > bound * (1 + 1e-6))
    assert bad.size == 0, f"{what}: {len(bad)} elements off, first {bad[:3].tolist()}"


@pytest.mark.parametrize("rows,cols,seed,mult", [(1, 16, 0, False), (5, 48, 1, True), (130, 208, 2, False),
                                                 (129, 4608, 3, True), (33, 6144, 4, True)])
def test_int8_quantize_bitexact(lib, rows, cols, seed, mult):
    rng = np.random.default_rng(seed)
    x = W.to_bf16(W.with_outlier_columns(rng, W.normal(rng, (rows, cols)), max(1, cols // 100), 30.0))
    if rows > 3:
        x[2] = 0
    m = (rng.uniform(0.25, 4.0, size=cols)).astype(F32) if mult else None
    t = B.int8_quantize(x.cuda(), torch.from_numpy(m).cuda() if m is not None else None)
    q, s = gpu_i8(t)
    rq, rs = O.int8_quantize_rows(f32(x), m)
    assert np.array_equal(s, rs), np.flatnonzero(s != rs)[:5]
    assert np.array_equal(q, rq), np.argwhere(q != rq)[:5]


def run_linear(M, N, K, kind="bias", seed=0, bias=True, **ex_gpu):
    rng = np.random.default_rng(seed)
    x = W.to_bf16(W.normal(rng, (M, K)))
    w = W.to_bf16(W.normal(rng, (N, K), 0.02))
    b = W.to_bf16(W.normal(rng, (N,), 0.01)) if bias else None
    a8, w8 = B.int8_quantize(x.cuda()), B.int8_quantize(w.cuda())
    out = B.int8_linear(a8, w8, kind, bias=b.cuda() if b is not None else None, **ex_gpu)
    torch.cuda.synchronize()
    qa, sa = O.int8_quantize_rows(f32(x))
    qw, sw = O.int8_quantize_rows(f32(w))
    return out, (qa, sa, qw, sw), (f32(b) if b is not None else None)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (130, 384, 96), (300, 512, 4608), (257, 256, 12288)])
def test_int8_linear_bias(lib, M, N, K):
    out, (qa, sa, qw, sw), b = run_linear(M, N, K)
    y, _ = O.int8_linear(qa, sa, qw, sw, b)
    terms = np.abs(y) + (np.abs(b)[None, :] if b is not None else 0)
    check_close(f32(out).astype(np.float64), y, terms, "bias")


def test_int8_linear_resid_gate(lib):
    M, N, K = 200, 512, 1024
    rng = np.random.default_rng(5)
    res = W.to_bf16(W.normal(rng, (M, N)))
    gate = torch.from_numpy(W.uniform(rng, (N,), 0.0, 1.0))
    out, (qa, sa, qw, sw), _ = run_linear(M, N, K, "resid_gate", seed=6, bias=False, residual=res.cuda(),
                                          gate=gate.cuda())
    y, _ = O.int8_linear(qa, sa, qw, sw)
    ref = O.epilogue(y, "resid_gate", residual=f32(res), gate=gate.numpy())
    check_close(f32(out).astype(np.float64), ref, np.abs(ref) + np.abs(f32(res)), "resid_gate")


def test_int8_linear_qknorm_and_gated_silu(lib):
    """Nonlinear epilogues: within 3e-3 normwise of the oracle (fast exponential, division and reciprocal
    square root in the epilogue)."""
    M, K = 130, 512
    rng = np.random.default_rng(7)
    gq, gk = W.to_bf16(W.uniform(rng, (256,), 0.5, 1.5)), W.to_bf16(W.uniform(rng, (256,), 0.5, 1.5))
    ex = dict(gamma_q=gq.cuda(), gamma_k=gk.cuda(), eps=1e-6, q_col0=0, k_col0=256, qk_cols=256, head_dim=256)
    out, (qa, sa, qw, sw), b = run_linear(M, 768, K, "qknorm", seed=8, **ex)
    y, _ = O.int8_linear(qa, sa, qw, sw, b)
    ref = O.epilogue(y, "qknorm", eps=1e-6, q_col0=0, k_col0=256, qk_cols=256, head_dim=256, gamma_q=f32(gq),
                     gamma_k=f32(gk))
    assert O.rel_err_normwise(f32(out), ref) <= 3e-3
    out, (qa, sa, qw, sw), b = run_linear(M, 512, K, "gated_silu", seed=9)
    y, _ = O.int8_linear(qa, sa, qw, sw, b)
    ref = O.epilogue(y, "gated_silu")
    assert O.rel_err_normwise(f32(out), ref) <= 3e-3


def test_w8a8_smoothquant_recipe(lib):
    """The recipe end to end: lambda from the activations' channel maxima (alpha = 0.5), activations scaled
    by 1/lambda and weights by lambda before their per-row INT8 quantisation; the quantised operands equal
    the oracle's byte for byte, and the output stays close to the unquantised product."""
    M, N, K = 256, 512, 1024
    rng = np.random.default_rng(11)
    xf = W.with_outlier_columns(rng, W.normal(rng, (M, K)), 10, 30.0)
    x, w = W.to_bf16(xf), W.to_bf16(W.normal(rng, (N, K), 0.02))
    lam = O.smoothquant_factors(np.max(np.abs(f32(x)), axis=0), f32(w), 0.5)
    inv_lam = (F32(1.0) / lam).astype(F32)
    a8 = B.int8_quantize(x.cuda(), torch.from_numpy(inv_lam).cuda())
    w8 = B.int8_quantize(w.cuda(), torch.from_numpy(lam).cuda())
    out = B.int8_linear(a8, w8, "bias")
    qa, sa = O.int8_quantize_rows(f32(x), inv_lam)
    qw, sw = O.int8_quantize_rows(f32(w), lam)
    ga, gw = gpu_i8(a8), gpu_i8(w8)
    assert np.array_equal(ga[0], qa) and np.array_equal(ga[1], sa)
    assert np.array_equal(gw[0], qw) and np.array_equal(gw[1], sw)
    y, _ = O.int8_linear(qa, sa, qw, sw)
    check_close(f32(out).astype(np.float64), y, np.abs(y), "smoothquant")
    exact = f32(x).astype(np.float64) @ f32(w).astype(np.float64).T
    assert O.rel_err_normwise(f32(out), exact) <= 2e-2


def test_int8_rows_do_not_depend_on_m(lib):
    rng = np.random.default_rng(12)
    x = W.to_bf16(W.normal(rng, (700, 1024)))
    w = B.int8_quantize(W.to_bf16(W.normal(rng, (512, 1024), 0.02)).cuda())
    full = B.int8_linear(B.int8_quantize(x.cuda()), w, "bias")
    part = B.int8_linear(B.int8_quantize(x[:100].cuda()), w, "bias")
    torch.cuda.synchronize()
    assert torch.equal(full[:100], part)
