"""GPU parity of the fused NVFP4 linear (nvfp4_linear through the C ABI) against the oracle.

The oracle runs on its own quantisation of the same seeded bf16 inputs; the GPU quantiser is checked
bit-exact against that quantisation first, so both sides multiply the same NVFP4 operands.  The bar
for GEMM + epilogue outputs (bf16) is a normwise max relative error of 2e-2 and, element by element,
2e-2 of max(|oracle|, 1e-2 * rms(oracle)).  Row independence is checked bitwise on the GPU.
"""
import os

import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O
from tests.helpers import (assert_close, assert_quant_bitexact, assert_requant_close, elementwise_ok, f32,
                           normwise_rel_err, oracle_quantize)

pytestmark = pytest.mark.gpu

TOL = 2e-2


def gpu_epi_kwargs(case):
    ex = case.extras
    if case.epilogue == "qknorm":
        return dict(gamma_q=ex["gamma_q"].cuda(), gamma_k=ex["gamma_k"].cuda(), eps=ex["eps"], q_col0=ex["q_col0"],
                    k_col0=ex["k_col0"], qk_cols=ex["qk_cols"], head_dim=ex["head_dim"])
    if case.epilogue == "resid_gate":
        return dict(residual=ex["residual"].cuda(), gate=ex["gate"].cuda())
    return {}


def oracle_epi_kwargs(case):
    ex = case.extras
    if case.epilogue == "qknorm":
        return dict(gamma_q=f32(ex["gamma_q"]), gamma_k=f32(ex["gamma_k"]), eps=ex["eps"], q_col0=ex["q_col0"],
                    k_col0=ex["k_col0"], qk_cols=ex["qk_cols"], head_dim=ex["head_dim"])
    if case.epilogue == "resid_gate":
        return dict(residual=f32(ex["residual"]), gate=f32(ex["gate"]))
    return {}


def run_gpu(case, aq=None, out_fp4=None, want_bf16=True):
    aq = B.quantize(case.x.cuda()) if aq is None else aq
    wq = B.quantize(case.w.cuda())
    bias = case.bias.cuda() if case.bias is not None else None
    out = B.linear(aq, wq, case.epilogue, bias=bias, out_fp4=out_fp4, want_bf16=want_bf16, **gpu_epi_kwargs(case))
    B.check_device_error()
    return aq, wq, out


def run_oracle(case, rows=None, a_ref=None, w_ref=None, out_g=None):
    a_ref = oracle_quantize(case.x) if a_ref is None else a_ref
    w_ref = oracle_quantize(case.w) if w_ref is None else w_ref
    bias = f32(case.bias) if case.bias is not None else None
    return a_ref, w_ref, O.linear(a_ref, w_ref, case.epilogue, bias=bias, rows=rows, out_g=out_g,
                                  **oracle_epi_kwargs(case))


def check(got, ref, what):
    """Normwise and elementwise parity (helpers.assert_close) at the 2e-2 bar."""
    return assert_close(got, ref, what, TOL)


# ------------------------------------------------------------------------------------------
# small and ragged cases, whole outputs
# ------------------------------------------------------------------------------------------

def test_tiny_workload_full(lib):
    case = W.tiny()
    aq, wq, out = run_gpu(case)
    a_ref, w_ref, ref = run_oracle(case)
    assert_quant_bitexact(aq, a_ref, case.M, case.K)
    assert_quant_bitexact(wq, w_ref, case.N, case.K)
    check(f32(out), ref["y"], "tiny")
    assert elementwise_ok(f32(out), ref["y"]) <= 1.0


@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (127, 384, 320), (129, 256, 512), (300, 512, 1024),
                                   (64, 128, 4608), (257, 768, 192)])
def test_bias_ragged(lib, M, N, K):
    case = W.case_bias(M, N, K, seed=M + N + K, w_std=0.05)
    aq, wq, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], f"bias {M}x{N}x{K}")


def test_no_bias(lib):
    case = W.case_bias(200, 256, 256, seed=3)
    case.bias = None
    _, _, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], "no bias")


@pytest.mark.parametrize("kind", ["bias", "qknorm", "gated_silu", "resid_gate"])
def test_unit_bias_every_epilogue(lib, kind):
    """A bias of standard deviation 1 on every epilogue, against the oracle element by element: a bias that
    is dropped, read from the wrong column block or added after the norm moves outputs by O(1)."""
    M, K = 300, 768
    if kind == "bias":
        case = W.case_bias(M, 640, K, seed=21, w_std=0.05)
    elif kind == "qknorm":
        case = W.case_qkv(M, n_heads=2, K=K, seed=22)
    elif kind == "gated_silu":
        case = W.case_ffn_up(M, K=K, F=384, seed=23)
    else:
        case = W.case_ffn_down(M, N=640, F=K, seed=24)
    case.bias = W.to_bf16(np.random.default_rng(25).standard_normal(case.N).astype(np.float32))
    _, _, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], f"unit bias {kind}")
    if kind == "qknorm":
        # the normalised q and k heads and the bias-only v range each pass on their own
        for c0 in (0, 512, 1024):
            check(f32(out)[:, c0:c0 + 512], ref["y"][:, c0:c0 + 512], f"unit bias qknorm cols {c0}")


@pytest.mark.parametrize("M", [200, 1])
def test_qknorm_small(lib, M):
    case = W.case_qkv(M, n_heads=2, K=512, seed=5)
    _, _, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], "qknorm")
    # the normalised heads have rms ~ |gamma| scale, the v range keeps bias-only values
    got = f32(out)[:, :512].reshape(M, 2, 256)
    assert np.all(np.sqrt(np.mean(got ** 2, axis=2)) < 2.0)


def test_resid_gate_small(lib):
    case = W.case_ffn_down(150, N=384, F=512, seed=6)
    _, _, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], "resid_gate")


@pytest.mark.parametrize("M", [130, 100])
def test_gated_silu_with_requant_small(lib, M):
    # M = 100: on CTA pairs the second CTA's 128-row block lies wholly past M and past the scale
    # layout's padded rows, so it must write nothing
    case = W.case_ffn_up(M, K=512, F=256, seed=7)
    case.bias = W.to_bf16(np.random.default_rng(70).standard_normal(512).astype(np.float32) * 0.01)
    a_ref, w_ref, ref = run_oracle(case)
    g_out = np.float32(np.max(np.abs(ref["bf16"])) / np.float32(2688.0))
    q = B.QTensor.empty(case.M, case.n_out)
    q.g.fill_(float(g_out))
    aq, wq, out = run_gpu(case, out_fp4=q)
    check(f32(out), ref["y"], "gated silu")
    # the fused re-quantisation equals the quantiser applied to the kernel's own bf16 output
    q2 = B.quantize(out, g=float(g_out))
    torch.cuda.synchronize()
    assert torch.equal(q.codes, q2.codes)
    assert torch.equal(q.scales, q2.scales)
    # and it matches the oracle's re-quantisation of its own bf16 output up to one-step differences
    assert_requant_close(q, O.quantize(ref["bf16"], g_out), case.M, case.n_out)
    # fp4-only output (no bf16 written) gives the same codes
    q3 = B.QTensor.empty(case.M, case.n_out)
    q3.g.fill_(float(g_out))
    run_gpu(case, aq=aq, out_fp4=q3, want_bf16=False)
    assert torch.equal(q.codes, q3.codes) and torch.equal(q.scales, q3.scales)


@pytest.mark.parametrize("kind,M,N,K", [("bias", 200, 144, 512), ("bias", 300, 400, 1024), ("resid_gate", 130, 400, 768),
                                        ("bias", 257, 4624, 4608), ("resid_gate", 129, 4624, 1024),
                                        ("bias", 130, 400, 32768)])
def test_ragged_n(lib, kind, M, N, K):
    """N a multiple of 16 but not of 128: 128-wide tiles whose last one reaches past N (the weight's rows
    past N read as zeros, the epilogue reads no bias, residual or gate there, the stores are clipped)."""
    assert B.tile_n(N, K, kind) == 128
    if kind == "bias":
        case = W.case_bias(M, N, K, seed=N + K, w_std=0.02 if K < 32768 else 0.005,
                           x_dist="student_t" if K >= 32768 else "normal")
        case.bias = W.to_bf16(np.random.default_rng(N).standard_normal(N).astype(np.float32))
    else:
        case = W.case_ffn_down(M, N=N, F=K, seed=N + K)
    _, _, out = run_gpu(case)
    assert out.shape == (M, N)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], f"ragged N {kind} {M}x{N}x{K}")


def test_ragged_n_requant_and_amax(lib):
    """The NVFP4 output and the output amax of a ragged-N bias GEMM: the fused codes equal nvfp4_quantize
    of the kernel's own bf16 output bit for bit, padding scale bytes included (the last tile's blocks past
    N land in the row's 4-block padding or past it), and the amax is the bf16 output's."""
    M, N, K = 300, 400, 512
    case = W.case_bias(M, N, K, seed=41, w_std=0.05)
    aq, wq = B.quantize(case.x.cuda()), B.quantize(case.w.cuda())
    bias = case.bias.cuda()
    out = B.linear(aq, wq, "bias", bias=bias)
    g_out = bf16_absmax(out) / 2688.0
    # GEMM NVFP4 outputs need 16-byte code rows: 400 columns are 200 bytes, so the rows are padded to 208
    codes = torch.zeros(M, 208, dtype=torch.uint8, device="cuda")[:, : N // 2]
    q = B.QTensor(codes, torch.full((B.scale_bytes(M, N),), 0x55, dtype=torch.uint8, device="cuda"),
                  torch.full((1,), g_out, dtype=torch.float32, device="cuda"), M, N)
    # (the scales start as 0x55: the fused requant must write every scale byte, padding included, as the
    # quantiser does)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    out2 = B.linear(aq, wq, "bias", bias=bias, out_fp4=q, out_amax=amax)
    B.check_device_error()
    assert torch.equal(out, out2)
    q2 = B.quantize(out, g=g_out)
    torch.cuda.synchronize()
    assert torch.equal(q.codes, q2.codes) and torch.equal(q.scales, q2.scales)
    assert float(amax.item()) == bf16_absmax(out)


def test_tile_n_128_path_and_k_tail(lib):
    # N = 384 forces 128-wide tiles (two TMEM accumulators); K = 320 leaves a one-MMA tail stage
    case = W.case_bias(515, 384, 320, seed=9, w_std=0.05)
    assert B.tile_n(384, 320, "bias") == 128
    _, _, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], "bn128")


@pytest.mark.parametrize("kind,M,N", [("bias", 130, 256), ("bias", 257, 384), ("resid_gate", 129, 256),
                                      ("gated_silu", 131, 512)])
def test_split_k_long_reduction(lib, kind, M, N):
    """K >= 32768 runs as two K halves whose fp32 partials are summed before the epilogue."""
    K = 32768
    assert B.split_k(N, K, kind) == 2 and B.split_k(N, 4608, kind) == 1 and B.split_k(13824, K, "qknorm") == 1
    if kind == "bias":
        case = W.case_bias(M, N, K, seed=M, w_std=0.01, x_dist="student_t")
    elif kind == "resid_gate":
        case = W.case_ffn_down(M, N=N, F=K, seed=M)
    else:
        case = W.case_ffn_up(M, K=K, F=N // 2, seed=M)
    aq, wq, out = run_gpu(case)
    _, _, ref = run_oracle(case)
    check(f32(out), ref["y"], f"split-K {kind}")
    # which K half finishes first varies from run to run; the result may not
    bias = case.bias.cuda() if case.bias is not None else None
    for _ in range(3):
        again = B.linear(aq, wq, case.epilogue, bias=bias, **gpu_epi_kwargs(case))
        B.check_device_error()
        assert torch.equal(again, out)


# ------------------------------------------------------------------------------------------
# row independence (bitwise, on the GPU)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("T", [512, 1941])
def test_row_independence_text_projection(lib, T):
    """The T text rows project identically with or without the 4096 zero image rows appended, and
    each zero row projects to exactly the bias ("Most of the Tensor Was Zero")."""
    base = W.text_proj(T)
    padded = W.text_proj(T, zero_rows=W.IMG_TOKENS_1K)
    assert torch.equal(padded.x[:T], base.x)
    wq = B.quantize(base.w.cuda())
    bias = base.bias.cuda()
    a1 = B.quantize(base.x.cuda())
    a2 = B.quantize(padded.x.cuda())
    assert a1.g.item() == a2.g.item()
    o1 = B.linear(a1, wq, "bias", bias=bias)
    o2 = B.linear(a2, wq, "bias", bias=bias)
    B.check_device_error()
    assert torch.equal(o1, o2[:T])
    assert torch.equal(o2[T:], bias.expand(W.IMG_TOKENS_1K, -1))


# ------------------------------------------------------------------------------------------
# full-size workloads: every GPU output against the oracle on sampled rows
# ------------------------------------------------------------------------------------------

def sample_rows(M, n=48, seed=0):
    """Random rows plus both sides of every 128-row tile boundary (the 256-row pair tiles' included)."""
    rng = np.random.default_rng(seed)
    edges = np.arange(128, M, 128)
    fixed = np.concatenate([[0, 1, M // 2, M - 1], edges - 1, edges])
    rows = np.unique(np.concatenate([fixed[(fixed >= 0) & (fixed < M)], rng.choice(M, min(n, M), replace=False)]))
    return rows.astype(np.int64)


def test_qkv_1k_sampled(lib):
    case = W.qkv_1k()
    aq, wq, out = run_gpu(case)
    rows = sample_rows(case.M)
    a_ref = oracle_quantize(case.x)
    w_ref = oracle_quantize(case.w)
    assert_quant_bitexact(aq, a_ref, case.M, case.K)
    _, _, ref = run_oracle(case, rows=rows, a_ref=a_ref, w_ref=w_ref)
    check(f32(out)[rows], ref["y"], "qkv 1024^2")


def test_ffn_1k_chain_sampled(lib):
    up, down = W.ffn_1k()
    rows = sample_rows(up.M, n=32, seed=1)
    a_ref = oracle_quantize(up.x)
    w_up = oracle_quantize(up.w)
    _, _, r_up = run_oracle(up, rows=rows, a_ref=a_ref, w_ref=w_up)
    g_out = np.float32(np.max(np.abs(r_up["bf16"])) / np.float32(2688.0))
    q = B.QTensor.empty(up.M, up.n_out)
    q.g.fill_(float(g_out))
    _, _, out_up = run_gpu(up, out_fp4=q)
    check(f32(out_up)[rows], r_up["y"], "ffn up")
    # down projection consumes each side's own fused NVFP4 output
    res = f32(down.extras["residual"])[rows]
    gate = f32(down.extras["gate"])
    oq = O.quantize(r_up["bf16"], g_out)
    w_dn = oracle_quantize(down.w)
    r_dn = O.linear(oq, w_dn, "resid_gate", residual=res, gate=gate)
    wq_dn = B.quantize(down.w.cuda())
    out_dn = B.linear(q, wq_dn, "resid_gate", residual=down.extras["residual"].cuda(), gate=down.extras["gate"].cuda())
    B.check_device_error()
    check(f32(out_dn)[rows], r_dn["y"], "ffn down")


@pytest.mark.parametrize("T", [512, 1941])
def test_text_projection_sampled(lib, T):
    case = W.text_proj(T)
    aq, wq, out = run_gpu(case)
    rows = np.arange(T) if T == 512 else sample_rows(T, n=40, seed=2)
    _, _, ref = run_oracle(case, rows=rows)
    check(f32(out)[rows], ref["y"], f"text T={T}")


def test_one_cta_and_pair_kernels_agree(lib, tmp_path):
    """256-wide tiles run on CTA pairs by default; NVFP4_GEMM_PAIR=0 selects the one-CTA kernel.
    Both follow the oracle, and they give the same bits: the K order of every output is the same."""
    import subprocess
    import sys
    script = tmp_path / "one_cta.py"
    out_path = tmp_path / "one_cta.npy"
    script.write_text(
        "import sys, numpy as np, torch\n"
        f"sys.path.insert(0, {repr(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))})\n"
        "from tests.test_gpu_linear import run_gpu, f32\n"
        "from epilogue_gemm_nvfp4_b200 import workloads as W\n"
        "case = W.case_qkv(300, n_heads=2, K=768, seed=11)\n"
        "_, _, out = run_gpu(case)\n"
        f"np.save({repr(str(out_path))}, f32(out))\n")
    env = dict(os.environ, NVFP4_GEMM_PAIR="0")
    subprocess.run([sys.executable, str(script)], check=True, env=env, timeout=300)
    one = np.load(out_path)
    case = W.case_qkv(300, n_heads=2, K=768, seed=11)
    _, _, out = run_gpu(case)
    pair = f32(out)
    _, _, ref = run_oracle(case)
    check(one, ref["y"], "one-CTA kernel")
    check(pair, ref["y"], "pair kernel")
    assert np.array_equal(one, pair)


# ------------------------------------------------------------------------------------------
# fused output amax (delayed scale of the next call's requant)
# ------------------------------------------------------------------------------------------

def bf16_absmax(t):
    return float(t.float().abs().max().item())


@pytest.mark.parametrize("M", [300, 129])
def test_out_amax_equals_max_of_bf16_output(lib, M):
    case = W.case_bias(M, 512, 768, seed=M, w_std=0.05)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    aq = B.quantize(case.x.cuda())
    wq = B.quantize(case.w.cuda())
    out = B.linear(aq, wq, "bias", bias=case.bias.cuda(), out_amax=amax)
    B.check_device_error()
    assert float(amax.item()) == bf16_absmax(out)
    _, _, ref = run_oracle(case)
    assert abs(float(amax.item()) - float(np.max(np.abs(ref["y"])))) <= TOL * float(np.max(np.abs(ref["y"])))


def test_out_amax_with_fp4_only_output(lib):
    case = W.case_ffn_up(300, K=512, F=256, seed=8)
    aq = B.quantize(case.x.cuda())
    wq = B.quantize(case.w.cuda())
    bf16_out = B.linear(aq, wq, "gated_silu")
    q = B.QTensor.empty(300, 256)
    q.g.fill_(bf16_absmax(bf16_out) / 2688.0)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    B.linear(aq, wq, "gated_silu", out_fp4=q, want_bf16=False, out_amax=amax)
    B.check_device_error()
    assert float(amax.item()) == bf16_absmax(bf16_out)
    # the delayed scale is the one the quantiser computes for the same output
    q2 = B.quantize(bf16_out)
    torch.cuda.synchronize()
    assert float(q2.g.item()) == np.float32(np.float32(amax.item()) / np.float32(2688.0))


def test_out_amax_ignores_rows_past_m(lib):
    # x = 1 and w = -50/256 quantise to full-scale codes (block scale 448), so every real output is
    # acc * alpha + bias = -50 + 50 up to the rounding of the fp32 tensor scales (|y| ~ 1e-5); the
    # tile's rows past M (zero A rows) would read the bias alone, 50
    M, N, K = 100, 256, 256
    x = torch.ones(M, K, dtype=torch.bfloat16, device="cuda")
    w = torch.full((N, K), -50.0 / 256.0, dtype=torch.bfloat16, device="cuda")
    bias = torch.full((N,), 50.0, dtype=torch.bfloat16, device="cuda")
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    out = B.linear(B.quantize(x), B.quantize(w), "bias", bias=bias, out_amax=amax)
    B.check_device_error()
    assert bf16_absmax(out) < 1e-3
    assert float(amax.item()) == bf16_absmax(out)


def test_cuda_graph_capture_and_replay(lib):
    """Dynamic-scale quantise + fused linear captured in a CUDA graph replays to the eager bits.  The
    first dynamic quantise on a stream allocates that stream's reduction state, so it runs eagerly on
    the capture stream before the capture."""
    case = W.case_qkv(300, n_heads=2, K=512, seed=12)
    x = case.x.cuda()
    wq = B.quantize(case.w.cuda())
    bias = case.bias.cuda()
    aq = B.QTensor.empty(300, 512)
    out = torch.empty(300, case.n_out, dtype=torch.bfloat16, device="cuda")
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    epi = gpu_epi_kwargs(case)

    def run():
        B.quantize(x, out=aq)
        B.linear(aq, wq, "qknorm", bias=bias, out=out, out_amax=amax, **epi)

    cs = torch.cuda.Stream()
    with torch.cuda.stream(cs):
        run()
    cs.synchronize()
    B.check_device_error()
    eager, eager_codes, eager_g = out.clone(), aq.codes.clone(), aq.g.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        run()
    for _ in range(2):
        out.zero_()
        aq.codes.zero_()
        amax.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
        assert torch.equal(aq.codes, eager_codes) and torch.equal(aq.g, eager_g)
        assert float(amax.item()) == bf16_absmax(eager)
    B.check_device_error()
