"""Parity of the benchmarked configuration: the DiT-block linear set at 2048^2 (16896 tokens = 16384 image
+ 512 text, hidden 4608, seed 7), run exactly as bench.py times it (``bench.BlockSet.step``):

    dynamic quantise -> QKV [13824 x 4608] + bias + q/k head RMSNorm
    dynamic quantise -> out-proj [4608 x 4608] + bias
    dynamic quantise -> up [24576 x 4608] + gated SiLU, re-quantised to NVFP4 in the epilogue
    (that NVFP4 output) -> down [4608 x 12288] + residual + per-channel gate

Rows of a linear are independent ("Faster Ideogram 4 with Less Prompt Compute", "Most of the Tensor Was
Zero"), so the oracle evaluates sampled rows only, each with all its columns, on its own quantisation of
the same seeded inputs; the tensor scale of each activation still comes from the whole tensor.  The rows
include both sides of every 128-row tile boundary (and so of every 256-row CTA-pair tile).  The up
projection's NVFP4 output is quantised with the static decode scale the bench calibrates once; that scale
is a parameter of the operation ("the caller's static decode scale"), given to both sides alike.
"""
import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O
from tests.helpers import assert_close, f32

pytestmark = pytest.mark.gpu

TOL = 2e-2


def block_rows(M, n_random=24, seed=3):
    edges = np.arange(128, M, 128)
    rng = np.random.default_rng(seed)
    rows = np.concatenate([[0, M - 1], edges - 1, edges, rng.choice(M, n_random, replace=False)])
    return np.unique(rows).astype(np.int64)


def gpu_rows_of(q: B.QTensor, rows, M, K):
    """(codes one per byte [R, K], scales [R, K/16], g) of the given rows of a GPU NVFP4 tensor."""
    torch.cuda.synchronize()
    idx = torch.from_numpy(rows).cuda()
    codes = O.unpack_codes(q.codes.index_select(0, idx).cpu().numpy())
    scales = O.scales_from_mma_layout(q.scales.cpu().numpy(), M, K)[rows]
    return codes, scales, np.float32(q.g.cpu().item())


@pytest.fixture(scope="module")
def block():
    """One bench step on the GPU; the sampled rows of every output and NVFP4 activation, moved to the host."""
    import bench
    bs = bench.BlockSet()
    bs.step()
    torch.cuda.synchronize()
    B.check_device_error()
    M = bs.M
    rows = block_rows(M)
    idx = torch.from_numpy(rows).cuda()
    got = {k: f32(bs.out[k].index_select(0, idx)) for k in ("qkv", "out", "down")}
    aq = {k: gpu_rows_of(bs.aq[k], rows, M, W.HIDDEN) for k in ("qkv", "out", "up")}
    up_q = gpu_rows_of(bs.up_q, rows, M, W.FFN)
    data = dict(M=M, rows=rows, got=got, aq=aq, up_q=up_q, cases=bs.cases)
    del bs
    torch.cuda.empty_cache()
    return data


def oracle_activation(case, rows):
    """The oracle's quantisation of the sampled rows of an activation, with the whole tensor's scale."""
    x = f32(case.x)
    g = O.tensor_scale(x)
    return O.quantize(x[rows], g)


def assert_quant_rows_equal(got, ref, what):
    gc, gs, gg = got
    rc, rs, rg = ref
    assert gg == rg, f"{what}: tensor scale {gg} != {rg}"
    assert np.array_equal(gs, rs), f"{what}: {np.count_nonzero(gs != rs)} block scales differ"
    assert np.array_equal(gc, rc), f"{what}: {np.count_nonzero(gc != rc)} codes differ"


def test_block2k_qkv_headnorm(block):
    case = block["cases"]["qkv"]
    rows = block["rows"]
    a_ref = oracle_activation(case, rows)
    assert_quant_rows_equal(block["aq"]["qkv"], a_ref, "x_qkv quantisation")
    ex = case.extras
    ref = O.linear(a_ref, O.quantize(f32(case.w)), "qknorm", bias=f32(case.bias), gamma_q=f32(ex["gamma_q"]),
                   gamma_k=f32(ex["gamma_k"]), eps=ex["eps"], q_col0=ex["q_col0"], k_col0=ex["k_col0"],
                   qk_cols=ex["qk_cols"], head_dim=ex["head_dim"])["y"]
    got = block["got"]["qkv"]
    assert_close(got, ref, "block 2048^2 QKV")
    H = W.HIDDEN
    for name, c0 in (("q", 0), ("k", H), ("v", 2 * H)):
        assert_close(got[:, c0:c0 + H], ref[:, c0:c0 + H], f"block 2048^2 QKV, {name} range")


def test_block2k_out_projection(block):
    case = block["cases"]["out"]
    rows = block["rows"]
    a_ref = oracle_activation(case, rows)
    assert_quant_rows_equal(block["aq"]["out"], a_ref, "x_attn quantisation")
    ref = O.linear(a_ref, O.quantize(f32(case.w)), "bias", bias=f32(case.bias))["y"]
    assert_close(block["got"]["out"], ref, "block 2048^2 out-proj")


def test_block2k_ffn_up_requant_then_down(block):
    """Up with gated SiLU and the fused NVFP4 re-quantisation, then down on each side's own NVFP4 output."""
    up, down = block["cases"]["up"], block["cases"]["down"]
    rows = block["rows"]
    a_ref = oracle_activation(up, rows)
    assert_quant_rows_equal(block["aq"]["up"], a_ref, "x_ffn quantisation")
    gc, gs, g_out = block["up_q"]
    r_up = O.linear(a_ref, O.quantize(f32(up.w)), "gated_silu", out_g=g_out)
    # the calibrated static scale covers the sampled outputs (it came from the whole output's max)
    assert float(np.max(np.abs(r_up["bf16"]))) <= float(g_out) * 2688.0 * (1 + TOL)
    rc, rs, rg = r_up["q"]
    assert rg == g_out
    # the fused re-quantisation against the oracle's re-quantisation of its own bf16 output: the two bf16
    # outputs may differ in the last bit, which can move a scale by one E4M3 step or a code by one step
    ds = np.abs(gs.astype(np.int64) - rs.astype(np.int64))
    assert ds.max() <= 1 and np.mean(ds > 0) <= 1e-3, (ds.max(), np.mean(ds > 0))
    mag = lambda c: np.where(c & 8, -(c & 7), c & 7)
    dc = np.where(np.repeat(ds == 0, 16, axis=1), np.abs(mag(gc.astype(np.int64)) - mag(rc.astype(np.int64))), 0)
    assert dc.max() <= 1 and np.mean(dc > 0) <= 1e-3, (dc.max(), np.mean(dc > 0))
    # every dequantised NVFP4 output lies within one grid step of the oracle's fp64 gated SiLU: the E2M1
    # grid steps are at most 2 units of the block's decode scale d = e4m3(s) * g
    d = (O.e4m3_decode(gs).astype(np.float64) * np.float64(g_out))
    err = np.abs(O.dequantize(gc, gs, g_out).astype(np.float64) - r_up["y"])
    bound = np.repeat(2.0 * d, 16, axis=1) + TOL * np.abs(r_up["y"]) + 1e-30
    assert np.all(err <= bound), f"up NVFP4 output off by more than a grid step at {np.argwhere(err > bound)[:3]}"
    del r_up
    ex = down.extras
    ref = O.linear((rc, rs, rg), O.quantize(f32(down.w)), "resid_gate", residual=f32(ex["residual"])[rows],
                   gate=ex["gate"].numpy())["y"]
    assert_close(block["got"]["down"], ref, "block 2048^2 down")
