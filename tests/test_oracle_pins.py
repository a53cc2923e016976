"""Pins for the CPU oracle, against things other than the oracle itself.

Each test ties one oracle function to a closed form, a library routine
(ml_dtypes' float4_e2m1fn / float8_e4m3fn / bfloat16 casts, numpy fp64 matmul),
exact rational arithmetic, brute force on tiny inputs, or sizes the pages print.
The pins are chosen so that a plausible slip (a dropped term, a wrong sign or
index, a swapped operand, the wrong tie rule) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

from oracle import nvfp4_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------
# E2M1
# ------------------------------------------------------------------------------------------

def test_e2m1_decode_closed_form():
    # code = s<<3 | e<<1 | m: subnormal (e=0) m * 0.5, normal 2^(e-1) * (1 + m/2)
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        want = -mag if s else mag
        got = O.e2m1_decode(np.array([code]))[0]
        assert got == want and math.copysign(1, got) == math.copysign(1, want) or (mag == 0 and got == 0)


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(O.e2m1_decode(codes), ref)


def test_e2m1_ties_and_saturation():
    table = [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6), (6.0, 7), (7.0, 7),
             (1e30, 7), (-0.25, 8), (-0.1, 8), (-0.0, 8), (0.0, 0), (-5.0, 14), (0.2500001, 1),
             (4.9999995, 6), (5.0000005, 7), (-1e30, 15)]
    v = np.array([t[0] for t in table], dtype=np.float32)
    np.testing.assert_array_equal(O.e2m1_round(v), np.array([t[1] for t in table], np.uint8))


def test_e2m1_round_matches_ml_dtypes():
    rng = np.random.default_rng(1)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 10)])
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 3,
                        rng.uniform(-8, 8, 20000).astype(np.float32), near, -near,
                        np.array([0.0, -0.0, 6.0, -6.0, 100.0, -1e20], np.float32)])
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(O.e2m1_round(v), ref)


# ------------------------------------------------------------------------------------------
# E4M3
# ------------------------------------------------------------------------------------------

def test_e4m3_decode_matches_ml_dtypes():
    b = np.arange(0x7F, dtype=np.uint8)
    ref = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(O.e4m3_decode(b), ref)
    assert O.E4M3_VALUES[-1] == 448.0 and O.E4M3_VALUES[1] == 2.0 ** -9
    assert np.all(np.diff(O.E4M3_VALUES) > 0)


def test_e4m3_round_matches_ml_dtypes_below_464():
    rng = np.random.default_rng(2)
    vals = O.E4M3_VALUES.astype(np.float32)
    mids = ((O.E4M3_VALUES[1:] + O.E4M3_VALUES[:-1]) / 2).astype(np.float32)
    x = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
                        np.exp2(rng.uniform(-12, 8.8, 50000)).astype(np.float32),
                        np.array([2.0 ** -10, 2.0 ** -11, 1e-30, 0.0], np.float32)])
    x = x[x < 464]
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(O.e4m3_round_satfinite(x), ref)


def test_e4m3_saturates_at_448():
    x = np.array([448.0, 449.0, 464.0, 480.0, 1e9, 3e38], np.float32)
    assert np.all(O.e4m3_round_satfinite(x) == 0x7E)


# ------------------------------------------------------------------------------------------
# Block rule, brute force in exact rational arithmetic
# ------------------------------------------------------------------------------------------

def f32(q: Fraction) -> Fraction:
    """Round an exact rational to the nearest binary32 value, ties to even (finite range)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    assert Fraction(2) ** e <= a < Fraction(2) ** (e + 1)
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    n = a / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def brute_quantize_block(xs, g):
    """The block rule, step by step, in Fractions with explicit binary32 rounding."""
    g = Fraction(float(g))
    amax = max(abs(Fraction(float(x))) for x in xs)
    r = f32(amax / g)
    s_f = f32(r / 6)
    s_byte = int(np.array([float(s_f)], np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]) \
        if s_f <= 448 else 0x7E
    s_val = Fraction(float(np.array([s_byte], np.uint8).view(ml_dtypes.float8_e4m3fn)[0]))
    d = f32(s_val * g)
    if d == 0:
        return [0] * len(xs), s_byte
    inv = f32(1 / d)
    codes = []
    for x in xs:
        v = f32(Fraction(float(x)) * inv)
        c = int(np.array([float(v)], np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)[0]) & 0xF
        if v == 0 and float(x) < 0 or (v == 0 and math.copysign(1, float(x)) < 0):
            c = 0x8
        codes.append(c)
    return codes, s_byte


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_quantize_matches_rational_brute_force(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((6, 64)) * np.exp2(rng.integers(-6, 6, (6, 1)))).astype(np.float32)
    x[0, 3] *= 40.0                                   # an outlier that sets the tensor amax
    x[1, 16:32] = 0.0                                 # an all-zero block
    x[2, 32:48] *= 1e-4                               # a block whose scale underflows
    x = x.astype(ml_dtypes.bfloat16).astype(np.float32)
    codes, scales, g = O.quantize(x)
    assert g == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            want_c, want_s = brute_quantize_block(x[r, 16 * b:16 * b + 16], g)
            assert scales[r, b] == want_s, (r, b)
            assert list(codes[r, 16 * b:16 * b + 16]) == want_c, (r, b)


def test_block_with_tensor_amax_gets_scale_448():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 256)).astype(np.float32)
    x[7, 100] = 25.0
    _, scales, _ = O.quantize(x)
    assert scales[7, 100 // 16] in (0x7D, 0x7E)
    assert scales.max() <= 0x7E


def test_dequantize_error_bound():
    # each element is within half a grid step (times d) of its value, except where it saturates at 6*d
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 512)) * 3).astype(np.float32)
    codes, scales, g = O.quantize(x)
    xh = O.dequantize_exact(codes, scales, g)
    d = (O.e4m3_decode(scales) * np.float64(g)).repeat(16, axis=1)
    a = np.abs(x.astype(np.float64)) / d
    step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    err = np.abs(x - xh) / d
    sat = a > 6
    assert np.all(err[~sat] <= step[~sat] / 2 * (1 + 1e-6))
    assert np.all(np.abs(xh[sat]) == 6 * d[sat])


def test_codes_round_trip_through_dequantize():
    # a block holding +-6 at scale s (exact powers of two so every step is exact) re-quantises to itself
    rng = np.random.default_rng(5)
    for s_exp in range(-9, 9):
        codes = rng.integers(0, 16, (4, 32)).astype(np.uint8)
        codes[:, 0] = 0x7
        codes[:, 16] = 0xF
        s = np.full((4, 2), O.e4m3_round_satfinite(np.float32(2.0 ** s_exp)), np.uint8)
        x = O.dequantize(codes, s, np.float32(1.0))
        c2, s2, _ = O.quantize(x, g=np.float32(1.0))
        np.testing.assert_array_equal(s2, s)
        # -0 codes dequantise to +0.0 * d... the sign of a zero survives only through x's sign bit
        np.testing.assert_array_equal(c2 & 0x7, codes & 0x7)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4, 0xF, 0x8]], np.uint8)
    np.testing.assert_array_equal(O.pack_codes(codes), np.array([[0x21, 0x43, 0x8F]], np.uint8))
    np.testing.assert_array_equal(O.unpack_codes(O.pack_codes(codes)), codes)


def test_scale_layout_offsets():
    K = 512  # 32 blocks per row -> 8 atoms along K
    assert O.scale_atom_offset(0, 0, K) == 0
    assert O.scale_atom_offset(0, 1, K) == 1
    assert O.scale_atom_offset(1, 0, K) == 16
    assert O.scale_atom_offset(32, 0, K) == 4
    assert O.scale_atom_offset(96, 3, K) == 12 + 3
    assert O.scale_atom_offset(0, 4, K) == 512
    assert O.scale_atom_offset(128, 0, K) == 512 * 8
    M = 300
    off = O.scale_offsets(M, K)
    assert len(np.unique(off)) == off.size and off.max() < O.scale_buffer_bytes(M, K)
    assert O.scale_buffer_bytes(M, K) == 384 * 32
    for r, c in [(0, 0), (37, 5), (299, 31), (128, 17)]:
        assert off[r, c] == O.scale_atom_offset(r, c, K)
    s = np.random.default_rng(6).integers(0, 127, (M, 32)).astype(np.uint8)
    np.testing.assert_array_equal(O.scales_from_mma_layout(O.scales_to_mma_layout(s), M, K), s)


# ------------------------------------------------------------------------------------------
# GEMM and epilogues
# ------------------------------------------------------------------------------------------

def random_quantised(rng, rows, K, s_lo=0x20, s_hi=0x50):
    codes = rng.integers(0, 16, (rows, K)).astype(np.uint8)
    scales = rng.integers(s_lo, s_hi, (rows, K // 16)).astype(np.uint8)
    return codes, scales


def test_matmul_equals_exact_rational_sum():
    rng = np.random.default_rng(7)
    M, N, K = 5, 6, 64
    ac, asc = random_quantised(rng, M, K)
    wc, wsc = random_quantised(rng, N, K)
    ag, wg = np.float32(0.75), np.float32(1.25)
    got = O.matmul_exact(ac, asc, ag, wc, wsc, wg)
    E2 = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]

    def val(c, s):
        c, s = int(c), int(s)
        e, m = s >> 3, s & 7
        sv = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        v = E2[c & 7] * sv
        return -v if c & 8 else v
    for m in range(M):
        for n in range(N):
            exact = sum(val(ac[m, k], asc[m, k // 16]) * Fraction(float(ag)) *
                        val(wc[n, k], wsc[n, k // 16]) * Fraction(float(wg)) for k in range(K))
            assert abs(Fraction(got[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 60)


def test_matmul_matches_plain_loops_and_transpose_matters():
    rng = np.random.default_rng(8)
    ac, asc = random_quantised(rng, 4, 32)
    wc, wsc = random_quantised(rng, 3, 32)
    a = O.dequantize_exact(ac, asc, np.float32(1))
    w = O.dequantize_exact(wc, wsc, np.float32(1))
    loops = np.array([[sum(a[m, k] * w[n, k] for k in range(32)) for n in range(3)] for m in range(4)])
    np.testing.assert_allclose(O.matmul_exact(ac, asc, 1, wc, wsc, 1), loops, rtol=1e-14)


def test_rmsnorm_closed_forms():
    rng = np.random.default_rng(9)
    y = rng.standard_normal((3, 512)) * 5
    out = O.rmsnorm_heads(y, np.ones(256), 0.0)
    rms = np.sqrt(np.mean(out.reshape(3, 2, 256) ** 2, axis=2))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-12)
    # a head of equal values c maps to sign(c) * gamma; eps enters as sqrt(c^2 + eps)
    y = np.full((1, 256), -3.0)
    g = np.linspace(0.5, 1.5, 256)
    np.testing.assert_allclose(O.rmsnorm_heads(y, g, 0.0)[0], -g, rtol=1e-14)
    np.testing.assert_allclose(O.rmsnorm_heads(y, g, 7.0)[0], -3.0 / 4.0 * g, rtol=1e-14)
    # heads are normalised separately: scaling head 1 leaves head 0 unchanged
    y = rng.standard_normal((2, 512))
    y2 = y.copy(); y2[:, 256:] *= 100
    np.testing.assert_allclose(O.rmsnorm_heads(y, g, 1e-6)[:, :256], O.rmsnorm_heads(y2, g, 1e-6)[:, :256])


def test_qknorm_epilogue_ranges():
    rng = np.random.default_rng(10)
    acc = rng.standard_normal((2, 768 * 3 // 1)) * 4
    bias = rng.standard_normal(acc.shape[1])
    gq, gk = np.full(256, 2.0), np.full(256, 3.0)
    out = O.epilogue(acc, "qknorm", bias=bias, gamma_q=gq, gamma_k=gk, eps=0.0,
                     q_col0=0, k_col0=768, qk_cols=768, head_dim=256)
    y = acc + bias
    for c0, gam in ((0, 2.0), (768, 3.0)):
        h = out[:, c0:c0 + 768].reshape(2, 3, 256)
        np.testing.assert_allclose(np.sqrt(np.mean(h ** 2, axis=2)), gam, rtol=1e-12)
        # bias is added before the norm: the direction of each head is that of acc + bias
        yh = y[:, c0:c0 + 768].reshape(2, 3, 256)
        cos = np.sum(h * yh, axis=2) / np.linalg.norm(h, axis=2) / np.linalg.norm(yh, axis=2)
        np.testing.assert_allclose(cos, 1.0, rtol=1e-12)
    np.testing.assert_allclose(out[:, 1536:], y[:, 1536:])


def test_silu_identities_and_gated_half():
    a = np.linspace(-20, 20, 401)
    np.testing.assert_allclose(O.silu(a) - O.silu(-a), a, atol=1e-12)
    assert O.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(O.silu(np.array([40.0])), 40.0, rtol=1e-15)
    acc = np.concatenate([a[None, :], np.ones((1, 401))], axis=1)
    np.testing.assert_allclose(O.epilogue(acc, "gated_silu")[0], O.silu(a))
    # the first half is the gated one: swapping halves gives a different result
    swapped = np.concatenate([np.ones((1, 401)), a[None, :]], axis=1)
    assert not np.allclose(O.epilogue(swapped, "gated_silu")[0], O.silu(a))


def test_resid_gate_special_cases():
    rng = np.random.default_rng(11)
    acc = rng.standard_normal((4, 32))
    res = rng.standard_normal((4, 32))
    np.testing.assert_array_equal(O.epilogue(acc, "resid_gate", residual=res, gate=np.zeros(32)), res)
    b = rng.standard_normal(32)
    np.testing.assert_allclose(O.epilogue(acc, "resid_gate", bias=b, residual=np.zeros((4, 32)), gate=np.ones(32)),
                               O.epilogue(acc, "bias", bias=b))


def test_bf16_rounding_matches_ml_dtypes():
    rng = np.random.default_rng(12)
    v = (rng.standard_normal(100000) * 10).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(O.to_bf16_round(v), v.astype(ml_dtypes.bfloat16).astype(np.float32))


def test_row_independence_in_oracle():
    # "Most of the Tensor Was Zero": rows are independent, and a zero row projects to the bias.
    rng = np.random.default_rng(13)
    x = rng.standard_t(4, (8, 128)).astype(np.float32)
    w = (rng.standard_normal((64, 128)) * 0.005).astype(np.float32)
    bias = rng.standard_normal(64) * 0.01
    xz = np.concatenate([x, np.zeros((24, 128), np.float32)])
    aq, azq, wq = O.quantize(x), O.quantize(xz), O.quantize(w)
    assert aq[2] == azq[2]                            # zero rows leave amax, hence g, unchanged
    y1 = O.linear(aq, wq, "bias", bias=bias)["bf16"]
    y2 = O.linear(azq, wq, "bias", bias=bias)["bf16"]
    np.testing.assert_array_equal(y1, y2[:8])
    np.testing.assert_array_equal(y2[8:], np.broadcast_to(O.to_bf16_round(bias), (24, 64)))


def test_requant_is_quantize_of_bf16_output():
    rng = np.random.default_rng(14)
    aq = O.quantize(rng.standard_normal((16, 64)).astype(np.float32))
    wq = O.quantize((rng.standard_normal((64, 64)) * 0.1).astype(np.float32))
    out = O.linear(aq, wq, "gated_silu", out_g=np.float32(0.01))
    c, s, g = O.quantize(out["bf16"], np.float32(0.01))
    np.testing.assert_array_equal(out["q"][0], c)
    np.testing.assert_array_equal(out["q"][1], s)


# ------------------------------------------------------------------------------------------
# Sizes printed on the pages pin the workload shapes
# ------------------------------------------------------------------------------------------

def read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, v, unit, _ = [t.strip() for t in line.split("|")]
            rows[k] = (float(v), unit)
    return rows


def test_page_sizes_pin_workload_shapes():
    from epilogue_gemm_nvfp4_b200 import workloads as W
    p = read_golden("page_sizes.txt")
    assert W.IMG_TOKENS_1K + W.PROMPT_T == p["packed_positions_1k"][0]
    assert W.IMG_TOKENS_1K + W.LONG_PROMPT_T == p["long_prompt_positions_1k"][0]
    assert W.HIDDEN == p["hidden_width"][0] and W.TEXT_K == p["text_feature_width"][0]
    assert W.PROMPT_T * W.HIDDEN * 2 / 2 ** 20 == p["cached_text_bf16"][0]
    # two branches (positive, negative) of zero image rows, Qwen width, bf16
    assert 2 * W.IMG_TOKENS_1K * W.TEXT_K * 2 / 2 ** 30 == p["zero_rows_saving_1k"][0]
    assert 2 * W.IMG_TOKENS_2K * W.TEXT_K * 2 / 2 ** 30 == p["zero_rows_saving_2k"][0]
    assert W.N_HEADS * W.HEAD_DIM == W.HIDDEN


# ------------------------------------------------------------------------------------------
# fake quantisation (the forward of training through the quantiser's noise)
# ------------------------------------------------------------------------------------------

def test_fake_quantize_leaves_grid_values_unchanged():
    """Blocks already on the NVFP4 grid (e2m1 codes times one E4M3 value, with a full-scale code in each
    block, tensor scale 1) come back exactly: the round trip's fixed points, by the format's definition."""
    rng = np.random.default_rng(23)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    block_scales = np.array([0.25, 0.5, 1.0, 2.0, 8.0, 16.0])  # exact E4M3 values, 6 * s exact in bf16
    M, K = 8, 64
    x = np.empty((M, K))
    for r in range(M):
        for b in range(K // 16):
            v = grid[rng.integers(0, 8, 16)] * rng.choice([-1.0, 1.0], 16)
            v[rng.integers(0, 16)] = 6.0 * rng.choice([-1.0, 1.0])  # the block's amax is 6 * s
            x[r, 16 * b:16 * b + 16] = v * block_scales[(r + b) % len(block_scales)]
    x = x.astype(np.float32)
    y, g = O.fake_quantize(x, np.float32(1.0))
    assert g == np.float32(1.0)
    np.testing.assert_array_equal(y, x)


def test_fake_quantize_element_rounding_matches_ml_dtypes():
    """Each element is the ml_dtypes E2M1 rounding of x * inv, times d, rounded to bf16: an independent
    statement of the element step, with the block scale from the oracle's own quantiser."""
    rng = np.random.default_rng(29)
    x = (rng.standard_normal((16, 128)) * 3).astype(ml_dtypes.bfloat16).astype(np.float32)
    y, g = O.fake_quantize(x)
    _, scales, _ = O.quantize(x, g)
    d = (O.e4m3_decode(scales).astype(np.float32) * np.float32(g)).astype(np.float32)
    d = np.repeat(d, 16, axis=1)
    inv = np.where(d == 0, np.float32(0), (np.float32(1) / np.where(d == 0, np.float32(1), d)).astype(np.float32))
    v = (x * inv).astype(np.float32)
    e = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
    ref = (e * d).astype(np.float32).astype(ml_dtypes.bfloat16).astype(np.float32)
    np.testing.assert_array_equal(y, ref)


# ------------------------------------------------------------------------------------------
# adaLN prologue (RMSNorm, then (1 + scale) and shift per sample)
# ------------------------------------------------------------------------------------------

def test_adaln_without_modulation_is_torch_rms_norm():
    """scale = shift = 0 reduces the prologue to RMSNorm without a weight: torch's own rms_norm in fp64."""
    import torch
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 96)) * np.array([10.0 ** rng.integers(-3, 3) for _ in range(7)])[:, None]
    for eps in (1e-6, 0.5):
        u, rstd = O.adaln_modulate(x, np.zeros(96), np.zeros(96), eps=eps)
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (96,), eps=eps).numpy()
        np.testing.assert_allclose(u, ref, rtol=1e-13, atol=0)
        np.testing.assert_allclose(x * rstd[:, None], ref, rtol=1e-13, atol=0)


def test_adaln_closed_forms():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 64))
    shift = rng.standard_normal(64)
    # scale = -1 removes the normalised row: u is the shift, whatever x is
    u, _ = O.adaln_modulate(x, shift, -np.ones(64))
    np.testing.assert_array_equal(u, np.broadcast_to(shift, u.shape))
    # a constant row c normalises to c / sqrt(c^2 + eps); (1 + 0.5) * that + 0.25 rounds to bf16 1.75
    c = np.full((2, 32), 2.0)
    c[1] = -2.0
    u, rstd = O.adaln_modulate(c, np.full(32, 0.25), np.full(32, 0.5), eps=1e-6)
    np.testing.assert_allclose(rstd, 1.0 / math.sqrt(4.0 + 1e-6), rtol=1e-15)
    np.testing.assert_array_equal(O.to_bf16_round(u)[0], 1.75)
    np.testing.assert_array_equal(O.to_bf16_round(u)[1], -1.25)    # -1.5 + 0.25: the shift is not scaled
    # mean square of an unmodulated row is ms / (ms + eps)
    u, _ = O.adaln_modulate(x, None, None, eps=0.3)
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.mean(u * u, axis=1), ms / (ms + 0.3), rtol=1e-13)


def test_adaln_is_invariant_to_row_scale_when_eps_vanishes():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 128))
    sh, sc = rng.standard_normal(128), rng.standard_normal(128)
    u1, r1 = O.adaln_modulate(x, sh, sc, eps=1e-30)
    u2, r2 = O.adaln_modulate(x * 1024.0, sh, sc, eps=1e-30)
    np.testing.assert_allclose(u1, u2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r1, r2 * 1024.0, rtol=1e-12)


def test_adaln_sample_of_each_row():
    """rows [b*L, (b+1)*L) take sample b's vectors; L = 0 gives every row sample 0."""
    x = np.random.default_rng(6).standard_normal((7, 16))
    shift = np.arange(1, 4, dtype=np.float64)[:, None] * np.ones((3, 16))
    u, _ = O.adaln_modulate(x, shift, -np.ones((3, 16)), rows_per_sample=3)
    np.testing.assert_array_equal(u[:, 0], [1, 1, 1, 2, 2, 2, 3])
    u, _ = O.adaln_modulate(x, shift, -np.ones((3, 16)), rows_per_sample=0)
    np.testing.assert_array_equal(u[:, 0], np.ones(7))


def test_adaln_quantize_codes_approximate_the_modulated_row():
    """Each dequantised element is within half a code step of the bf16 modulated value (the block rule's
    error bound, with the 6-saturation of the E4M3 rounding allowed for), and g follows from amax(u)."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((33, 256)).astype(np.float32)
    sh, sc = 0.5 * rng.standard_normal(256), 0.5 * rng.standard_normal(256)
    (codes, scales, g), ub, rstd = O.adaln_quantize(x, sh, sc)
    assert g == np.float32(np.max(np.abs(ub)) / np.float32(2688.0))
    d = O.e4m3_decode(scales) * np.float64(g)
    err = np.abs(O.dequantize_exact(codes, scales, g) - ub).reshape(33, 16, 16)
    amax_b = np.abs(ub).reshape(33, 16, 16).max(axis=2)
    bound = np.maximum(d, 0) + np.maximum(amax_b - 6 * d, 0)    # one step of 2 * d at most, or the clip
    assert np.all(err.max(axis=2) <= bound + 1e-12)


# ------------------------------------------------------------------------------------------
# W8A8 INT8 linear
# ------------------------------------------------------------------------------------------

def test_int8_rows_ties_extremes_and_zero_rows():
    # amax 127 gives s = 1 exactly, so the codes are x rounded half to even
    x = np.array([[127.0, 0.5, 1.5, 2.5, -2.5, -0.5, 126.5, -3.49],
                  [0.0] * 8,
                  [-4.0, 1.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    q, s = O.int8_quantize_rows(x)
    assert s[0] == 1.0 and s[1] == 1.0
    assert q[0].tolist() == [127, 0, 2, 2, -2, 0, 126, -3]
    assert q[1].tolist() == [0] * 8
    assert q[2, 0] == -127 and s[2] == np.float32(4.0) / np.float32(127.0)
    assert q[2, 1] == 32                                         # 1 * 127/4 = 31.75 -> 32


def test_int8_rows_within_half_a_step_of_the_exact_quotient():
    """Brute force in exact rationals: every code is a nearest integer to x / s for the fp32 s."""
    rng = np.random.default_rng(9)
    x = (rng.standard_t(3, size=(6, 40)) * 10.0 ** rng.integers(-3, 3, size=(6, 1))).astype(np.float32)
    q, s = O.int8_quantize_rows(x)
    for r in range(6):
        amax = max(abs(Fraction(float(v))) for v in x[r])
        assert abs(Fraction(float(s[r])) - amax / 127) <= Fraction(float(s[r])) * Fraction(1, 2 ** 23)
        for v, c in zip(x[r], q[r]):
            e = abs(Fraction(float(v)) / Fraction(float(s[r])) - int(c))
            assert e <= Fraction(1, 2) + Fraction(1, 2 ** 16), (v, c)
        assert np.max(np.abs(q[r])) == 127


def test_int8_smoothing_divides_each_input_channel():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((4, 32)).astype(np.float32)
    mult = np.ones(32, np.float32)
    mult[5] = 0.25                                               # lambda = 4 for channel 5
    q1, s1 = O.int8_quantize_rows(x, mult)
    x2 = x.copy()
    x2[:, 5] /= 4.0
    q2, s2 = O.int8_quantize_rows(x2)
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


def test_smoothquant_factors_balance_the_channel_ranges():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((48, 32)) * 0.02
    act = np.abs(rng.standard_normal(32)) * 10 + 0.1
    act[3], w[:, 7] = 0.0, 0.0                                  # dead channels keep lambda = 1
    lam = O.smoothquant_factors(act, w, 0.5).astype(np.float64)
    wmax = np.max(np.abs(w), axis=0)
    live = (act > 0) & (wmax > 0)
    # alpha = 1/2 gives the activation and weight columns the same range after the migration
    np.testing.assert_allclose((act / lam)[live], (wmax * lam)[live], rtol=2e-7)
    assert lam[3] == 1.0 and lam[7] == 1.0
    # alpha = 1 moves all of it into the weights, alpha = 0 none of the activations' range
    np.testing.assert_allclose(O.smoothquant_factors(act, w, 1.0)[live], act[live], rtol=1e-7)
    np.testing.assert_allclose(O.smoothquant_factors(act, w, 0.0)[live], 1.0 / wmax[live], rtol=1e-7)
    # and the unquantised product is unchanged: (x / lambda) (W lambda)^T = x W^T
    x = rng.standard_normal((5, 32))
    np.testing.assert_allclose((x / lam) @ (w * lam).T, x @ w.T, rtol=1e-12, atol=1e-15)


def test_int8_linear_exact_integer_product_and_scaling():
    rng = np.random.default_rng(12)
    qa = rng.integers(-127, 128, size=(3, 20)).astype(np.int8)
    qw = rng.integers(-127, 128, size=(4, 20)).astype(np.int8)
    sa = np.array([0.5, 0.01, 3.0], np.float32)
    sw = np.array([0.25, 1e-3, 2.0, 7.0], np.float32)
    bias = np.array([1.0, -1.0, 0.0, 0.5])
    y, yb = O.int8_linear(qa, sa, qw, sw, bias)
    for m in range(3):
        for n in range(4):
            acc = sum(int(qa[m, k]) * int(qw[n, k]) for k in range(20))
            want = Fraction(acc) * Fraction(float(sa[m])) * Fraction(float(sw[n])) + Fraction(bias[n])
            assert abs(Fraction(y[m, n]) - want) <= abs(want) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 60)
    np.testing.assert_array_equal(yb, O.to_bf16_round(y))


def test_w8a8_error_bound():
    """|y - x W^T| <= sum_k (|x| e_w + |w| e_x + e_x e_w), e = half a quantisation step per row."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal((6, 64)).astype(np.float32)
    w = (rng.standard_normal((8, 64)) * 0.05).astype(np.float32)
    qa, sa = O.int8_quantize_rows(x)
    qw, sw = O.int8_quantize_rows(w)
    y, _ = O.int8_linear(qa, sa, qw, sw)
    ex, ew = sa.astype(np.float64)[:, None] / 2, sw.astype(np.float64)[:, None] / 2
    bound = (np.abs(x).astype(np.float64) @ np.ones((64, 8))) * ew.T + ex * (np.ones((6, 64)) @ np.abs(w).T) \
        + 64 * ex * ew.T
    assert np.all(np.abs(y - x.astype(np.float64) @ w.astype(np.float64).T) <= bound * (1 + 1e-6))


def test_adaln_is_equivariant_to_column_permutations():
    """RMSNorm and a per-column modulation commute with any permutation of the columns."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((6, 48))
    sh, sc = rng.standard_normal(48), rng.standard_normal(48)
    p = rng.permutation(48)
    u, r = O.adaln_modulate(x, sh, sc)
    up, rp = O.adaln_modulate(x[:, p], sh[p], sc[p])
    np.testing.assert_allclose(up, u[:, p], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(rp, r, rtol=1e-14)


def test_int8_rows_scale_by_powers_of_two():
    """Multiplying a row by 2^k leaves its codes unchanged and multiplies its scale by 2^k exactly."""
    rng = np.random.default_rng(15)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    q, s = O.int8_quantize_rows(x)
    for k in (-7, 3, 20):
        q2, s2 = O.int8_quantize_rows(x * np.float32(2.0 ** k))
        assert np.array_equal(q2, q)
        assert np.array_equal(s2, (s * np.float32(2.0 ** k)).astype(np.float32))


def test_quantize_scales_by_powers_of_two_with_the_tensor():
    """NVFP4 of 2^k x has the codes and block scales of x and a tensor scale 2^k times larger."""
    rng = np.random.default_rng(16)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    c, s, g = O.quantize(x)
    for k in (-5, 4):
        c2, s2, g2 = O.quantize(x * np.float32(2.0 ** k))
        assert np.array_equal(c2, c) and np.array_equal(s2, s)
        assert g2 == np.float32(g * np.float32(2.0 ** k))
