"""CPU oracle for the NVFP4 linear layer with fused epilogues.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, table or
constant generator with the CUDA library; the two meet only in the seeded
input generator, which holds none of the method's arithmetic.

What the method computes comes from "Serving sub-second Ideogram v4 without
quality loss": every forward pass of the DiT runs its big matrix products in
NVFP4, a 4-bit floating-point format with native Blackwell support, and each
product is followed by a small op (RMSNorm over 256-wide attention heads, a
gated SiLU) that is fused into the same kernel so the product never makes a
round trip through memory.  "Faster Ideogram 4 with Less Prompt Compute"
adds the text-conditioning projection (a linear with a bias, section "Most of
the Tensor Was Zero") and the requirement that a linear treat rows
independently (sections "Most of the Tensor Was Zero" and "The NF4 Exactness
Problem").

The pages never spell out the NVFP4 encoding.  The oracle follows the plainest
reading that the rest supports, stated once here and listed in the design notes:

  * E2M1 element codes: sign bit 3, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} for
    codes 0..7; rounding is to the nearest magnitude, ties to the even code,
    saturating at 6; the sign is kept, so a negative input that rounds to zero
    gives code 0x8.
  * One unsigned E4M3 scale per 16 consecutive elements of a row (bias 7, max
    448, subnormals down to 2^-9), rounded to nearest-even and saturated at 448.
  * One fp32 per-tensor decode scale g = amax / (6 * 448) (g = 1 when amax = 0).
  * Block rule, each step one IEEE binary32 operation rounded to nearest even:
    r = amax_b / g; s_f = r / 6; s = E4M3(s_f); d = float(s) * g;
    if d == 0 all codes are 0, else inv = 1 / d and code_i = E2M1(x_i * inv).
  * Dequantised value = e2m1(code) * d.  The GEMM oracle uses the exact value
    e2m1(code) * float(s) * g in fp64.

Every other step (the matrix product, bias, per-head RMSNorm, gated SiLU,
residual + gate, the bf16 output rounding and the NVFP4 re-quantisation of an
output) is the plain definition written out in fp64.
"""
from __future__ import annotations

import numpy as np
import torch

# ---------------------------------------------------------------------------------------------
# E2M1 elements
# ---------------------------------------------------------------------------------------------

#: magnitudes of E2M1 codes 0..7 (2 exponent bits, 1 mantissa bit, no inf/nan)
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit codes (uint8, low nibble) -> fp64 values."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    mag = E2M1_MAGNITUDES[c & 0x7]
    return np.where(c & 0x8, -mag, mag)


def e2m1_round(v: np.ndarray) -> np.ndarray:
    """float32 values -> E2M1 codes: nearest magnitude, ties to the even code, saturate at 6.

    Brute force over the eight magnitudes.  Magnitudes above 6 are first clamped
    to 6 (saturation), so every distance below is exact in fp64.
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.minimum(np.abs(v).astype(np.float64), 6.0)
    best = np.zeros(a.shape, dtype=np.uint8)
    best_d = np.abs(a - E2M1_MAGNITUDES[0])
    for code in range(1, 8):
        d = np.abs(a - E2M1_MAGNITUDES[code])
        take = (d < best_d) | ((d == best_d) & (code % 2 == 0))
        best = np.where(take, np.uint8(code), best)
        best_d = np.where(take, d, best_d)
    neg = np.signbit(v)
    return np.where(neg, best | np.uint8(0x8), best).astype(np.uint8)


# ---------------------------------------------------------------------------------------------
# E4M3 block scales (unsigned use: the sign bit is always 0)
# ---------------------------------------------------------------------------------------------

def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3 bytes (sign 0) -> fp64.  Exponent bias 7; exponent field 0 is subnormal."""
    b = np.asarray(b, dtype=np.int64)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    return np.where(e == 0, sub, normal)


#: the 127 finite non-negative E4M3 values, byte 0x00..0x7E, in increasing order
E4M3_VALUES = e4m3_decode(np.arange(0x7F))


def e4m3_round_satfinite(x: np.ndarray) -> np.ndarray:
    """Non-negative float32 -> E4M3 byte: nearest representable value, ties to even, clamp at 448."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.any(x < 0) or not np.all(np.isfinite(x)):
        raise ValueError("E4M3 block scales are finite and non-negative")
    hi = np.searchsorted(E4M3_VALUES, x, side="left")       # first value >= x
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_hi = np.abs(E4M3_VALUES[hi] - x)
    d_lo = np.abs(x - E4M3_VALUES[lo])
    # adjacent representable values have adjacent byte codes, so "even byte" is "even mantissa"
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    return np.where(pick_lo, lo, hi).astype(np.uint8)


# ---------------------------------------------------------------------------------------------
# Quantiser, dequantiser, scale layout
# ---------------------------------------------------------------------------------------------

F32 = np.float32
BLOCK = 16


def tensor_scale(x: np.ndarray) -> np.float32:
    """Per-tensor decode scale g = amax / 2688 in fp32 (2688 = 6 * 448); 1 when amax is 0."""
    amax = F32(np.max(np.abs(np.asarray(x, dtype=F32)))) if np.size(x) else F32(0)
    if amax == 0:
        return F32(1.0)
    return F32(amax / F32(2688.0))


def quantize(x: np.ndarray, g: np.float32 | None = None, chunk_rows: int = 512):
    """x float32 [M,K] (bf16 values) -> (codes uint8 [M,K], scales uint8 [M,K/16], g).

    Codes are returned one per byte; ``pack_codes`` packs them two per byte.
    Rows are processed ``chunk_rows`` at a time only to bound host memory; the
    block rule touches one 16-element block at a time, so chunking changes nothing.
    """
    x = np.asarray(x, dtype=F32)
    M, K = x.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    g = tensor_scale(x) if g is None else F32(g)
    codes = np.empty((M, K), dtype=np.uint8)
    scales = np.empty((M, K // BLOCK), dtype=np.uint8)
    for r0 in range(0, M, chunk_rows):
        r1 = min(M, r0 + chunk_rows)
        codes[r0:r1], scales[r0:r1] = _quantize_blocks(x[r0:r1], g)
    return codes, scales, g


def _quantize_blocks(x: np.ndarray, g: np.float32):
    """The block rule on rows of x with a given g."""
    M, K = x.shape
    blocks = x.reshape(M, K // BLOCK, BLOCK)
    amax_b = np.max(np.abs(blocks), axis=2).astype(F32)
    r = (amax_b / g).astype(F32)
    s_f = (r / F32(6.0)).astype(F32)
    s = e4m3_round_satfinite(s_f)
    d = (e4m3_decode(s).astype(F32) * g).astype(F32)
    zero = d == 0
    inv = (F32(1.0) / np.where(zero, F32(1.0), d)).astype(F32)
    v = (blocks * inv[:, :, None]).astype(F32)
    codes = e2m1_round(v)
    codes = np.where(zero[:, :, None], np.uint8(0), codes)
    return codes.reshape(M, K), s


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[M,K] codes -> [M,K/2] bytes; element 2j in the low nibble, element 2j+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def dequantize(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    """codes [M,K], scales [M,K/16] -> float32 e2m1(code) * d with d = float(s) * g (both fp32 RN)."""
    M, K = codes.shape
    d = (e4m3_decode(scales).astype(F32) * F32(g)).astype(F32)
    vals = e2m1_decode(codes).astype(F32).reshape(M, K // BLOCK, BLOCK)
    return (vals * d[:, :, None]).astype(F32).reshape(M, K)


def fake_quantize(x: np.ndarray, g: np.float32 | None = None):
    """The forward value of training through the quantiser's own noise ("Serving sub-second Ideogram v4
    without quality loss", the passage on quantization-aware distillation: the student learns through
    its 4-bit rounding with a straight-through estimator, whose forward is the quantised value).  That
    value is the NVFP4 round trip: the block rule, then e2m1(code) * d, rounded to bf16.
    x float32 [M,K] (bf16 values) -> (y float32 of bf16 values [M,K], g)."""
    codes, scales, g = quantize(x, g)
    return to_bf16_round(dequantize(codes, scales, g)), g


def dequantize_exact(codes: np.ndarray, scales: np.ndarray, g) -> np.ndarray:
    """fp64 e2m1(code) * float(s) * g, exact (3 + 4 + 24 significant bits fit in 53)."""
    M, K = codes.shape
    vals = e2m1_decode(codes).reshape(M, K // BLOCK, BLOCK)
    return (vals * e4m3_decode(scales)[:, :, None] * np.float64(F32(g))).reshape(M, K)


def scale_atom_offset(r: int, c: int, K: int) -> int:
    """Byte offset of the scale of row r, 16-block c in the padded tensor-core scale layout.

    The buffer is a grid of 512-byte atoms, each holding 128 rows x 4 blocks;
    atoms run along K first, then along rows.  Inside an atom, row r and
    block c sit at (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4).
    """
    k_atoms = -(-(K // BLOCK) // 4)
    atom = (r // 128) * k_atoms + (c // 4)
    return atom * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def scale_offsets(M: int, K: int) -> np.ndarray:
    """``scale_atom_offset`` for every (row, block) at once: int64 [M, K/16]."""
    r = np.arange(M, dtype=np.int64)[:, None]
    c = np.arange(K // BLOCK, dtype=np.int64)[None, :]
    k_atoms = -(-(K // BLOCK) // 4)
    atom = (r // 128) * k_atoms + (c // 4)
    return atom * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def scale_buffer_bytes(M: int, K: int) -> int:
    rows = -(-M // 128) * 128
    cols = -(-(K // BLOCK) // 4) * 4
    return rows * cols


def scales_to_mma_layout(scales: np.ndarray) -> np.ndarray:
    """Row-major scales [M, K/16] -> padded atom layout (padding bytes are 0)."""
    M, nb = scales.shape
    K = nb * BLOCK
    out = np.zeros(scale_buffer_bytes(M, K), dtype=np.uint8)
    out[scale_offsets(M, K)] = scales
    return out


def scales_from_mma_layout(buf: np.ndarray, M: int, K: int) -> np.ndarray:
    return np.asarray(buf, dtype=np.uint8)[scale_offsets(M, K)]


# ---------------------------------------------------------------------------------------------
# GEMM + fused epilogues (fp64)
# ---------------------------------------------------------------------------------------------

def to_bf16_round(y: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 (torch CPU cast), returned as float32 values."""
    return torch.from_numpy(np.asarray(y, dtype=np.float64)).to(torch.bfloat16).float().numpy()


def matmul_exact(a_codes, a_scales, a_g, w_codes, w_scales, w_g) -> np.ndarray:
    """acc[m,n] = sum_k a_hat[m,k] * w_hat[n,k] on the exactly dequantised operands (fp64)."""
    a = dequantize_exact(a_codes, a_scales, a_g)
    w = dequantize_exact(w_codes, w_scales, w_g)
    return a @ w.T


def rmsnorm_heads(y: np.ndarray, gamma: np.ndarray, eps: float, head_dim: int = 256) -> np.ndarray:
    """Per-row, per-head RMSNorm: y_h / sqrt(mean(y_h^2) + eps) * gamma, gamma shared by all heads."""
    M, W = y.shape
    h = y.reshape(M, W // head_dim, head_dim)
    rms = np.sqrt(np.mean(h * h, axis=2, keepdims=True) + eps)
    return (h / rms * np.asarray(gamma, dtype=np.float64)[None, None, :]).reshape(M, W)


def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def epilogue(acc: np.ndarray, kind: str, bias=None, **ex) -> np.ndarray:
    """Apply one fused epilogue to the fp64 accumulator; returns fp64 (before bf16 rounding).

    kind: 'bias'        y = acc + bias
          'qknorm'      y = acc + bias, then per-head RMSNorm on [q_col0, q_col0+qk_cols) with
                        gamma_q and on [k_col0, k_col0+qk_cols) with gamma_k; other columns bias only
          'gated_silu'  y = acc + bias; a = y[:, :N/2], b = y[:, N/2:]; out = silu(a) * b
          'resid_gate'  out = residual + gate[n] * (acc + bias)
    """
    y = acc.astype(np.float64).copy()
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    if kind == "bias":
        return y
    if kind == "qknorm":
        hd = ex.get("head_dim", 256)
        eps = ex["eps"]
        for c0, gam in ((ex["q_col0"], ex["gamma_q"]), (ex["k_col0"], ex["gamma_k"])):
            sl = slice(c0, c0 + ex["qk_cols"])
            y[:, sl] = rmsnorm_heads(y[:, sl], gam, eps, hd)
        return y
    if kind == "gated_silu":
        half = y.shape[1] // 2
        return silu(y[:, :half]) * y[:, half:]
    if kind == "resid_gate":
        res = np.asarray(ex["residual"], dtype=np.float64)
        gate = np.asarray(ex["gate"], dtype=np.float64)
        return res + gate[None, :] * y
    raise ValueError(kind)


def linear(a_q, w_q, kind="bias", bias=None, rows=None, out_g=None, **ex):
    """Full NVFP4 linear on quantised operands.

    a_q, w_q: (codes [*,K], scales [*,K/16], g) as returned by ``quantize``.
    rows: optional row indices of A to evaluate (rows are independent).
    Returns dict with 'y' (fp64 epilogue output), 'bf16' (float32 holding bf16
    values) and, when ``out_g`` is given, 'q' = quantize(bf16 output, out_g).
    """
    ac, asc, ag = a_q
    if rows is not None:
        ac, asc = ac[rows], asc[rows]
        if "residual" in ex:
            ex = dict(ex, residual=np.asarray(ex["residual"])[rows])
    acc = matmul_exact(ac, asc, ag, *w_q)
    y = epilogue(acc, kind, bias=bias, **ex)
    yb = to_bf16_round(y)
    out = dict(y=y, bf16=yb)
    if out_g is not None:
        out["q"] = quantize(yb, out_g)
    return out


# ---------------------------------------------------------------------------------------------
# adaLN prologue of the quantiser (fp64, then one bf16 rounding)
# ---------------------------------------------------------------------------------------------

def adaln_modulate(x, shift=None, scale=None, eps: float = 1e-6, rows_per_sample: int = 0):
    """The op in front of a DiT block's QKV and FFN-up products, as the plain definition in fp64.

    "Serving sub-second Ideogram v4 without quality loss" (paragraph on kernel fusion) names RMSNorm
    as one of the small ops that chase the big products, and "Quantizing a Dual-Branch Flow-Matching
    Diffusion Transformer for Consumer GPUs" (related-work paragraph on W8A8) names adaLN's
    modulation, generated at run time, as what the hidden state goes through before a linear.
    Neither page writes the formula; the reading is the usual adaLN form on an RMS-normalised row:

        rstd[r] = 1 / sqrt(mean_k x[r,k]^2 + eps)
        u[r,k]  = x[r,k] * rstd[r] * (1 + scale[b,k]) + shift[b,k],   b = r // rows_per_sample

    (b = 0 for every row when rows_per_sample is 0).  shift / scale are [S, C] (or [C]); None means
    zeros.  Returns (u fp64 [M, C], rstd fp64 [M]).
    """
    x = np.asarray(x, dtype=np.float64)
    M, C = x.shape
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=1) + eps)
    sample = (np.arange(M) // rows_per_sample) if rows_per_sample else np.zeros(M, dtype=np.int64)

    def per_row(v):
        if v is None:
            return np.zeros((M, C), dtype=np.float64)
        return np.asarray(v, dtype=np.float64).reshape(-1, C)[sample]

    u = x * rstd[:, None] * (1.0 + per_row(scale)) + per_row(shift)
    return u, rstd


def adaln_quantize(x, shift=None, scale=None, eps: float = 1e-6, rows_per_sample: int = 0,
                   g: np.float32 | None = None):
    """The quantiser with the adaLN prologue: the modulated row is rounded once to bf16 (the value an
    unfused model would hold in memory) and quantised by the block rule.  With g None the tensor scale
    is amax(|u|) / 2688 of that bf16 tensor.  Returns ((codes, scales, g), u_bf16, rstd)."""
    u, rstd = adaln_modulate(x, shift, scale, eps, rows_per_sample)
    ub = to_bf16_round(u)
    return quantize(ub, g), ub, rstd


# ---------------------------------------------------------------------------------------------
# W8A8 INT8 linear (the other format the pages compare against NVFP4)
# ---------------------------------------------------------------------------------------------

def smoothquant_factors(act_absmax, w, alpha: float = 0.5):
    """SmoothQuant migration strength alpha ("Quantizing a Dual-Branch Flow-Matching Diffusion Transformer
    for Consumer GPUs", section on the method: the smoothing vector lambda_j = s_j^alpha /
    max_i |W_ij|^(1 - alpha) divides the activations' input channel j and multiplies the weights').
    act_absmax: per-input-channel max |x| from calibration [K]; w: [N, K].  A channel whose activation
    or weight column is all zero keeps lambda = 1.  Returned as fp32 (the value the kernels receive)."""
    s = np.asarray(act_absmax, dtype=np.float64)
    wmax = np.max(np.abs(np.asarray(w, dtype=np.float64)), axis=0)
    ok = (s > 0) & (wmax > 0)
    lam = np.ones_like(s)
    lam[ok] = s[ok] ** alpha / wmax[ok] ** (1.0 - alpha)
    return lam.astype(F32)


def int8_quantize_rows(x, act_mult=None):
    """Symmetric per-row INT8 ([Dual-Branch], method: per-token dynamic activations and per-output-row
    weights).  Each step is one binary32 operation rounded to nearest even:
        x'  = x * act_mult[k]        (the SmoothQuant divide, as a multiply by act_mult = 1 / lambda)
        s   = max_k |x'| / 127       (the decode scale; 1 for an all-zero row)
        inv = 127 / max_k |x'|       (0 for an all-zero row)
        q   = clamp(RNE(x' * inv), -127, 127)
    x float32 [M, K] -> (q int8 [M, K], s float32 [M])."""
    x = np.asarray(x, dtype=F32)
    if act_mult is not None:
        x = (x * np.asarray(act_mult, dtype=F32)[None, :]).astype(F32)
    amax = np.max(np.abs(x), axis=1).astype(F32) if x.shape[1] else np.zeros(x.shape[0], F32)
    zero = amax == 0
    s = np.where(zero, F32(1.0), (amax / F32(127.0)).astype(F32)).astype(F32)
    inv = np.where(zero, F32(0.0), (F32(127.0) / np.where(zero, F32(1.0), amax)).astype(F32)).astype(F32)
    v = (x * inv[:, None]).astype(F32)
    q = np.clip(np.rint(v), -127, 127).astype(np.int8)      # rint: ties to even
    return q, s


def int8_linear(qa, sa, qw, sw, bias=None):
    """y[m,n] = (sum_k qa[m,k] * qw[n,k]) * sa[m] * sw[n] + bias[n]: the integer product exactly (int64),
    the scaling in fp64.  Returns (y fp64, y rounded to bf16)."""
    acc = np.asarray(qa, dtype=np.int64) @ np.asarray(qw, dtype=np.int64).T
    y = acc.astype(np.float64) * np.asarray(sa, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :]
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y, to_bf16_round(y)


def rel_err_normwise(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / max |ref| over the whole tensor."""
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(np.asarray(got, dtype=np.float64) - ref)) / (den if den > 0 else 1.0))
