"""Seeded synthetic tensors shaped like the DiT linear layers on the pages.

This module only draws random numbers and lays them out; it holds none of the
NVFP4 arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it without sharing any of the method.

Shapes follow "Faster Ideogram 4 with Less Prompt Compute" (section
"Conditioning a Denoising Step": hidden width 4,608, 4,096 image positions at
1024^2 plus a 512-token prompt = 4,608 packed positions, a 1,941-token prompt,
the 53,248-wide text features) and "Serving sub-second Ideogram v4 without
quality loss" (256-dimension attention heads, gated SiLU).  Every tensor is
drawn with numpy's ``default_rng(seed)`` in float32 and rounded once to bf16
(round-to-nearest-even, torch's CPU cast).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

HIDDEN = 4608          # DiT hidden width
HEAD_DIM = 256         # attention head width
N_HEADS = HIDDEN // HEAD_DIM   # 18
FFN = 12288            # gated-SiLU inner width
TEXT_K = 53248         # text-encoder feature width
IMG_TOKENS_1K = 4096   # image positions at 1024^2
IMG_TOKENS_2K = 16384  # image positions at 2048^2
PROMPT_T = 512         # main-profile prompt length
LONG_PROMPT_T = 1941   # near-maximum prompt length


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy array -> bf16 torch CPU tensor (RNE)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def with_outlier_columns(rng: np.random.Generator, a: np.ndarray, n_cols: int, factor: float) -> np.ndarray:
    """Scale ``n_cols`` randomly chosen columns of ``a`` by ``factor`` (activation outlier channels)."""
    if n_cols > 0:
        cols = rng.choice(a.shape[1], n_cols, replace=False)
        a[:, cols] *= np.float32(factor)
    return a


def student_t(rng: np.random.Generator, shape, df: float = 4.0) -> np.ndarray:
    return rng.standard_t(df, size=shape).astype(np.float32)


def uniform(rng: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    return rng.uniform(lo, hi, size=shape).astype(np.float32)


@dataclass
class LinearCase:
    """One linear layer: activation x [M,K], weight w [N,K] (nn.Linear layout), extras by epilogue."""
    name: str
    x: torch.Tensor | None
    w: torch.Tensor
    bias: torch.Tensor | None = None
    epilogue: str = "bias"              # bias | qknorm | gated_silu | resid_gate
    extras: dict = field(default_factory=dict)
    rows: int | None = None             # M when x is not materialised (input comes from a previous layer)

    @property
    def M(self): return self.x.shape[0] if self.x is not None else self.rows

    @property
    def K(self): return self.w.shape[1]

    @property
    def N(self): return self.w.shape[0]

    @property
    def n_out(self):
        return self.N // 2 if self.epilogue == "gated_silu" else self.N


def case_bias(M, N, K, seed=0, x_std=1.0, w_std=0.02, b_std=0.01, outlier_cols=0,
              outlier_factor=20.0, x_dist="normal", name="bias") -> LinearCase:
    rng = np.random.default_rng(seed)
    if x_dist == "student_t":
        x = student_t(rng, (M, K))
    else:
        x = normal(rng, (M, K), x_std)
    x = with_outlier_columns(rng, x, outlier_cols, outlier_factor)
    w = normal(rng, (N, K), w_std)
    b = normal(rng, (N,), b_std)
    return LinearCase(name, to_bf16(x), to_bf16(w), to_bf16(b), "bias")


def case_qkv(M, n_heads=N_HEADS, K=HIDDEN, seed=0, outlier_frac=0.01, outlier_factor=30.0,
             w_std=0.015, b_std=0.01, eps=1e-6, name="qkv") -> LinearCase:
    """QKV projection: N = 3 * n_heads * 256 columns, q | k | v, per-head RMSNorm on q and k."""
    rng = np.random.default_rng(seed)
    width = n_heads * HEAD_DIM
    N = 3 * width
    x = normal(rng, (M, K))
    x = with_outlier_columns(rng, x, int(round(outlier_frac * K)), outlier_factor)
    w = normal(rng, (N, K), w_std)
    b = normal(rng, (N,), b_std)
    gq = uniform(rng, (HEAD_DIM,), 0.5, 1.5)
    gk = uniform(rng, (HEAD_DIM,), 0.5, 1.5)
    return LinearCase(name, to_bf16(x), to_bf16(w), to_bf16(b), "qknorm",
                      dict(gamma_q=to_bf16(gq), gamma_k=to_bf16(gk), eps=eps,
                           q_col0=0, k_col0=width, qk_cols=width, head_dim=HEAD_DIM))


def case_ffn_up(M, K=HIDDEN, F=FFN, seed=0, w_std=0.015, name="ffn_up") -> LinearCase:
    """Up projection W [2F, K]: rows [0,F) give a, rows [F,2F) give b; out = silu(a) * b, [M, F]."""
    rng = np.random.default_rng(seed)
    x = normal(rng, (M, K))
    w = normal(rng, (2 * F, K), w_std)
    return LinearCase(name, to_bf16(x), to_bf16(w), None, "gated_silu")


def case_ffn_down(M, N=HIDDEN, F=FFN, seed=0, w_std=0.01, with_x=True, name="ffn_down") -> LinearCase:
    """Down projection W [N, F] with out = residual + gate[n] * y.

    With ``with_x=False`` no activation is drawn: in a DiT block the input is the
    NVFP4 output of the gated-SiLU up projection.
    """
    rng = np.random.default_rng(seed)
    w = normal(rng, (N, F), w_std)
    res = normal(rng, (M, N))
    gate = uniform(rng, (N,), 0.0, 1.0)
    x = to_bf16(normal(rng, (M, F))) if with_x else None
    return LinearCase(name, x, to_bf16(w), None, "resid_gate",
                      dict(residual=to_bf16(res), gate=torch.from_numpy(gate)), rows=M)


def case_text(T, K=TEXT_K, N=HIDDEN, seed=0, w_std=0.005, b_std=0.01, zero_rows=0,
              name="text") -> LinearCase:
    """Text-conditioning projection [T, 53248] -> [T, 4608] with bias; Student-t (df=4) features.

    ``zero_rows`` appends that many all-zero rows (the image positions of the
    packed conditioning tensor), for the row-independence check.
    """
    rng = np.random.default_rng(seed)
    x = student_t(rng, (T, K))
    w = normal(rng, (N, K), w_std)
    b = normal(rng, (N,), b_std)
    if zero_rows:
        x = np.concatenate([x, np.zeros((zero_rows, K), np.float32)], axis=0)
    return LinearCase(name, to_bf16(x), to_bf16(w), to_bf16(b), "bias")


@dataclass
class AdalnCase:
    """A DiT hidden state x [M, C] and its adaLN vectors shift, scale [S, C] (one pair per sample;
    row r belongs to sample r // rows_per_sample, or to sample 0 when rows_per_sample is 0)."""
    name: str
    x: torch.Tensor
    shift: torch.Tensor
    scale: torch.Tensor
    rows_per_sample: int = 0
    eps: float = 1e-6


def case_adaln(M, C=HIDDEN, samples=1, seed=0, outlier_frac=0.01, outlier_factor=30.0, mod_std=0.5,
               name="adaln") -> AdalnCase:
    """x N(0,1) with 1% outlier channels x30 (as the QKV input); shift, scale N(0, mod_std^2) per sample."""
    rng = np.random.default_rng(seed)
    x = normal(rng, (M, C))
    x = with_outlier_columns(rng, x, int(round(outlier_frac * C)), outlier_factor)
    shift = normal(rng, (samples, C), mod_std)
    scale = normal(rng, (samples, C), mod_std)
    L = 0 if samples == 1 else -(-M // samples)
    return AdalnCase(name, to_bf16(x), to_bf16(shift), to_bf16(scale), L)


# ---- the named workloads -------------------------------------------------------------------

def tiny(seed=0) -> LinearCase:
    """x [256,512] N(0,1) with 4 outlier columns x20, W [512,512] N(0,0.02^2), bias N(0,0.01^2)."""
    return case_bias(256, 512, 512, seed=seed, w_std=0.02, outlier_cols=4, outlier_factor=20.0,
                     name="tiny_256x512x512")


def qkv_1k(seed=0) -> LinearCase:
    return case_qkv(IMG_TOKENS_1K + PROMPT_T, seed=seed, name="qkv_1024sq")


def ffn_1k(seed=0) -> tuple[LinearCase, LinearCase]:
    M = IMG_TOKENS_1K + PROMPT_T
    return (case_ffn_up(M, seed=seed, name="ffn_up_1024sq"),
            case_ffn_down(M, seed=seed + 1, name="ffn_down_1024sq"))


def text_proj(T=PROMPT_T, zero_rows=0, seed=0) -> LinearCase:
    return case_text(T, seed=seed, zero_rows=zero_rows, name=f"text_T{T}+{zero_rows}z")


def block_2k(seed=7, M=IMG_TOKENS_2K + PROMPT_T) -> dict:
    """The DiT-block linear set at 2048^2: QKV(+q/k RMSNorm), out-proj, gated-SiLU up, down(+res/gate)."""
    return dict(
        qkv=case_qkv(M, seed=seed, name="block2k_qkv"),
        out=case_bias(M, HIDDEN, HIDDEN, seed=seed + 1, w_std=0.015, name="block2k_out"),
        up=case_ffn_up(M, seed=seed + 2, name="block2k_up"),
        down=case_ffn_down(M, seed=seed + 3, with_x=False, name="block2k_down"),
    )


def adaln_2k(seed=7, M=IMG_TOKENS_2K + PROMPT_T) -> AdalnCase:
    """The hidden state in front of the QKV / FFN-up products at 2048^2, with its adaLN modulation."""
    return case_adaln(M, seed=seed, name="adaln_2048sq")


def flops(case: LinearCase) -> float:
    return 2.0 * case.M * case.N * case.K
