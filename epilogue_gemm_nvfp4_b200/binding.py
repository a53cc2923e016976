"""ctypes binding of libnvfp4 (the C ABI in include/nvfp4.h): argument marshalling only.

Every step of the NVFP4 path runs in the library's CUDA kernels; this module
turns torch tensors into the C structs (device pointers, sizes, the current
CUDA stream) and raises when the library reports an error.  There is no CPU
fallback: if the shared library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

#: every function the header declares
EXPORTS = ("nvfp4_quantize", "nvfp4_linear", "nvfp4_dequantize", "nvfp4_amax", "nvfp4_scale_bytes",
           "nvfp4_scale_offset", "nvfp4_get_device_error", "nvfp4_linear_tile_n", "nvfp4_linear_split_k",
           "nvfp4_status_string", "nvfp4_version", "nvfp4_linear_noalloc", "nvfp4_linear_noalloc_scratch_bytes",
           "nvfp4_fake_quantize", "nvfp4_adaln_quantize", "nvfp4_int8_quantize", "nvfp4_int8_linear")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_MISALIGNED, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_SCRATCH_LIMIT = range(7)
EPI_BIAS, EPI_QKNORM, EPI_GATED_SILU, EPI_RESID_GATE = range(4)
EPI_KINDS = {"bias": EPI_BIAS, "qknorm": EPI_QKNORM, "gated_silu": EPI_GATED_SILU, "resid_gate": EPI_RESID_GATE}


class CTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("ld_codes", ctypes.c_int64)]


class CEpilogue(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("bias", ctypes.c_void_p), ("gamma_q", ctypes.c_void_p),
                ("gamma_k", ctypes.c_void_p), ("eps", ctypes.c_float), ("head_dim", ctypes.c_int32),
                ("q_col0", ctypes.c_int64), ("k_col0", ctypes.c_int64), ("qk_cols", ctypes.c_int64),
                ("residual", ctypes.c_void_p), ("ld_residual", ctypes.c_int64), ("gate", ctypes.c_void_p),
                ("out_nvfp4", ctypes.c_int32), ("out_amax", ctypes.c_void_p)]


class CAdaln(ctypes.Structure):
    _fields_ = [("shift", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("ld_mod", ctypes.c_int64),
                ("rows_per_sample", ctypes.c_int64), ("eps", ctypes.c_float), ("rstd", ctypes.c_void_p),
                ("u_out", ctypes.c_void_p), ("ld_u", ctypes.c_int64)]


class CInt8Tensor(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld", ctypes.c_int64)]


class NvFp4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libnvfp4.so (in-tree).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m epilogue_gemm_nvfp4_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    TP = ctypes.POINTER(CTensor)
    EP = ctypes.POINTER(CEpilogue)
    AP = ctypes.POINTER(CAdaln)
    IP = ctypes.POINTER(CInt8Tensor)
    sig = {
        "nvfp4_quantize": (I32, [P, I64, I64, I64, I32, TP, P]),
        "nvfp4_linear": (I32, [TP, TP, EP, P, I64, TP, P]),
        "nvfp4_linear_noalloc": (I32, [TP, TP, EP, P, I64, TP, P]),
        "nvfp4_linear_noalloc_scratch_bytes": (SZ, []),
        "nvfp4_dequantize": (I32, [TP, P, I64, P]),
        "nvfp4_fake_quantize": (I32, [P, I64, I64, I64, I32, P, P, I64, P]),
        "nvfp4_adaln_quantize": (I32, [P, I64, I64, I64, AP, I32, TP, P]),
        "nvfp4_int8_quantize": (I32, [P, I64, I64, I64, P, IP, P]),
        "nvfp4_int8_linear": (I32, [IP, IP, EP, P, I64, TP, P]),
        "nvfp4_amax": (I32, [P, I64, I64, I64, P, P]),
        "nvfp4_scale_bytes": (SZ, [I64, I64]),
        "nvfp4_scale_offset": (I64, [I64, I64, I64]),
        "nvfp4_get_device_error": (I32, [P]),
        "nvfp4_linear_tile_n": (I32, [I64, I64, I32]),
        "nvfp4_linear_split_k": (I32, [I64, I64, I32]),
        "nvfp4_status_string": (ctypes.c_char_p, [I32]),
        "nvfp4_version": (I32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().nvfp4_status_string(status).decode()


def _check(status: int, what: str):
    if status != OK:
        raise NvFp4Error(status, what)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ------------------------------------------------------------------------------------------
# NVFP4 tensor held in torch device memory
# ------------------------------------------------------------------------------------------

@dataclass
class QTensor:
    """An NVFP4 tensor: packed codes uint8 [rows, cols/2], padded scale bytes, fp32 decode scale [1]."""
    codes: torch.Tensor
    scales: torch.Tensor
    g: torch.Tensor
    rows: int
    cols: int

    @classmethod
    def empty(cls, rows: int, cols: int, device="cuda") -> "QTensor":
        lib = load()
        nbytes = int(lib.nvfp4_scale_bytes(rows, cols))
        return cls(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                   torch.empty(nbytes, dtype=torch.uint8, device=device),
                   torch.empty(1, dtype=torch.float32, device=device), rows, cols)

    def c(self) -> CTensor:
        return CTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.g.data_ptr(), self.rows, self.cols,
                       self.codes.stride(0))


def scale_bytes(rows: int, cols: int) -> int:
    return int(load().nvfp4_scale_bytes(rows, cols))


def scale_offset(r: int, kb: int, cols: int) -> int:
    return int(load().nvfp4_scale_offset(r, kb, cols))


def tile_n(N: int, K: int, kind: str) -> int:
    return int(load().nvfp4_linear_tile_n(N, K, EPI_KINDS[kind]))


def split_k(N: int, K: int, kind: str) -> int:
    return int(load().nvfp4_linear_split_k(N, K, EPI_KINDS[kind]))


def quantize(x: torch.Tensor, out: QTensor | None = None, g: float | torch.Tensor | None = None,
             static: bool = False, stream=None) -> QTensor:
    """bf16 [rows, cols] (CUDA) -> NVFP4.  By default the tensor scale is computed on the device.
    With ``g`` the given decode scale is stored in out.g and used; with ``static=True`` the scale
    already held in out.g is used."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    out = QTensor.empty(rows, cols, x.device) if out is None else out
    if g is not None:
        out.g.copy_(torch.as_tensor(g, dtype=torch.float32).reshape(1))
    compute = g is None and not static
    ct = out.c()
    _check(load().nvfp4_quantize(_ptr(x), rows, cols, x.stride(0), int(compute), ctypes.byref(ct),
                                 _stream(stream)), "nvfp4_quantize")
    return out


def fake_quantize(x: torch.Tensor, y: torch.Tensor | None = None, g: float | torch.Tensor | None = None,
                  scale: torch.Tensor | None = None, static: bool = False,
                  stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """y = dequantize(quantize(x)) in bf16, one pass.  By default g is computed on the device and
    returned in ``scale`` (one fp32 element); with ``g`` the given decode scale is stored there and
    used; with ``static=True`` the value already in ``scale`` is used."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    y = torch.empty((rows, cols), dtype=torch.bfloat16, device=x.device) if y is None else y
    scale = torch.empty(1, dtype=torch.float32, device=x.device) if scale is None else scale
    if g is not None:
        scale.copy_(torch.as_tensor(g, dtype=torch.float32).reshape(1))
    compute = g is None and not static
    _check(load().nvfp4_fake_quantize(_ptr(x), rows, cols, x.stride(0), int(compute), _ptr(scale), _ptr(y),
                                      y.stride(0), _stream(stream)), "nvfp4_fake_quantize")
    return y, scale


def adaln_quantize(x: torch.Tensor, shift: torch.Tensor | None = None, scale: torch.Tensor | None = None,
                   eps: float = 1e-6, rows_per_sample: int = 0, out: QTensor | None = None,
                   g: float | torch.Tensor | None = None, static: bool = False, rstd: torch.Tensor | None = None,
                   u_out: torch.Tensor | None = None, stream=None) -> QTensor:
    """NVFP4 of u = bf16(RMSNorm(x) * (1 + scale) + shift) through nvfp4_adaln_quantize.  shift / scale are
    bf16 [cols] or [samples, cols] (row r uses sample r // rows_per_sample).  The tensor scale follows
    ``quantize``: computed on the device by default, ``g`` given, or ``static`` (out.g as it is).
    ``rstd`` (fp32 [rows]) and ``u_out`` (bf16 [rows, cols]) receive the per-row 1/rms and u when given."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    out = QTensor.empty(rows, cols, x.device) if out is None else out
    if g is not None:
        out.g.copy_(torch.as_tensor(g, dtype=torch.float32).reshape(1))
    compute = g is None and not static
    mods = [m for m in (shift, scale) if m is not None]
    for m in mods:
        assert m.is_cuda and m.dtype == torch.bfloat16 and m.stride(-1) == 1 and m.shape[-1] == cols
    samples = 1 if rows_per_sample <= 0 or rows_per_sample >= rows else -(-rows // rows_per_sample)
    ld_mod = cols
    if mods:
        dims = {m.dim() for m in mods}
        assert dims in ({1}, {2}), "shift and scale are both [cols] or both [samples, cols]"
        if dims == {2}:
            ld_mod = mods[0].stride(0)
            assert all(m.stride(0) == ld_mod and m.shape[0] >= samples for m in mods), \
                "shift and scale need the same sample stride and one row per sample"
        else:
            assert samples == 1, "per-sample modulation needs [samples, cols] vectors"
    desc = CAdaln(_ptr(shift), _ptr(scale), int(ld_mod), int(rows_per_sample), float(eps), _ptr(rstd),
                  _ptr(u_out), u_out.stride(0) if u_out is not None else 0)
    ct = out.c()
    _check(load().nvfp4_adaln_quantize(_ptr(x), rows, cols, x.stride(0), ctypes.byref(desc), int(compute),
                                       ctypes.byref(ct), _stream(stream)), "nvfp4_adaln_quantize")
    return out


def dequantize(q: QTensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = torch.empty((q.rows, q.cols), dtype=torch.bfloat16, device=q.codes.device) if out is None else out
    ct = q.c()
    _check(load().nvfp4_dequantize(ctypes.byref(ct), _ptr(out), out.stride(0), _stream(stream)), "nvfp4_dequantize")
    return out


def amax(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    rows, cols = x.shape
    _check(load().nvfp4_amax(_ptr(x), rows, cols, x.stride(0), _ptr(out), _stream(stream)), "nvfp4_amax")
    return out


def make_epilogue(kind: str = "bias", bias=None, gamma_q=None, gamma_k=None, eps=1e-6, q_col0=0, k_col0=0,
                  qk_cols=0, head_dim=256, residual=None, gate=None, out_nvfp4=False, out_amax=None) -> CEpilogue:
    """``out_amax``: fp32 device tensor of one element (zeroed by the caller) that the kernel raises to
    max |bf16 output|."""
    return CEpilogue(EPI_KINDS[kind], _ptr(bias), _ptr(gamma_q), _ptr(gamma_k), float(eps), int(head_dim),
                     int(q_col0), int(k_col0), int(qk_cols), _ptr(residual),
                     residual.stride(0) if residual is not None else 0, _ptr(gate), int(bool(out_nvfp4)),
                     _ptr(out_amax))


def linear(a: QTensor, w: QTensor, kind: str = "bias", bias=None, out: torch.Tensor | None = None,
           out_fp4: QTensor | None = None, want_bf16: bool = True, stream=None, **epi) -> torch.Tensor | None:
    """Fused NVFP4 linear through nvfp4_linear.  ``out_fp4`` (with its g set) turns on the NVFP4
    re-quantisation of the output; ``want_bf16=False`` skips the bf16 output then."""
    n_out = w.rows // 2 if kind == "gated_silu" else w.rows
    if out is None and want_bf16:
        out = torch.empty((a.rows, n_out), dtype=torch.bfloat16, device=a.codes.device)
    desc = make_epilogue(kind, bias=bias, out_nvfp4=out_fp4 is not None, **epi)
    ca, cw = a.c(), w.c()
    cq = out_fp4.c() if out_fp4 is not None else None
    _check(load().nvfp4_linear(ctypes.byref(ca), ctypes.byref(cw), ctypes.byref(desc), _ptr(out),
                               out.stride(0) if out is not None else 0,
                               ctypes.byref(cq) if cq is not None else None, _stream(stream)), "nvfp4_linear")
    return out


# ------------------------------------------------------------------------------------------
# W8A8 INT8 path
# ------------------------------------------------------------------------------------------

@dataclass
class Int8Tensor:
    """Per-row INT8: codes int8 [rows, cols] and the fp32 decode scale of each row [rows]."""
    q: torch.Tensor
    scale: torch.Tensor
    rows: int
    cols: int

    @classmethod
    def empty(cls, rows: int, cols: int, device="cuda") -> "Int8Tensor":
        return cls(torch.empty((rows, cols), dtype=torch.int8, device=device),
                   torch.empty(max(rows, 1), dtype=torch.float32, device=device), rows, cols)

    def c(self) -> CInt8Tensor:
        return CInt8Tensor(self.q.data_ptr(), self.scale.data_ptr(), self.rows, self.cols, self.q.stride(0))


def int8_quantize(x: torch.Tensor, col_mult: torch.Tensor | None = None, out: Int8Tensor | None = None,
                  stream=None) -> Int8Tensor:
    """bf16 [rows, cols] -> per-row INT8 through nvfp4_int8_quantize; ``col_mult`` (fp32 [cols]) multiplies
    each column first (1 / lambda for activations, lambda for a weight under SmoothQuant)."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, cols = x.shape
    if col_mult is not None:
        assert col_mult.is_cuda and col_mult.dtype == torch.float32 and col_mult.numel() == cols
    out = Int8Tensor.empty(rows, cols, x.device) if out is None else out
    ct = out.c()
    _check(load().nvfp4_int8_quantize(_ptr(x), rows, cols, x.stride(0), _ptr(col_mult), ctypes.byref(ct),
                                      _stream(stream)), "nvfp4_int8_quantize")
    return out


def int8_linear(a: Int8Tensor, w: Int8Tensor, kind: str = "bias", bias=None, out: torch.Tensor | None = None,
                out_fp4: QTensor | None = None, want_bf16: bool = True, stream=None, **epi) -> torch.Tensor | None:
    """Fused W8A8 linear through nvfp4_int8_linear (the epilogue arguments of ``linear``)."""
    n_out = w.rows // 2 if kind == "gated_silu" else w.rows
    if out is None and want_bf16:
        out = torch.empty((a.rows, n_out), dtype=torch.bfloat16, device=a.q.device)
    desc = make_epilogue(kind, bias=bias, out_nvfp4=out_fp4 is not None, **epi)
    ca, cw = a.c(), w.c()
    cq = out_fp4.c() if out_fp4 is not None else None
    _check(load().nvfp4_int8_linear(ctypes.byref(ca), ctypes.byref(cw), ctypes.byref(desc), _ptr(out),
                                    out.stride(0) if out is not None else 0,
                                    ctypes.byref(cq) if cq is not None else None, _stream(stream)),
           "nvfp4_int8_linear")
    return out


def get_device_error(stream=None) -> int:
    return int(load().nvfp4_get_device_error(_stream(stream)))


def check_device_error(stream=None):
    _check(get_device_error(stream), "device")
