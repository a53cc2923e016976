"""Shared helpers for the parity tests: moving seeded inputs to the GPU and to the oracle."""
import numpy as np
import torch

from oracle import nvfp4_oracle as O


def f32(t: torch.Tensor) -> np.ndarray:
    """bf16/fp32 torch tensor (any device) -> float32 numpy (exact for bf16)."""
    return t.detach().float().cpu().numpy()


def oracle_quantize(x_bf16: torch.Tensor, g=None):
    """Oracle quantisation of a bf16 tensor: (codes [M,K], scales [M,K/16], g)."""
    return O.quantize(f32(x_bf16), g)


def gpu_qtensor_bytes(q):
    """(packed codes numpy [M,K/2], scale buffer numpy, g float32) of a binding.QTensor."""
    torch.cuda.synchronize()
    return q.codes.cpu().numpy(), q.scales.cpu().numpy(), np.float32(q.g.cpu().item())


def assert_quant_bitexact(q, ref, M, K):
    """GPU NVFP4 tensor == oracle (codes, scales, g) byte for byte, padding included."""
    codes, scales, g = gpu_qtensor_bytes(q)
    rc, rs, rg = ref
    assert g == rg, (g, rg)
    want_codes = O.pack_codes(rc)
    bad = np.argwhere(codes != want_codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    want_scales = O.scales_to_mma_layout(rs)
    assert scales.shape == want_scales.shape, (scales.shape, want_scales.shape)
    bad = np.flatnonzero(scales != want_scales)
    assert bad.size == 0, f"{bad.size} scale bytes differ, first offsets {bad[:5].tolist()}"


def normwise_rel_err(got, ref) -> float:
    return O.rel_err_normwise(got, ref)


def assert_close(got, ref, what, tol=2e-2):
    """The parity bar of a GEMM + epilogue output (bf16) against the oracle's fp64 value: the normwise max
    relative error max|got - ref| / max|ref| <= tol, and element by element |got - ref| <= tol *
    max(|ref|, 1e-2 * rms(ref)), so that a wrong bias, a misplaced column block or a wrong small value
    fails even where the largest outputs hide it from the normwise measure.  Returns the normwise error."""
    got = np.asarray(got)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = normwise_rel_err(got, ref)
    assert err <= tol, f"{what}: normwise rel err {err:.3e} > {tol}"
    worst = elementwise_ok(got, ref, rel=tol)
    if worst > 1.0:
        ref64 = np.asarray(ref, np.float64)
        rms = np.sqrt(np.mean(ref64 * ref64))
        ratio = np.abs(np.asarray(got, np.float64) - ref64) / np.maximum(np.abs(ref64), 1e-2 * rms)
        idx = np.unravel_index(np.argmax(ratio), ratio.shape)
        raise AssertionError(f"{what}: elementwise error {worst * tol:.3e} relative at {idx}: got {got[idx]}, "
                             f"oracle {ref64[idx]}")
    return err


def elementwise_ok(got, ref, rel=2e-2, floor_frac=1e-2):
    """Elementwise |got-ref| <= rel * max(|ref|, floor_frac * rms(ref)); returns the worst ratio."""
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 1.0
    den = np.maximum(np.abs(ref), floor_frac * rms)
    return float(np.max(np.abs(got - ref) / den)) / rel


def assert_requant_close(q, ref, M, K, max_frac=1e-3):
    """A fused re-quantised output against the oracle's re-quantisation of its own bf16 output.

    The two bf16 outputs may differ in the last bit, which can move a block scale by one E4M3 step
    or a code by one E2M1 step.  Everything else must match: the fraction of differing scale bytes
    and codes stays below ``max_frac`` and every difference is one step.
    """
    codes, scales, g = gpu_qtensor_bytes(q)
    rc, rs, rg = ref
    assert g == rg
    got_s = O.scales_from_mma_layout(scales, M, K).astype(np.int64)
    ds = np.abs(got_s - rs.astype(np.int64))
    assert ds.max(initial=0) <= 1 and np.mean(ds > 0) <= max_frac, (ds.max(initial=0), np.mean(ds > 0))
    got_c = O.unpack_codes(codes).astype(np.int64)
    same_scale = np.repeat(ds == 0, 16, axis=1)
    mag = lambda c: np.where(c & 8, -(c & 7), c & 7)          # signed magnitude index
    dc = np.abs(mag(got_c) - mag(rc.astype(np.int64)))
    dc = np.where(same_scale, dc, 0)
    assert dc.max(initial=0) <= 1 and np.mean(dc > 0) <= max_frac, (dc.max(initial=0), np.mean(dc > 0))


def assert_quant_arrays_close(got, ref, max_frac=1e-3):
    """Row-major (codes [M,K] one per byte, scales [M,K/16], g) against the oracle's, when the two inputs
    may differ in the last bf16 bit: g equal, and every differing scale byte or code one step apart,
    each kind of difference in at most ``max_frac`` of the entries."""
    gc, gs, gg = got
    rc, rs, rg = ref
    assert gg == rg, (gg, rg)
    ds = np.abs(gs.astype(np.int64) - rs.astype(np.int64))
    assert ds.max(initial=0) <= 1 and np.mean(ds > 0) <= max_frac, (ds.max(initial=0), np.mean(ds > 0))
    mag = lambda c: np.where(c & 8, -(c & 7), c & 7)
    dc = np.abs(mag(gc.astype(np.int64)) - mag(rc.astype(np.int64)))
    dc = np.where(np.repeat(ds == 0, 16, axis=1), dc, 0)
    assert dc.max(initial=0) <= 1 and np.mean(dc > 0) <= max_frac, (dc.max(initial=0), np.mean(dc > 0))
