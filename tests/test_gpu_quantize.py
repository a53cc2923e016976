"""GPU parity of the bandwidth kernels through the C ABI: quantise (both scale modes), amax and
dequantise must equal the oracle byte for byte, padding included."""
import numpy as np
import pytest
import torch

from epilogue_gemm_nvfp4_b200 import binding as B
from epilogue_gemm_nvfp4_b200 import workloads as W
from oracle import nvfp4_oracle as O
from tests.helpers import assert_quant_bitexact, f32, oracle_quantize

pytestmark = pytest.mark.gpu


def rand_bf16(rows, cols, seed, scale=1.0, dist="normal"):
    rng = np.random.default_rng(seed)
    a = W.student_t(rng, (rows, cols)) if dist == "t" else W.normal(rng, (rows, cols), scale)
    return W.to_bf16(a)


@pytest.mark.parametrize("rows,cols,seed", [(1, 16, 0), (5, 48, 1), (130, 208, 2), (127, 64, 3), (129, 512, 4),
                                            (300, 4608, 5), (33, 53248, 6)])
def test_quantize_bitexact_ragged(lib, rows, cols, seed):
    x = rand_bf16(rows, cols, seed, dist="t" if seed % 2 else "normal")
    q = B.quantize(x.cuda())
    assert_quant_bitexact(q, oracle_quantize(x), rows, cols)


def test_quantize_static_scale_and_saturation(lib):
    x = rand_bf16(256, 512, 7)
    g = np.float32(0.0005)  # small g: many block scales clamp at 448 and many codes at 6
    q = B.quantize(x.cuda(), g=float(g))
    ref = oracle_quantize(x, g)
    assert (ref[1] == 0x7E).any()
    assert_quant_bitexact(q, ref, 256, 512)


def test_quantize_zero_and_tiny_blocks(lib):
    x = rand_bf16(128, 256, 8)
    x[3] = 0
    x[5, :16] = 1e-30
    x[6] = -x[6].abs()
    q = B.quantize(x.cuda())
    assert_quant_bitexact(q, oracle_quantize(x), 128, 256)
    z = torch.zeros(64, 64, dtype=torch.bfloat16)
    qz = B.quantize(z.cuda())
    assert qz.g.item() == 1.0
    assert_quant_bitexact(qz, oracle_quantize(z), 64, 64)


def test_quantize_strided_input(lib):
    x = rand_bf16(70, 1024, 9)
    xs = x.cuda()[:, 256:768]
    assert xs.stride(0) == 1024
    q = B.quantize(xs)
    assert_quant_bitexact(q, oracle_quantize(x[:, 256:768].contiguous()), 70, 512)


def test_amax(lib):
    x = rand_bf16(513, 4608, 10, dist="t")
    got = B.amax(x.cuda()).item()
    assert got == float(np.max(np.abs(f32(x))))
    xs = x.cuda()[:, :2304]
    assert B.amax(xs).item() == float(np.max(np.abs(f32(x[:, :2304]))))


@pytest.mark.parametrize("rows,cols,seed", [(130, 208, 11), (256, 4608, 12)])
def test_dequantize_bitexact(lib, rows, cols, seed):
    x = rand_bf16(rows, cols, seed)
    q = B.quantize(x.cuda())
    got = B.dequantize(q)
    c, s, g = oracle_quantize(x)
    want = O.to_bf16_round(O.dequantize(c, s, g))
    np.testing.assert_array_equal(f32(got), want)
    B.check_device_error()


@pytest.mark.parametrize("name", ["tiny", "qkv_x", "qkv_w", "text_x", "text_w"])
def test_quantize_bitexact_workload_tensors(lib, name):
    if name == "tiny":
        case = W.tiny()
        tensors = [case.x, case.w]
    elif name.startswith("qkv"):
        case = W.qkv_1k()
        tensors = [case.x if name == "qkv_x" else case.w]
    else:
        case = W.text_proj(W.PROMPT_T)
        tensors = [case.x if name == "text_x" else case.w]
    for t in tensors:
        q = B.quantize(t.cuda())
        assert_quant_bitexact(q, oracle_quantize(t), *t.shape)


def test_dynamic_scale_state_is_per_call_and_per_stream(lib):
    """The dynamic scale's amax reduction keeps {amax, CTAs done} per stream and clears it in the last
    CTA: a large tensor followed by a 100x smaller one on the same stream, and a call on a second
    stream, each get their own g."""
    rng = np.random.default_rng(41)
    big = W.to_bf16(rng.standard_normal((300, 512)).astype(np.float32) * 50.0)
    small = W.to_bf16(rng.standard_normal((300, 512)).astype(np.float32) * 0.5)
    ref = {id(big): oracle_quantize(big), id(small): oracle_quantize(small)}
    for x in (big, small, big, small):
        assert_quant_bitexact(B.quantize(x.cuda()), ref[id(x)], 300, 512)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        q = B.quantize(small.cuda())
    side.synchronize()
    assert_quant_bitexact(q, ref[id(small)], 300, 512)
    assert_quant_bitexact(B.quantize(big.cuda()), ref[id(big)], 300, 512)


# ------------------------------------------------------------------------------------------
# fake quantisation: y = dequantise(quantise(x)) in one pass
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols,seed", [(1, 16, 0), (130, 208, 2), (300, 4608, 5), (33, 53248, 6)])
def test_fake_quantize_bitexact(lib, rows, cols, seed):
    x = rand_bf16(rows, cols, seed, dist="t" if seed % 2 else "normal")
    y, g = B.fake_quantize(x.cuda())
    ref_y, ref_g = O.fake_quantize(f32(x))
    torch.cuda.synchronize()
    assert float(g.item()) == float(ref_g)
    np.testing.assert_array_equal(f32(y), ref_y)
    # and it equals the library's own quantise followed by dequantise
    q = B.quantize(x.cuda())
    np.testing.assert_array_equal(f32(y), f32(B.dequantize(q)))


def test_fake_quantize_static_scale_and_strides(lib):
    base = rand_bf16(96, 512 + 64, 17)
    x = base.cuda()[:, 32:32 + 512]             # row stride 576 elements, 64-byte offset
    y = torch.empty(96, 512 + 16, dtype=torch.bfloat16, device="cuda")[:, :512]
    g = 0.7 / 2688.0
    out, scale = B.fake_quantize(x, y=y, g=g)
    torch.cuda.synchronize()
    assert out.data_ptr() == y.data_ptr()
    ref_y, _ = O.fake_quantize(f32(base)[:, 32:32 + 512], np.float32(g))
    np.testing.assert_array_equal(f32(out), ref_y)


def test_empty_inputs_through_the_abi(lib):
    """rows == 0 / M == 0: the quantiser writes no codes and its dynamic scale is 1 (the all-zero rule), the
    scale padding rows are zero, and the fused linear returns without touching its output.  Called through
    the C ABI with real buffers (torch reports a null data pointer for a tensor with no elements)."""
    import ctypes
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    x = torch.ones((1, 512), dtype=torch.bfloat16, device="cuda")
    codes = torch.full((1, 256), 0x77, dtype=torch.uint8, device="cuda")
    scales = torch.full((B.scale_bytes(0, 512) or 1,), 0x55, dtype=torch.uint8, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    t = B.CTensor(codes.data_ptr(), scales.data_ptr(), g.data_ptr(), 0, 512, 256)
    assert lib.nvfp4_quantize(x.data_ptr(), 0, 512, 512, 1, ctypes.byref(t), stream) == B.OK
    torch.cuda.synchronize()
    assert g.item() == 1.0
    assert torch.all(codes == 0x77)          # no row to encode
    # the fused linear with an empty activation: nothing is launched, the output keeps its contents
    wq = B.quantize(rand_bf16(256, 512, 3).cuda())
    out = torch.full((1, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    desc = B.make_epilogue("bias")
    cw = wq.c()
    assert lib.nvfp4_linear(ctypes.byref(t), ctypes.byref(cw), ctypes.byref(desc), out.data_ptr(), 256, None,
                            stream) == B.OK
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
    B.check_device_error()
