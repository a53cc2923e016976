"""The fused linear's plain product against cuBLASLt's NVFP4 GEMM (torch scaled_mm), an implementation
independent of both this library and the oracle.

The library's block-scale layout is the 32 x 4 x 4 atom layout cuBLASLt reads, so both consume the same
quantised bytes: E2M1 codes, E4M3 scales per 16 elements and the fp32 tensor scales (cuBLASLt's
TensorWise second level).  On these shapes both accumulate each K = 64 block product in fp32 in K order
and round once to bf16, and the outputs are identical bit for bit."""
import pytest
import torch

pytestmark = pytest.mark.gpu

SHAPES = [(4608, 13824, 4608), (4608, 4608, 12288)]  # QKV and down projections at 1024^2


def _cublaslt_nvfp4(xq, wq):
    import torch.nn.functional as F
    recipe = [F.ScalingType.BlockWise1x16, F.ScalingType.TensorWise]
    swz = [F.SwizzleType.SWIZZLE_32_4_4, F.SwizzleType.NO_SWIZZLE]
    return F.scaled_mm(xq.codes.view(torch.float4_e2m1fn_x2), wq.codes.view(torch.float4_e2m1fn_x2).t(),
                       [xq.scales.view(torch.float8_e4m3fn), xq.g], recipe,
                       [wq.scales.view(torch.float8_e4m3fn), wq.g], recipe,
                       swizzle_a=swz, swizzle_b=swz, output_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_plain_product_is_bit_identical_to_cublaslt(M, N, K):
    from epilogue_gemm_nvfp4_b200 import binding as B
    gen = torch.Generator(device="cuda").manual_seed(3)
    xq = B.quantize(torch.randn(M, K, device="cuda", dtype=torch.bfloat16, generator=gen))
    wq = B.quantize(torch.randn(N, K, device="cuda", dtype=torch.bfloat16, generator=gen) * 0.02)
    ours = B.linear(xq, wq, "bias", bias=torch.zeros(N, device="cuda", dtype=torch.bfloat16))
    torch.cuda.synchronize()
    B.check_device_error()
    try:
        ref = _cublaslt_nvfp4(xq, wq)
    except (AttributeError, RuntimeError, TypeError) as e:
        pytest.skip(f"torch has no NVFP4 scaled_mm here: {type(e).__name__}: {e}")
    assert ours.shape == ref.shape
    diff = (ours.float() - ref.float()).abs().max().item()
    assert torch.equal(ours, ref), f"largest difference {diff}"
