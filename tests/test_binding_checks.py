"""The Python binding checks its tensor arguments before anything reaches
CUDA: host tensors, wrong dtypes, wrong shapes, undersized output buffers
and foreign objects raise TypeError or ValueError (here, with no GPU, the
call would otherwise fail later or hand a host pointer to a kernel)."""
import pytest
import torch


@pytest.fixture(scope="module")
def ql():
    from bit_quantized_linear_block_b200 import qlinear
    return qlinear


def _bf16(*shape):
    return torch.zeros(*shape, dtype=torch.bfloat16)


def test_host_tensors_are_rejected(ql):
    x = _bf16(4, 128)
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_route(x, x)
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_gamma_sums(x, x)
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_route_from_sums(torch.zeros(2, dtype=torch.float64))
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_tensor_amax(x)
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_quantize_act(x, ql.QL_ROUTE_NVFP4)
    with pytest.raises(ValueError, match="CUDA"):
        ql.qlinear_prepare_weights(_bf16(16, 128))


def test_wrong_dtypes_and_shapes_are_rejected(ql):
    with pytest.raises(TypeError, match="bfloat16"):
        ql.qlinear_route(torch.zeros(8), torch.zeros(8))
    with pytest.raises(TypeError, match="float64"):
        ql.qlinear_route_from_sums(torch.zeros(2, dtype=torch.float32))
    with pytest.raises(TypeError, match="Tensor"):
        ql.qlinear_tensor_amax([[0.0] * 128])
    with pytest.raises(TypeError, match="bfloat16"):
        ql.qlinear_prepare_weights(torch.zeros(16, 128))


def test_weights_must_be_packed(ql):
    with pytest.raises(TypeError, match="PackedWeights"):
        ql.qlinear_gemm(ql.QL_ROUTE_NVFP4, {"codes": torch.zeros(1)}, 1, object())
    with pytest.raises(TypeError, match="PackedWeights"):
        ql.ForwardPlan(4, "weights", ql.QL_ROUTE_NVFP4, "cpu")


def test_activation_buffer_sizes(ql):
    """Sizes of the quantized-activation buffers, as the C ABI lays them out:
    NVFP4 codes K/2 bytes per row (K for the decomposed pair) with scales in
    the MMA layout; integer codes one int8 or f16 per element with one fp32
    scale per row; the Q-ARVD codes Kp bytes per row with one scale."""
    M, K = 300, 640
    b = ql._act_bytes(M, K, ql.QL_ROUTE_NVFP4)
    assert b == dict(codes=M * K // 2, sf_mma=ql.lib.qlinear_sf_bytes(M, K), sf_rowmajor=M * K // 16, scales=4)
    b = ql._act_bytes(M, K, ql.QL_ACT_NVFP4_DECOMP)
    assert b["codes"] == M * K and b["sf_mma"] == ql.lib.qlinear_sf_bytes(M, 2 * K)
    assert b["sf_rowmajor"] == M * 2 * K // 16
    for fmt in (ql.QL_ROUTE_INT8, ql.QL_ROUTE_INT6):
        assert ql._act_bytes(M, K, fmt) == dict(codes=M * K, sf_mma=None, sf_rowmajor=None, scales=4 * M)
    for fmt in (ql.QL_ACT_INT8_F16, ql.QL_ACT_INT6_F16):
        assert ql._act_bytes(M, K, fmt)["codes"] == 2 * M * K
    assert ql._act_bytes(0, K, ql.QL_ROUTE_INT8)["scales"] == 4          # one scale slot even when empty
    assert ql._act_bytes(M, K, ql.QL_ROUTE_BF16) == dict(codes=2 * M * K, sf_mma=None, sf_rowmajor=None,
                                                        scales=None)
    with pytest.raises(ValueError, match="Q-ARVD"):
        ql._act_bytes(M, K, ql.QL_ACT_INT8_TENSOR)
    with pytest.raises(ValueError, match="unknown"):
        ql._act_bytes(M, K, 99)


def test_unknown_activation_format_is_rejected_first(ql):
    with pytest.raises(ValueError, match="CUDA"):      # the input check comes first
        ql.qlinear_quantize_act(_bf16(4, 128), 99)
