"""GPU parity of the fused decode path (activation quantization inside the
GEMM): bf16 outputs bit-identical to w4a8_quantize_act + w4a8_gemm (same
codes, scales and accumulation) and within 1 bf16 ulp of the oracle, with
split-K push, a single split, ragged N, zero rows, rounding ties and
outliers, up to the largest slice of X the kernel holds in registers."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from boundary_inputs import boundary_rows
from gpu_util import assert_bf16_within_1ulp, bf16_bits, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    assert w4.w4a8_get_status() == 0
    yield
    assert w4.w4a8_get_status() == 0


CASES = [
    # (M, N, K, activation kind)
    (1, 4096, 4096, "normal"),     # split 8, push
    (2, 4096, 4096, "heavy"),      # outliers widen the scale
    (4, 4096, 4096, "rowzero"),    # largest register slice with split-K, zero rows
    (3, 200, 512, "normal"),       # ragged N
    (5, 256, 768, "ties"),         # values on rounding ties
    (8, 5000, 256, "normal"),      # largest pushed tile, ragged N
    (4, 28672, 512, "normal"),     # one split, largest register slice
    (2, 28672, 768, "heavy"),      # one split, 6 k tiles
    (16, 28672, 128, "rowzero"),   # one split, full token tile
    (1, 1024, 128, "ties"),        # one k tile
]


@pytest.mark.parametrize("core", ["library", "tensor_core"])
@pytest.mark.parametrize("M,N,K,kind", CASES)
def test_fused_matches_two_calls_and_oracle(M, N, K, kind, core):
    """``library``: the library's choice (the CUDA-core form where it applies);
    ``tensor_core``: the tensor-core fused kernel forced by its flag."""
    assert w4.w4a8_gemm_fused_supported(M, N, K), (M, N, K, w4.w4a8_gemm_schedule(M, N, K))
    X = wl.random_matrix(M, K, 8000 + M + K, std=1.0, kind=kind)
    W = wl.random_matrix(N, K, 9000 + N + K, std=0.02)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xd = X.cuda()
    flags = w4.W4A8_FLAG_PDL | (w4.W4A8_FLAG_TENSOR_CORE if core == "tensor_core" else 0)
    Y = w4.w4a8_gemm_fused(Xd, pk, flags=flags)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    Xq, sx = w4.w4a8_quantize_act(Xd)
    Y2 = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    _, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.numpy()))
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "fused M=%d N=%d K=%d" % (M, N, K))


@pytest.mark.parametrize("absmax", [(1.0, 7.5e4), (1.0e-30,), (3.0e-3, 2.0e33)])
def test_fused_codes_at_rounding_boundaries(absmax):
    # activations a few ulps either side of the quantizer's rounding
    # boundaries: the fused kernel's codes (seen through the outputs) must be
    # the quantizer kernel's, and the outputs the oracle's
    N, K = 4096, 4352
    X = boundary_rows(K, absmax)
    M = X.shape[0]
    assert w4.w4a8_gemm_fused_supported(M, N, K)
    W = wl.random_matrix(N, K, 77, std=0.02)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xd = torch.from_numpy(X).cuda()
    Y = w4.w4a8_gemm_fused(Xd, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    Xq, sx = w4.w4a8_quantize_act(Xd)
    Y2 = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    Xq_ref, sx_ref = oracle.quantize_act(X)
    _, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.numpy()))
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "fused boundary rows %s" % (absmax,))


def test_fused_unsupported_shapes_are_rejected_before_launch():
    W = wl.random_matrix(256, 4096, 1, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    # 17 and 64 tokens: past the 16-token tile and the decode form's limit
    for M in (17, 64):
        assert not w4.w4a8_gemm_fused_supported(M, 256, 4096)
        with pytest.raises(w4.W4A8Error) as e:
            w4.w4a8_gemm_fused(torch.zeros(M, 4096, device="cuda"), pk)
        assert e.value.code == w4.ERR_UNSUPPORTED_SHAPE
    # 8 and 16 tokens over 4096 k: the decode form only (the tensor-core
    # fused kernel cannot hold the CTA's slice of X in its registers)
    for M in (8, 16):
        assert w4.w4a8_gemm_fused_supported(M, 256, 4096)
        with pytest.raises(w4.W4A8Error) as e:
            w4.w4a8_gemm_fused(torch.zeros(M, 4096, device="cuda"), pk,
                               flags=w4.W4A8_FLAG_TENSOR_CORE)
        assert e.value.code == w4.ERR_UNSUPPORTED_SHAPE
    assert w4.w4a8_get_status() == 0
