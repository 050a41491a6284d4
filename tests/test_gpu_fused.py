"""GPU parity of the fused activation-quantization + GEMM entry point
(w4a8_gemm_fused): the bf16 output must be bit-identical to the two-call
path (w4a8_quantize_act then w4a8_gemm), and the INT8 codes and scales it
writes must be bit-exact against the CPU oracle.  Shapes cover the fused
kernel (16- and 32-token tiles, with and without split-K, push and gather
reductions) and the fallback to the two kernels."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
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
    # (M, N, K, kind)
    (1, 4096, 4096, "normal"),    # 16-token tile, split 8, push reduction
    (3, 200, 384, "normal"),      # ragged N, few k tiles
    (8, 4096, 4096, "heavy"),     # push reduction, outliers
    (9, 4096, 4096, "normal"),    # 16-token tile, gather reduction
    (16, 1024, 2048, "rowzero"),  # zero token rows
    (17, 4096, 4096, "ties"),     # 32-token tile
    (32, 256, 8192, "normal"),    # 32-token tile, long K
    (1, 2048, 8192, "normal"),    # no split when few tiles need it? (schedule decides)
    (2, 28672, 512, "normal"),    # many channel blocks, one k tile per CTA
    (33, 512, 1024, "normal"),    # falls back to two kernels
    (16, 28672, 8192, "normal"),  # fused reads too large: falls back
]


@pytest.mark.parametrize("M,N,K,kind", CASES)
def test_fused_matches_two_calls_and_oracle(M, N, K, kind):
    X = wl.random_matrix(M, K, 300 + M + K, std=1.0, kind=kind)
    W = wl.random_matrix(N, K, 400 + N, std=0.02)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xd = X.cuda()
    Y, Xq, sx = w4.w4a8_gemm_fused(Xd, pk)
    xq2, sx2 = w4.w4a8_quantize_act(Xd)
    Y2 = w4.w4a8_gemm(xq2, sx2, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    # and against the oracle on sampled outputs
    rng = np.random.default_rng(M + N)
    ms = rng.integers(0, M, 128)
    ns = rng.integers(0, N, 128)
    wq = oracle.quantize_weights(W.numpy())
    _, y_ref = oracle.w4a8_gemm_sampled(Xq_ref, sx_ref, wq, ms, ns)
    assert_bf16_within_1ulp(bf16_bits(Y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()]), y_ref)


def test_fused_pdl_chain_repeated():
    """Fused calls chained with programmatic dependent launch, repeated: the
    same bits every time (cluster absmax exchange and reductions included)."""
    K = 4096
    W = wl.random_matrix(4096, K, 7, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    Xs = [wl.random_matrix(M, K, 70 + M).cuda() for M in (1, 2, 4, 8, 16, 32)]
    ref = []
    for X in Xs:
        xq, s = w4.w4a8_quantize_act(X)
        ref.append(w4.w4a8_gemm(xq, s, pk).clone())
    for rep in range(3):
        outs = [w4.w4a8_gemm_fused(X, pk, flags=w4.W4A8_FLAG_PDL)[0] for X in Xs]
        torch.cuda.synchronize()
        for a, b in zip(outs, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert w4.w4a8_get_status() == 0
