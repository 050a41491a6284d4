"""GPU parity of the W8A8 comparison kernel (INT8 weights, one scale per
channel, no dequantization) against the CPU oracle: INT8 weights and INT32
accumulators bit-exact, bf16 outputs within 1 bf16 ulp of the oracle's FP64
epilogue.  The shapes cover every tile width, split-K in both its push and
gather forms, ragged M and N, and the decode sweep at full size."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from gpu_util import assert_bf16_within_1ulp, bf16_bits, check_block, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    assert w4.w4a8_get_status() == 0
    yield
    assert w4.w4a8_get_status() == 0


@pytest.mark.parametrize("N,K,kind,seed", [(256, 512, "normal", 0), (200, 384, "rowzero", 1),
                                           (8, 128, "ties", 2), (128, 256, "heavy", 3),
                                           (64, 128, "zeros", 4)])
def test_w8_weight_quantization_bit_exact(N, K, kind, seed):
    W = wl.random_matrix(N, K, 3000 + seed, std=0.02, kind=kind)
    Wq_ref, sw_ref = oracle.w8a8_quantize_weights(W.numpy())
    Wq, sw = w4.w8a8_quantize_weights(W.cuda())
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    assert np.array_equal(sw.cpu().numpy(), sw_ref)


def _run(M, N, K, seed, wkind="normal", xkind="normal", flags=0):
    X = wl.random_matrix(M, K, 1000 + seed, std=1.0, kind=xkind)
    W = wl.random_matrix(N, K, 2000 + seed, std=0.02, kind=wkind)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Wq_ref, sw_ref = oracle.w8a8_quantize_weights(W.numpy())
    acc_ref, y_ref = oracle.w8a8_gemm(Xq_ref, sx_ref, Wq_ref, sw_ref)
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    Wq, sw = w4.w8a8_quantize_weights(W.cuda())
    acc = w4.w8a8_gemm_i32(Xq, Wq)
    Y = w4.w8a8_gemm(Xq, sx, Wq, sw, flags=flags)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    return acc.cpu().numpy(), bf16_bits(Y), acc_ref, y_ref


SHAPES = [
    (16, 256, 512),     # one 16-token tile
    (1, 128, 128),      # one tile, one k block
    (1, 256, 4096),     # decode: split-K, push reduction
    (8, 512, 4096),     # push reduction at its largest M
    (12, 256, 4096),    # split-K, gather reduction
    (3, 200, 384),      # ragged N and M
    (17, 256, 1024),    # 32-token tile
    (33, 384, 2048),    # 64-token tile
    (100, 136, 512),    # 256-token tile, ragged N
    (300, 256, 512),    # two token tiles of 256
    (513, 128, 128),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_w8a8_gemm_parity(M, N, K):
    acc, y, acc_ref, y_ref = _run(M, N, K, seed=M * 5 + N + K)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref, "W8A8 M=%d N=%d K=%d" % (M, N, K))


@pytest.mark.parametrize("wkind,xkind", [("rowzero", "rowzero"), ("ties", "ties"),
                                         ("heavy", "heavy"), ("zeros", "normal")])
def test_w8a8_value_patterns(wkind, xkind):
    acc, y, acc_ref, y_ref = _run(40, 256, 512, seed=21, wkind=wkind, xkind=xkind)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref)


def test_w8a8_int32_extremes():
    """|acc| up to K * 127 * 127 with every product the same sign."""
    M, N, K = 4, 128, 8192
    Xq = torch.full((M, K), 127, dtype=torch.int8, device="cuda")
    Xq[1] = -127
    Wq = torch.full((N, K), 127, dtype=torch.int8, device="cuda")
    Wq[5] = -127
    acc = w4.w8a8_gemm_i32(Xq, Wq).cpu().numpy()
    ref = oracle.gemm_i32(Xq.cpu().numpy(), Wq.cpu().numpy())
    assert np.array_equal(acc, ref) and abs(int(ref.max())) == K * 127 * 127


def test_w8a8_pdl_flag_matches_plain():
    acc, y, acc_ref, y_ref = _run(4, 512, 2048, seed=31, flags=w4.W4A8_FLAG_PDL)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref)


def test_w8a8_host_side_rejections():
    L = w4.lib()
    Xq = torch.zeros(4, 256, dtype=torch.int8, device="cuda")
    Wq = torch.zeros(128, 256, dtype=torch.int8, device="cuda")
    sx = torch.ones(4, device="cuda")
    sw = torch.ones(128, device="cuda")
    Y = torch.empty(4, 128, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    p = lambda t: t.data_ptr()
    assert L.w8a8_gemm(p(Xq), p(sx), p(Wq), p(sw), 4, 128, 200, p(Y), 0, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w8a8_gemm(p(Xq), p(sx), p(Wq) + 8, p(sw), 4, 128, 256, p(Y), 0, st) == w4.ERR_MISALIGNED
    assert L.w8a8_gemm(p(Xq), p(sx), p(Wq), None, 4, 128, 256, p(Y), 0, st) == w4.ERR_INVALID_ARG
    assert L.w8a8_gemm(p(Xq), p(sx), p(Wq), p(sw), 4, 128, 256, p(Y), 2, st) == w4.ERR_INVALID_ARG
    assert L.w8a8_gemm(p(Xq), p(sx), p(Wq), p(sw), 0, 128, 256, p(Y), 0, st) == w4.OK
    assert w4.w4a8_get_status() == 0


@pytest.mark.parametrize("M", [1, 8, 16, 64, 256])
def test_w8a8_decode_sweep_full_size(M):
    """N = K = 4096 (the decode sweep) in the schedule the benchmark times:
    every output element against the oracle's W8A8 product."""
    N = K = 4096
    layer = wl.WORKLOADS["decode_sweep_4096"].layers[0]
    W = wl.layer_weights("decode_sweep_4096", layer)
    X = wl.layer_activations("decode_sweep_4096", layer, M)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Wq_ref, sw_ref = oracle.w8a8_quantize_weights(W.numpy())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    Wq, sw = w4.w8a8_quantize_weights(W.cuda())
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    acc = w4.w8a8_gemm_i32(Xq, Wq)
    Y = w4.w8a8_gemm(Xq, sx, Wq, sw, flags=w4.W4A8_FLAG_PDL)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    acc_ref, y_ref = oracle.w8a8_gemm(Xq_ref, sx_ref, Wq_ref, sw_ref)
    check_block(acc.cpu().numpy(), Y, acc_ref, y_ref, "W8A8 sweep M=%d" % M)
