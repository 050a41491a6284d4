"""GPU parity of the ablation study's kernel variants: every variant
computes exactly the library's product (INT32 bit-exact against the oracle,
bf16 within 1 ulp), on both tile widths, with and without split-K."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from gpu_util import assert_bf16_within_1ulp, bf16_bits, require_gpu

pytestmark = pytest.mark.gpu

VARIANTS = ["baseline", "naive_dequant", "serial", "one_group", "group_issues_mma"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    assert w4.w4a8_get_status() == 0
    yield
    assert w4.w4a8_get_status() == 0


_cache = {}


def _case(M, N, K, kind):
    key = (M, N, K, kind)
    if key not in _cache:
        X = wl.random_matrix(M, K, 600 + M + K, std=1.0, kind="normal")
        W = wl.random_matrix(N, K, 700 + N + K, std=0.02, kind=kind)
        Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
        acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.numpy()))
        pk = w4.w4a8_quantize_weights(W.cuda())
        Xq, sx = w4.w4a8_quantize_act(X.cuda())
        _cache.clear()
        _cache[key] = (pk, Xq, sx, acc_ref, y_ref)
    return _cache[key]


@pytest.mark.parametrize("M,N,K,kind", [(1, 256, 4096, "normal"),    # 16-token tile, split-K
                                        (16, 384, 1024, "heavy"),    # 16-token tile, s_u8 up to 16
                                        (40, 256, 2048, "normal"),   # 256-token tile, split-K
                                        (300, 200, 512, "ties")])    # two 256-token tiles, ragged N
@pytest.mark.parametrize("variant", VARIANTS)
def test_variant_parity(variant, M, N, K, kind):
    pk, Xq, sx, acc_ref, y_ref = _case(M, N, K, kind)
    acc = w4.w4a8_gemm_variant(variant, Xq, None, pk, i32=True)
    Y = w4.w4a8_gemm_variant(variant, Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "%s M=%d" % (variant, M))


def test_variant_rejections():
    L = w4.lib()
    st = torch.cuda.current_stream().cuda_stream
    assert L.w4a8_gemm_variant(9, None, None, None, 0, 128, 256, None, None, 0, st) == w4.ERR_INVALID_ARG
    x = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.w4a8_gemm_variant(1, None, None, None, 1, 128, 256, x.data_ptr(), x.data_ptr(), 0, st) == w4.ERR_INVALID_ARG
