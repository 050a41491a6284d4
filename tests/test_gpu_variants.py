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
    assert L.w4a8_gemm_variant(11, None, None, None, 0, 128, 256, None, None, 0, st) == w4.ERR_INVALID_ARG
    x = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.w4a8_gemm_variant(1, None, None, None, 1, 128, 256, x.data_ptr(), x.data_ptr(), 0, st) == w4.ERR_INVALID_ARG


@pytest.mark.parametrize("M,N,K,kind", [(256, 256, 512, "normal"),     # one CTA pair
                                        (512, 512, 1024, "heavy"),     # 2 token tiles x 2 pairs
                                        (1000, 256, 2048, "ties"),     # ragged last token tile
                                        (256, 1024, 128, "normal"),    # one k tile
                                        (300, 512, 1024, "normal"),    # 2 tiles of 160 (runtime width)
                                        (600, 256, 512, "heavy")])     # 3 tiles of 224 (runtime width)
def test_cta_pair_variant_parity(M, N, K, kind):
    pk, Xq, sx, acc_ref, y_ref = _case(M, N, K, kind)
    acc = w4.w4a8_gemm_variant("cta_pair", Xq, None, pk, i32=True)
    Y = w4.w4a8_gemm_variant("cta_pair", Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "cta_pair M=%d" % M)


def test_cta_pair_needs_even_channel_blocks():
    pk, Xq, sx, _, _ = _case(256, 384, 256, "normal")   # 3 channel blocks
    with pytest.raises(w4.W4A8Error) as e:
        w4.w4a8_gemm_variant("cta_pair", Xq, sx, pk)
    assert e.value.code == w4.ERR_UNSUPPORTED_SHAPE


def test_default_path_takes_the_cta_pair_at_large_m():
    """A prefill-like shape runs the pair form by default (splits 1, 256-token
    tiles, even channel blocks) and matches the oracle."""
    M, N, K = 2048, 2048, 1024
    assert w4.w4a8_gemm_schedule(M, N, K)[:2] == (256, 1)
    pk, Xq, sx, acc_ref, y_ref = _case(M, N, K, "normal")
    acc = w4.w4a8_gemm_i32(Xq, pk)
    Y = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "default pair")


def test_cta_pair_repeated_runs_are_identical():
    """The pair's cross-CTA hand-off (the odd CTA's weight slots and token
    half feed the even CTA's MMAs) gives the same bits run after run."""
    M, N, K = 1024, 1024, 4096
    pk, Xq, sx, acc_ref, _ = _case(M, N, K, "normal")
    for _ in range(6):
        acc = w4.w4a8_gemm_variant("cta_pair", Xq, None, pk, i32=True)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert w4.w4a8_get_status() == 0


PERSISTENT_CASES = [
    # (M, N, K, group, kind)
    (300, 256, 512, 64, "normal"),     # one pair, two tiles (192 + 108 tokens)
    (1000, 512, 2048, 64, "heavy"),    # 6 token tiles x 2 pairs, last tile 40 rows
    (4100, 1024, 1024, 64, "ties"),    # 22 token tiles x 4 pairs: some pairs take two rounds
    (16, 256, 256, 64, "rowzero"),     # a single small tile
    (500, 200, 384, 128, "normal"),    # ragged N (padded to one pair), group 128
    (192, 256, 128, 64, "normal"),     # exactly one tile, one k tile
]


@pytest.mark.parametrize("M,N,K,group,kind", PERSISTENT_CASES)
def test_persistent_pair_parity(M, N, K, group, kind):
    """The persistent CTA-pair form (double-buffered accumulators, epilogue
    overlapped with the next tile): INT32 bit-exact, bf16 within 1 ulp of the
    oracle and bit-identical to the non-persistent kernels."""
    X = wl.random_matrix(M, K, 300 + M, std=1.0, kind=kind)
    W = wl.random_matrix(N, K, 301 + N + K, std=0.02)
    wq = oracle.quantize_weights(W.numpy(), group=group)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, wq, group=group)
    pk = w4.w4a8_quantize_weights(W.cuda(), group=group)
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    acc = w4.w4a8_gemm_variant("persistent", Xq, None, pk, i32=True)
    Y = w4.w4a8_gemm_variant("persistent", Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
    Yb = w4.w4a8_gemm_variant("baseline", Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "persistent M=%d N=%d K=%d" % (M, N, K))
    assert torch.equal(Y.view(torch.int16), Yb.view(torch.int16))


def test_persistent_pair_repeated_runs_match_default():
    """Many tiles per pair (phases carried across tiles), run repeatedly in a
    PDL chain: the same bits every time, and the same bits as the default
    call (the per-tile CTA-pair kernel)."""
    M, N, K = 3000, 2048, 1024
    X = wl.random_matrix(M, K, 17, std=1.0)
    W = wl.random_matrix(N, K, 18, std=0.02)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    ref = w4.w4a8_gemm_variant("baseline", Xq, sx, pk)
    torch.cuda.synchronize()
    for _ in range(10):
        outs = [w4.w4a8_gemm_variant("persistent", Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
                for _ in range(3)]
        torch.cuda.synchronize()
        for Y in outs:
            assert torch.equal(Y.view(torch.int16), ref.view(torch.int16))
    assert w4.w4a8_get_status() == 0
    Yd = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert torch.equal(Yd.view(torch.int16), ref.view(torch.int16))


def test_persistent_pair_refusals():
    pk, Xq, sx, _, _ = _case(256, 384, 256, "normal")   # 3 channel blocks: no pairs
    with pytest.raises(w4.W4A8Error) as e:
        w4.w4a8_gemm_variant("persistent", Xq, None, pk, i32=True)
    assert e.value.code == w4.ERR_UNSUPPORTED_SHAPE
