"""GPU parity of the decode forms for a few tokens -- warp-level INT8 MMAs
(W4A8_KERNEL_WARP_MMA, the library's choice) and CUDA-core dp4a (an
ablation variant) -- against the CPU oracle and against the tcgen05 kernel:
INT32 accumulators
bit-exact, bf16 within 1 ulp of the oracle's FP64 epilogue and bit-identical
to the tensor-core kernel's (same accumulators, same fp32 epilogue).  Covers
one split and split-K clusters of 2..7 CTAs (ragged last split), ragged N,
group 128, zero rows, outliers, one k tile, the largest M, the header check,
chains with programmatic dependent launch, repeated runs, and the fused form
(fp32 activations quantized inside the kernel)."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from boundary_inputs import boundary_rows
from gpu_util import assert_bf16_within_1ulp, bf16_bits, check_block, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    assert w4.w4a8_get_status() == 0
    yield
    assert w4.w4a8_get_status() == 0


CASES = [
    # (M, N, K, group, activation kind)
    (1, 4096, 4096, 64, "normal"),     # one split, whole rows
    (2, 200, 384, 64, "normal"),       # ragged N, 3 k tiles
    (3, 256, 128, 64, "ties"),         # one k tile
    (4, 1024, 4224, 64, "heavy"),      # 33 k tiles: 2 splits, last one k tile
    (5, 384, 8192, 128, "normal"),     # group 128, 2 splits
    (6, 136, 11008, 64, "rowzero"),    # 86 k tiles: 3 splits (29, 29, 28), zero rows
    (7, 512, 28672, 64, "normal"),     # 224 k tiles: 7 splits
    (8, 640, 2048, 64, "heavy"),       # one group of 8 tokens, full
    (8, 8, 32768, 64, "normal"),       # 8 splits (the cluster limit), N < one slice
    (9, 4096, 4096, 64, "normal"),     # two token groups (warp-MMA form only)
    (13, 200, 11008, 64, "rowzero"),   # two groups, 3 splits, ragged N
    (16, 1024, 4096, 128, "ties"),     # largest M, group 128
]


def _inputs(M, N, K, group, kind, seed):
    X = wl.random_matrix(M, K, seed, std=1.0, kind=kind)
    W = wl.random_matrix(N, K, seed + 1, std=0.02)
    return X, W


FORMS = ["warp_mma", "dp4a"]


@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("M,N,K,group,kind", CASES)
def test_decode_form_matches_oracle_and_tensor_core(M, N, K, group, kind, form):
    if form == "dp4a" and M > 8:
        pytest.skip("the dp4a form takes at most 8 tokens")
    X, W = _inputs(M, N, K, group, kind, 700 + M + N + K)
    wq = oracle.quantize_weights(W.numpy(), group=group)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, wq, group=group)
    pk = w4.w4a8_quantize_weights(W.cuda(), group=group)
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    acc = w4.w4a8_gemm_variant(form, Xq, None, pk, i32=True)
    Y = w4.w4a8_gemm_variant(form, Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
    Yt = w4.w4a8_gemm_variant("tensor_core", Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    check_block(acc.cpu().numpy(), Y, acc_ref, y_ref, "%s M=%d N=%d K=%d" % (form, M, N, K))
    assert torch.equal(Y.view(torch.int16), Yt.view(torch.int16))


def test_default_dispatch_uses_the_decode_form_for_few_tokens():
    assert w4.w4a8_gemm_kernel_kind(1, 4096, 4096) == w4.KERNEL_WARP_MMA
    assert w4.w4a8_gemm_kernel_kind(256, 4096, 4096) == w4.KERNEL_TENSOR_CORE
    X, W = _inputs(2, 512, 1024, 64, "normal", 31)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    Y = w4.w4a8_gemm(Xq, sx, pk)
    Yd = w4.w4a8_gemm_variant("warp_mma", Xq, sx, pk)
    Yt = w4.w4a8_gemm(Xq, sx, pk, flags=w4.W4A8_FLAG_TENSOR_CORE)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Yd.view(torch.int16))
    assert torch.equal(Y.view(torch.int16), Yt.view(torch.int16))


@pytest.mark.parametrize("form,M", [("warp_mma", 17), ("dp4a", 9)])
def test_decode_form_refuses_shapes_outside_its_limits(form, M):
    pk = w4.w4a8_quantize_weights(torch.randn(128, 256, device="cuda") * 0.02)
    Xq = torch.zeros(M, 256, dtype=torch.int8, device="cuda")
    with pytest.raises(w4.W4A8Error) as e:
        w4.w4a8_gemm_variant(form, Xq, None, pk, i32=True)
    assert e.value.code == w4.ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("form", FORMS)
def test_decode_header_mismatch_is_reported_without_stores(form):
    W = wl.random_matrix(256, 256, 3, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    wrong = w4.PackedWeights(pk.data, 128, 256, 64)
    Xq = torch.ones(2, 256, dtype=torch.int8, device="cuda")
    out = torch.full((2, 128), 7, dtype=torch.int32, device="cuda")
    w4.w4a8_gemm_variant(form, Xq, None, wrong, i32=True, out=out)
    assert w4.w4a8_get_status() == w4.ERR_BAD_PACKED
    assert int((out != 7).sum()) == 0


@pytest.mark.parametrize("form", FORMS)
def test_decode_pdl_chain_and_repeated_runs(form):
    """Quantize -> GEMM chains with programmatic dependent launch, one split
    and a 3-CTA cluster, run repeatedly: the same bits every time as the
    plain launches."""
    for K in (4096, 11008):
        W = wl.random_matrix(384, K, 41 + K, std=0.02).cuda()
        pk = w4.w4a8_quantize_weights(W)
        Ms = (1, 3, 4, 8) + ((12, 16) if form == "warp_mma" else ())
        Xs = [wl.random_matrix(M, K, 50 + M, std=1.0).cuda() for M in Ms]
        torch.cuda.synchronize()
        ref = []
        for X in Xs:
            Xq, sx = w4.w4a8_quantize_act(X)
            ref.append(w4.w4a8_gemm_variant(form, Xq, sx, pk))
        torch.cuda.synchronize()
        for _ in range(20):
            outs = []
            for X in Xs:
                Xq, sx = w4.w4a8_quantize_act(X, flags=w4.W4A8_FLAG_PDL)
                outs.append(w4.w4a8_gemm_variant(form, Xq, sx, pk, flags=w4.W4A8_FLAG_PDL))
            torch.cuda.synchronize()
            for a, b in zip(outs, ref):
                assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert w4.w4a8_get_status() == 0


FUSED_CASES = [
    # (M, N, K, kind): one split (K <= 4096)
    (1, 4096, 4096, "normal"),
    (2, 4096, 4096, "heavy"),
    (4, 200, 512, "rowzero"),
    (8, 1024, 4096, "ties"),
    (3, 256, 128, "normal"),
    (16, 4096, 4096, "heavy"),
    (11, 200, 1024, "rowzero"),
]


@pytest.mark.parametrize("M,N,K,kind", FUSED_CASES)
def test_fused_decode_form_matches_two_calls_and_oracle(M, N, K, kind):
    assert w4.w4a8_gemm_fused_supported(M, N, K)
    X, W = _inputs(M, N, K, 64, kind, 900 + M + K)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xd = X.cuda()
    Y = w4.w4a8_gemm_fused(Xd, pk, flags=w4.W4A8_FLAG_PDL)
    Xq, sx = w4.w4a8_quantize_act(Xd)
    Y2 = w4.w4a8_gemm_variant("tensor_core", Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    _, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.numpy()))
    assert_bf16_within_1ulp(bf16_bits(Y), y_ref, "fused decode form M=%d N=%d K=%d" % (M, N, K))


def test_fused_decode_form_codes_at_rounding_boundaries():
    """Rows aimed at every rounding boundary of x / s_x, scales from 1e-39
    to 2e33: the fused kernel's in-kernel codes give the same output as the
    standalone quantizer followed by the product."""
    K = 4096
    X = torch.from_numpy(boundary_rows(K)).cuda()  # 6 rows
    W = wl.random_matrix(256, K, 77, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    Y = w4.w4a8_gemm_fused(X, pk)
    Xq, sx = w4.w4a8_quantize_act(X)
    acc = w4.w4a8_gemm_variant("tensor_core", Xq, None, pk, i32=True)
    Y2 = w4.w4a8_gemm_variant("tensor_core", Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    Xq_ref, sx_ref = oracle.quantize_act(X.cpu().numpy())
    acc_ref, _ = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.cpu().numpy()))
    assert np.array_equal(acc.cpu().numpy(), acc_ref)


@pytest.mark.parametrize("name,layer_name", [("decode_sweep_4096", "square"),
                                             ("llama7b_like", "qkv"),
                                             ("llama7b_like", "down"),
                                             ("llama70b_like", "down")])
def test_decode_form_full_size_layers(name, layer_name):
    """The decode layers at full size for M = 1..16 through the warp-MMA
    decode form: every output element against the oracle."""
    layer = [L for L in wl.WORKLOADS[name].layers if L.name == layer_name][0]
    N, K = layer.N, layer.K
    W = wl.layer_weights(name, layer)
    wq = oracle.quantize_weights(W.numpy())
    pk = w4.w4a8_quantize_weights(W.cuda())
    del W
    for M in (1, 2, 4, 8, 16):
        X = wl.make_activations(M, K, 1234 + M, 0.01, 20.0)
        Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
        acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, wq)
        Xq, sx = w4.w4a8_quantize_act(X.cuda())
        acc = w4.w4a8_gemm_variant("warp_mma", Xq, None, pk, i32=True)
        Y = w4.w4a8_gemm_variant("warp_mma", Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
        torch.cuda.synchronize()
        assert w4.w4a8_get_status() == 0
        check_block(acc.cpu().numpy(), Y, acc_ref, y_ref, "%s %s M=%d" % (name, layer_name, M))
