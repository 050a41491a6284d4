"""GPU parity of the grouped (mixture-of-experts) W4A8 GEMM against the CPU
oracle: INT32 accumulators bit-exact and bf16 outputs within 1 bf16 ulp,
for group layouts with empty experts, groups longer than one token tile,
split-K decode (push and gather reductions) and the Mixtral-like layers at
full size; invalid row offsets are reported without any store."""
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


def _run(counts, N, K, seed, max_rows=None, flags=0):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    X = wl.random_matrix(M, K, 4000 + seed, std=1.0)
    Ws = [wl.random_matrix(N, K, 5000 + 17 * seed + g, std=0.02) for g in range(E)]
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    wqs = [oracle.quantize_weights(W.numpy()) for W in Ws]
    acc_ref, y_ref = oracle.w4a8_grouped_gemm(Xq_ref, sx_ref, wqs, offsets)
    gw = w4.w4a8_quantize_grouped_weights(torch.stack(Ws).cuda())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    off = torch.from_numpy(offsets).cuda()
    mr = max(counts) if max_rows is None else max_rows
    acc = w4.w4a8_grouped_gemm_i32(Xq, gw, off, max_rows=mr)
    Y = w4.w4a8_grouped_gemm(Xq, sx, gw, off, max_rows=mr, flags=flags)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    return acc.cpu().numpy(), bf16_bits(Y), acc_ref, y_ref


CASES = [
    # (rows per expert, N, K)
    ([1, 0, 2, 0, 0, 1, 0, 0], 512, 4096),    # decode: split-K, push reduction
    ([3, 9, 0, 12], 256, 4096),                # split-K, gather reduction (max 12 rows)
    ([17, 0, 40, 3], 384, 1024),               # 64-token tiles, empty expert
    ([300, 5, 0], 256, 512),                   # 256-token tiles, two tiles in one group
    ([10, 10, 10], 200, 384),                  # ragged N
    ([0, 0, 7], 128, 128),                     # only the last expert has rows
    ([33], 256, 256),                          # one group = a dense GEMM
    ([150, 90, 0, 200], 4096, 1024),           # 208-token tiles (runtime width), no split
]


@pytest.mark.parametrize("counts,N,K", CASES)
def test_grouped_gemm_parity(counts, N, K):
    acc, y, acc_ref, y_ref = _run(counts, N, K, seed=len(counts) * 3 + N + K)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref, "grouped %s N=%d K=%d" % (counts, N, K))


def test_grouped_gemm_loose_row_bound_and_pdl():
    """max_rows may exceed every group's rows (tiles past them exit)."""
    acc, y, acc_ref, y_ref = _run([5, 2, 9], 256, 1024, seed=41, max_rows=16,
                                  flags=w4.W4A8_FLAG_PDL)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref)


def test_grouped_gemm_matches_dense_calls_per_expert():
    """The grouped call equals one dense call per expert on its rows."""
    counts, N, K = [6, 0, 20, 1], 256, 2048
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    X = wl.random_matrix(int(offsets[-1]), K, 77).cuda()
    W = torch.stack([wl.random_matrix(N, K, 78 + g, std=0.02) for g in range(4)]).cuda()
    gw = w4.w4a8_quantize_grouped_weights(W)
    Xq, sx = w4.w4a8_quantize_act(X)
    Y = w4.w4a8_grouped_gemm(Xq, sx, gw, torch.from_numpy(offsets).cuda(), max_rows=20)
    for g in range(4):
        r0, r1 = int(offsets[g]), int(offsets[g + 1])
        if r1 > r0:
            Yd = w4.w4a8_gemm(Xq[r0:r1].contiguous(), sx[r0:r1].contiguous(), gw.expert(g))
            assert torch.equal(Y[r0:r1].view(torch.int16), Yd.view(torch.int16))
    assert w4.w4a8_get_status() == 0


@pytest.mark.parametrize("offsets", [[0, 5, 3, 8],      # out of order
                                     [0, 2, 4, 9],      # last offset past M_total
                                     [0, 1, 8, 8]])     # a group longer than max_rows
def test_grouped_gemm_bad_offsets_reported(offsets):
    N, K, M = 256, 512, 8
    gw = w4.w4a8_quantize_grouped_weights(torch.stack(
        [wl.random_matrix(N, K, 90 + g, std=0.02) for g in range(3)]).cuda())
    Xq, sx = w4.w4a8_quantize_act(wl.random_matrix(M, K, 93).cuda())
    off = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    Y = w4.w4a8_grouped_gemm(Xq, sx, gw, off, max_rows=5)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == w4.ERR_BAD_OFFSETS
    assert w4.w4a8_get_status() == 0   # read-and-clear
    del Y


def test_grouped_host_side_rejections():
    L = w4.lib()
    st = torch.cuda.current_stream().cuda_stream
    off = torch.zeros(3, dtype=torch.int32, device="cuda")
    p = lambda t: t.data_ptr()
    assert L.w4a8_grouped_gemm(None, None, None, 0, p(off), 4, 2, 128, 256, None, 0, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_grouped_gemm(None, None, None, 2, p(off), 4, 5, 128, 256, None, 0, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_grouped_gemm(None, None, None, 2, p(off) + 2, 4, 2, 128, 256, p(off), 0, st) == w4.ERR_MISALIGNED
    assert L.w4a8_grouped_gemm(None, None, None, 2, None, 0, 0, 128, 256, None, 0, st) == w4.OK
    assert w4.w4a8_get_status() == 0


@pytest.mark.parametrize("layer_name,tokens", [("down", 16), ("gate_up", 1), ("down", 512)])
def test_mixtral_like_full_size(layer_name, tokens):
    """The Mixtral-like expert layers at full size, in the benchmark's
    schedule: every output element against the grouped oracle product."""
    name = "mixtral_like"
    w = wl.MOE_WORKLOADS[name]
    layer = [L for L in w.layers if L.name == layer_name][0]
    N, K = layer.N, layer.K
    offsets, tok = wl.moe_routing(name, tokens)
    X = wl.moe_activations(name, layer, tokens)[tok].contiguous()
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    wqs, gdata = [], []
    b = w4.w4a8_packed_weight_bytes(N, K)
    data = torch.empty(w.experts * b, dtype=torch.uint8, device="cuda")
    for e in range(w.experts):
        We = wl.moe_expert_weights(name, layer, e)
        wqs.append(oracle.quantize_weights(We.numpy()))
        w4.w4a8_quantize_weights(We.cuda(), out=data[e * b:(e + 1) * b])
        del We
    gw = w4.GroupedPackedWeights(data, w.experts, N, K, 64)
    off = offsets.cuda()
    mr = int((offsets[1:] - offsets[:-1]).max())
    acc = w4.w4a8_grouped_gemm_i32(Xq, gw, off, max_rows=mr)
    Y = w4.w4a8_grouped_gemm(Xq, sx, gw, off, max_rows=mr, flags=w4.W4A8_FLAG_PDL)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    acc_ref, y_ref = oracle.w4a8_grouped_gemm(Xq_ref, sx_ref, wqs, offsets.numpy())
    check_block(acc.cpu().numpy(), Y, acc_ref, y_ref,
                "mixtral %s tokens=%d" % (layer_name, tokens))


def test_grouped_prefill_shape_uses_the_wide_tile():
    """The case above runs without split-K on the 256-token configuration,
    its tile width sized to the largest group."""
    T, splits, _ = w4.w4a8_grouped_gemm_schedule(4, 440, 200, 4096, 1024)
    assert (T, splits) == (256, 1)
