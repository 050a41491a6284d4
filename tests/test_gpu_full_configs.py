"""GPU parity at the full sizes of the five synthetic workloads (tiny, decode
sweep N=K=4096, 7B-like layers, 70B-like layers, prefill), in the schedule
the benchmark times.

Everything the oracle can afford at full size is compared whole: the packed
weights (unpacked) and the INT8 activations are bit-exact.  The INT32
accumulators and bf16 outputs are compared on sampled positions (corners,
ragged tile edges and seeded random picks) computed one by one by the
oracle, and every accumulator takes part in two exact integer invariants
that hold at any size: row sums  sum_n acc[m,n] = Xq[m] . colsum_n(W8)  and
column sums  sum_m acc[m,n] = W8[n] . colsum_m(Xq).
"""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from gpu_util import assert_bf16_within_1ulp, bf16_bits, require_gpu

pytestmark = pytest.mark.gpu

_weights = {}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    yield
    _weights.clear()
    torch.cuda.empty_cache()


def _layer(name, layer):
    key = (name, layer.name)
    if key not in _weights:
        _weights.clear()
        torch.cuda.empty_cache()
        W = wl.layer_weights(name, layer)
        ref = oracle.quantize_weights(W.numpy())
        pk = w4.w4a8_quantize_weights(W.cuda())
        u = w4.w4a8_unpack_weights(pk)
        for k in ("codes", "s_u8", "a", "s_w"):
            assert np.array_equal(u[k].cpu().numpy(), ref[k]), (name, layer.name, k)
        del u
        W8 = oracle.dequant_weights(ref["codes"], ref["s_u8"], ref["a"])
        colsum_w = W8.sum(axis=0, dtype=np.int64)
        _weights[key] = (ref, pk, W8, colsum_w)
    return _weights[key]


def _samples(M, N, rng, count=384):
    ms = [0, M - 1, min(M - 1, 15), min(M - 1, 16), M // 2]
    ns = [0, N - 1, min(N - 1, 127), min(N - 1, 128), N // 2]
    pts = [(m, n) for m in ms for n in ns]
    pts += list(zip(rng.integers(0, M, count).tolist(), rng.integers(0, N, count).tolist()))
    a = np.array(pts, dtype=np.int64)
    return a[:, 0], a[:, 1]


def _all_cases():
    out = []
    for name in wl.WORKLOADS:
        for M, layer in wl.cases(name):
            out.append(pytest.param(name, M, layer, id="%s-%s-M%d" % (name, layer.name, M)))
    return out


@pytest.mark.parametrize("name,M,layer", _all_cases())
def test_full_size_case(name, M, layer):
    ref_w, pk, W8, colsum_w = _layer(name, layer)
    N, K = layer.N, layer.K
    X = wl.layer_activations(name, layer, M)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)
    del X

    acc = w4.w4a8_gemm_i32(Xq, pk)
    Y = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0

    rng = np.random.default_rng(M * 31 + N)
    ms, ns = _samples(M, N, rng)
    acc_ref, y_ref = oracle.w4a8_gemm_sampled(Xq_ref, sx_ref, ref_w, ms, ns)
    acc_s = acc[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()].cpu().numpy()
    y_s = bf16_bits(Y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()])
    assert np.array_equal(acc_s, acc_ref)
    assert_bf16_within_1ulp(y_s, y_ref, "%s M=%d" % (layer.name, M))

    # exact invariants over every accumulator
    row_ref = Xq_ref.astype(np.int64) @ colsum_w
    row_got = acc.sum(dim=1, dtype=torch.int64).cpu().numpy()
    assert np.array_equal(row_got, row_ref)
    colsum_x = Xq_ref.sum(axis=0, dtype=np.int64)
    col_ref = W8.astype(np.int64) @ colsum_x
    col_got = acc.sum(dim=0, dtype=torch.int64).cpu().numpy()
    assert np.array_equal(col_got, col_ref)
