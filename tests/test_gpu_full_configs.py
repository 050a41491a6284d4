"""GPU parity at the full sizes of the five synthetic workloads (tiny, decode
sweep N=K=4096, 7B-like layers, 70B-like layers, prefill), in the schedule
and launch flags the benchmark times.

Every output is compared element by element against the CPU oracle:

* the packed weights (unpacked) and the INT8 activations are bit-exact;
* every INT32 accumulator equals the oracle's integer product exactly;
* every bf16 output is within 1 bf16 ulp of the oracle's FP64 epilogue
  (review page "LiquidGEMM": INT8 x INT8 products accumulated in INT32, the
  FP scales applied afterwards), and exactly zero where the accumulator is.

The one case whose full oracle product would take minutes on the host
(M=16384, N=28672, K=8192: 3.85e12 multiply-adds) is compared on complete
output tiles instead: two whole 256 x 256 tiles (the CTA-pair tile) in each
raster band of 8 token tiles, the first and the last tile, every element of
each; plus the exact row- and column-sum invariants over all accumulators:
  sum_n acc[m,n] = Xq[m] . colsum_n(W8),   sum_m acc[m,n] = W8[n] . colsum_m(Xq).
"""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from gpu_util import check_block, require_gpu

pytestmark = pytest.mark.gpu

# full oracle products up to this many multiply-adds (the largest below it is
# 8192^3 = 5.5e11, about 20 s on 16 host cores); above it, complete tiles
FULL_PRODUCT_MACS = 1.0e12
TILE = 256          # the CTA-pair output tile: 256 channels x 256 tokens
RASTER_BAND = 8     # token tiles per raster band of the dense launch

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
        _weights[key] = (ref, pk)
    return _weights[key]


def _rows_of(ref_w, n0, n1):
    return {k: ref_w[k][n0:n1] for k in ("codes", "s_u8", "a", "s_w")}


def _tiles(M, N):
    """Complete output tiles checked for the largest case: two per raster
    band (different channel blocks), the first and the last."""
    mt, nt = -(-M // TILE), -(-N // TILE)
    picks = {(0, 0), (mt - 1, nt - 1)}
    for b in range(-(-mt // RASTER_BAND)):
        first = b * RASTER_BAND
        rows = min(RASTER_BAND, mt - first)
        picks.add((first + (5 * b + 1) % rows, (29 * b + 3) % nt))
        picks.add((first + (3 * b + 6) % rows, (17 * b + 50) % nt))
    return sorted(picks)


def _all_cases():
    out = []
    for name in wl.WORKLOADS:
        for M, layer in wl.cases(name):
            out.append(pytest.param(name, M, layer, id="%s-%s-M%d" % (name, layer.name, M)))
    return out


@pytest.mark.parametrize("name,M,layer", _all_cases())
def test_full_size_case(name, M, layer):
    ref_w, pk = _layer(name, layer)
    N, K = layer.N, layer.K
    X = wl.layer_activations(name, layer, M)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)
    del X

    acc = w4.w4a8_gemm_i32(Xq, pk)
    Y = w4.w4a8_gemm(Xq, sx, pk, flags=w4.W4A8_FLAG_PDL)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    what = "%s %s M=%d" % (name, layer.name, M)

    if float(M) * N * K <= FULL_PRODUCT_MACS:
        acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, ref_w)
        check_block(acc.cpu().numpy(), Y, acc_ref, y_ref, what)
        return

    for mt, nt in _tiles(M, N):
        m0, m1 = mt * TILE, min(M, (mt + 1) * TILE)
        n0, n1 = nt * TILE, min(N, (nt + 1) * TILE)
        acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref[m0:m1], sx_ref[m0:m1], _rows_of(ref_w, n0, n1))
        check_block(acc[m0:m1, n0:n1].cpu().numpy(), Y[m0:m1, n0:n1], acc_ref, y_ref,
                    "%s tile (%d, %d)" % (what, mt, nt))
    # exact invariants over every accumulator
    W8 = oracle.dequant_weights(ref_w["codes"], ref_w["s_u8"], ref_w["a"])
    colsum_w = W8.sum(axis=0, dtype=np.int64)
    row_ref = Xq_ref.astype(np.int64) @ colsum_w
    assert np.array_equal(acc.sum(dim=1, dtype=torch.int64).cpu().numpy(), row_ref)
    colsum_x = Xq_ref.sum(axis=0, dtype=np.int64)
    col_ref = W8.astype(np.int64) @ colsum_x
    assert np.array_equal(acc.sum(dim=0, dtype=torch.int64).cpu().numpy(), col_ref)


def test_tile_picks_cover_every_band():
    """The largest case's tile picks reach every raster band and both ends."""
    M, N = 16384, 28672
    picks = _tiles(M, N)
    mt = M // TILE
    bands = {m // RASTER_BAND for m, _ in picks}
    assert bands == set(range(mt // RASTER_BAND))
    assert (0, 0) in picks and (mt - 1, N // TILE - 1) in picks
