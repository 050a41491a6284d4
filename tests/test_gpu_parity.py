"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
identical seeded inputs.  Packed weights, INT8 activations and INT32
accumulators must be bit-exact; bf16 outputs within 1 bf16 ulp of the
oracle's FP64 epilogue (the tolerance the LiquidGEMM build targets; the GPU
converts acc to fp32 and multiplies by the fp32 scale product before its
single bf16 rounding)."""
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


def _oracle_weights(W, group=64):
    return oracle.quantize_weights(W.numpy(), group=group)


def _check_packed(pk, ref):
    u = w4.w4a8_unpack_weights(pk)
    for key in ("codes", "s_u8", "a", "s_w"):
        got = u[key].cpu().numpy()
        assert np.array_equal(got, ref[key]), key


WEIGHT_CASES = [
    # (N, K, group, kind, seed)
    (256, 512, 64, "normal", 0),
    (200, 384, 64, "normal", 1),     # ragged N (partial last channel block)
    (8, 128, 64, "normal", 2),       # less than one channel block, one k block
    (136, 256, 128, "normal", 3),    # group 128
    (130, 256, 64, "rowzero", 4),    # zero channels
    (128, 256, 64, "ties", 5),       # many quantizer inputs on rounding ties
    (128, 512, 64, "heavy", 6),      # outliers: wide groups, s_u8 up to 16
    (64, 128, 64, "const", 7),       # constant groups: s_u8 = 1
    (128, 128, 64, "zeros", 8),      # all-zero layer
]


@pytest.mark.parametrize("N,K,group,kind,seed", WEIGHT_CASES)
def test_weight_quantization_bit_exact(N, K, group, kind, seed):
    W = wl.random_matrix(N, K, seed, std=0.02, kind=kind)
    ref = _oracle_weights(W, group)
    pk = w4.w4a8_quantize_weights(W.cuda(), group=group)
    _check_packed(pk, ref)
    if kind == "heavy":
        assert ref["s_u8"].max() >= 9


ACT_CASES = [(1, 16, "normal"), (5, 512, "normal"), (16, 4096, "normal"),
             (257, 384, "normal"), (9, 256, "rowzero"), (7, 512, "ties"),
             (33, 1024, "heavy"), (3, 128, "zeros"), (2, 160, "const")]


@pytest.mark.parametrize("M,K,kind", ACT_CASES)
def test_activation_quantization_bit_exact(M, K, kind):
    X = wl.random_matrix(M, K, 100 + M + K, std=1.0, kind=kind)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    assert np.array_equal(Xq.cpu().numpy(), Xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)


def test_activation_codes_at_rounding_boundaries():
    # entries a few ulps either side of (k + 1/2) s_x for every code k, over
    # scales from subnormal to huge: the codes must still be the oracle's
    X = boundary_rows(4352)
    Xq_ref, sx_ref = oracle.quantize_act(X)
    Xq, sx = w4.w4a8_quantize_act(torch.from_numpy(X).cuda())
    assert np.array_equal(sx.cpu().numpy(), sx_ref)
    got = Xq.cpu().numpy()
    bad = np.argwhere(got != Xq_ref)
    assert bad.size == 0, "%d codes differ, first at %s: x=%r got %d want %d" % (
        len(bad), tuple(bad[0]), float(X[tuple(bad[0])]), int(got[tuple(bad[0])]),
        int(Xq_ref[tuple(bad[0])]))


def test_wrong_output_buffers_are_refused():
    X = torch.randn(4, 256, device="cuda")
    pk = w4.w4a8_quantize_weights(torch.randn(300, 256, device="cuda") * 0.02)
    Xq, sx = w4.w4a8_quantize_act(X)
    for bad in (torch.empty(4, 299, dtype=torch.bfloat16, device="cuda"),
                torch.empty(4, 300, dtype=torch.float32, device="cuda"),
                torch.empty(300, 4, dtype=torch.bfloat16, device="cuda").t()):
        with pytest.raises(TypeError):
            w4.w4a8_gemm(Xq, sx, pk, out=bad)
    with pytest.raises(TypeError):
        w4.w4a8_quantize_act(X, out=torch.empty(4, 255, dtype=torch.int8, device="cuda"))
    with pytest.raises(TypeError):
        w4.w4a8_quantize_act(X, scale_out=torch.empty(3, device="cuda"))
    Y = torch.empty(4, 300, dtype=torch.bfloat16, device="cuda")
    assert w4.w4a8_gemm(Xq, sx, pk, out=Y) is Y
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0


def test_activation_quantization_empty():
    Xq, sx = w4.w4a8_quantize_act(torch.zeros(0, 128, device="cuda"))
    assert Xq.shape == (0, 128) and sx.shape == (0,)


def _run_case(M, N, K, seed, wkind="normal", xkind="normal", group=64):
    X = wl.random_matrix(M, K, 1000 + seed, std=1.0, kind=xkind)
    W = wl.random_matrix(N, K, 2000 + seed, std=0.02, kind=wkind)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    wq = _oracle_weights(W, group)
    acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, wq, group=group)
    pk = w4.w4a8_quantize_weights(W.cuda(), group=group)
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    acc = w4.w4a8_gemm_i32(Xq, pk)
    Y = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    return acc.cpu().numpy(), bf16_bits(Y), acc_ref, y_ref


GEMM_SHAPES = [
    (16, 256, 512),     # the tiny correctness workload's shape
    (1, 128, 128),      # one tile, one k block
    (1, 256, 4096),     # decode: deep split-K
    (3, 200, 384),      # ragged N and M
    (17, 256, 1024),    # two token tiles of 16 -> T=32 tile, ragged
    (33, 384, 256),
    (64, 128, 2048),
    (100, 136, 512),    # T=128 tile, ragged N
    (129, 256, 256),    # T=256 tile, ragged
    (256, 128, 384),
    (300, 256, 512),    # two token tiles of 256
    (513, 128, 128),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_parity(M, N, K):
    acc, y, acc_ref, y_ref = _run_case(M, N, K, seed=M * 7 + N + K)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref, "M=%d N=%d K=%d" % (M, N, K))


@pytest.mark.parametrize("wkind,xkind", [("rowzero", "rowzero"), ("ties", "ties"),
                                         ("heavy", "heavy"), ("const", "const"),
                                         ("zeros", "normal"), ("normal", "zeros")])
def test_gemm_parity_value_patterns(wkind, xkind):
    acc, y, acc_ref, y_ref = _run_case(40, 256, 512, seed=11, wkind=wkind, xkind=xkind)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref)


def test_gemm_parity_group128():
    acc, y, acc_ref, y_ref = _run_case(24, 256, 512, seed=12, group=128)
    assert np.array_equal(acc, acc_ref)
    assert_bf16_within_1ulp(y, y_ref)


def test_gemm_int32_extremes():
    """Largest accumulators the format can produce: every activation at +-127
    and every weight group at the top of the protective range."""
    M, N, K = 4, 128, 8192
    X = torch.full((M, K), 3.0)
    X[1] = -3.0
    X[2, ::2] = -3.0
    W = torch.full((N, K), 0.5)
    W[:, 0] = -0.5
    acc, y, acc_ref, y_ref = _run_case_from(X, W)
    assert np.array_equal(acc, acc_ref)
    assert np.abs(acc_ref).max() > 100_000_000
    assert_bf16_within_1ulp(y, y_ref)


def _run_case_from(X, W, group=64):
    M, K = X.shape
    N = W.shape[0]
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    wq = _oracle_weights(W, group)
    acc_ref, y_ref = oracle.w4a8_gemm(Xq_ref, sx_ref, wq, group=group)
    pk = w4.w4a8_quantize_weights(W.cuda(), group=group)
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    acc = w4.w4a8_gemm_i32(Xq, pk)
    Y = w4.w4a8_gemm(Xq, sx, pk)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), bf16_bits(Y), acc_ref, y_ref


def test_gemm_deterministic_and_stream():
    X = wl.random_matrix(5, 1024, 31).cuda()
    W = wl.random_matrix(384, 1024, 32, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    Xq, sx = w4.w4a8_quantize_act(X)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        y1 = w4.w4a8_gemm(Xq, sx, pk, stream=s)
        y2 = w4.w4a8_gemm(Xq, sx, pk, stream=s)
    s.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_gemm_empty_m():
    W = wl.random_matrix(128, 256, 1, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    Y = w4.w4a8_gemm(torch.zeros(0, 256, dtype=torch.int8, device="cuda"),
                     torch.zeros(0, device="cuda"), pk)
    assert Y.shape == (0, 128)


def test_host_side_rejections():
    W = wl.random_matrix(128, 256, 1, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    L = w4.lib()
    Xq = torch.zeros(4, 256, dtype=torch.int8, device="cuda")
    sx = torch.ones(4, device="cuda")
    Y = torch.empty(4, 128, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    p = lambda t: t.data_ptr()
    # K not a multiple of 128
    assert L.w4a8_gemm(p(Xq), p(sx), p(pk.data), 4, 128, 200, p(Y), st) == w4.ERR_UNSUPPORTED_SHAPE
    # misaligned activations
    assert L.w4a8_gemm(p(Xq) + 1, p(sx), p(pk.data), 4, 128, 256, p(Y), st) == w4.ERR_MISALIGNED
    # missing output
    assert L.w4a8_gemm(p(Xq), p(sx), p(pk.data), 4, 128, 256, None, st) == w4.ERR_INVALID_ARG
    # unknown launch flag
    assert L.w4a8_gemm_ex(p(Xq), p(sx), p(pk.data), 4, 128, 256, p(Y), 6, st) == w4.ERR_INVALID_ARG
    # bad group
    assert L.w4a8_quantize_weights(p(W), 128, 256, 32, p(pk.data), st) == w4.ERR_INVALID_ARG
    assert w4.w4a8_get_status() == 0


def test_packed_header_mismatch_is_reported():
    """A packed buffer used with a smaller N than it was built for: the kernel
    reads only inside the buffer, stores nothing, and reports it."""
    W = wl.random_matrix(256, 256, 3, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    wrong = w4.PackedWeights(pk.data, 128, 256, 64)
    Xq = torch.ones(2, 256, dtype=torch.int8, device="cuda")
    out = torch.full((2, 128), 7, dtype=torch.int32, device="cuda")
    w4.w4a8_gemm_i32(Xq, wrong, out=out)
    assert w4.w4a8_get_status() == w4.ERR_BAD_PACKED
    assert int((out != 7).sum()) == 0


@pytest.mark.parametrize("N,K", [(256, 256), (200, 384)])
def test_packed_buffer_every_byte_written(N, K):
    """A buffer pre-filled with garbage comes back fully defined: the header
    beyond its fields and the gap before the first tile are zero, padding
    channels have zero scales, and two packings of the same weights into
    differently pre-filled buffers are byte-identical (the buffer can be
    saved and reloaded)."""
    W = wl.random_matrix(N, K, 13, std=0.02).cuda()
    nbytes = w4.w4a8_packed_weight_bytes(N, K)
    outs = []
    for fill in (0xAB, 0x00):
        buf = torch.full((nbytes,), fill, dtype=torch.uint8, device="cuda")
        w4.w4a8_quantize_weights(W, out=buf)
        outs.append(buf.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    b = outs[0]
    n_pad = -(-N // 128) * 128
    assert not b[48:256].any()
    sw_end = 256 + 4 * n_pad
    tiles = -(-sw_end // 256) * 256
    assert not b[sw_end:tiles].any()
    assert not b[256 + 4 * N:sw_end].any()  # scales of the padding channels


def test_bounded_wait_reports_timeout_and_context_survives():
    w4.w4a8_debug_timeout_probe(2_000_000)  # 2 ms limit, nothing ever arrives
    assert w4.w4a8_get_status() == w4.ERR_TIMEOUT
    assert w4.w4a8_get_status() == 0
    acc, y, acc_ref, y_ref = _run_case(3, 128, 256, seed=5)
    assert np.array_equal(acc, acc_ref)


def test_pdl_chain_matches_plain_calls():
    """Chains of quantize -> GEMM launched with programmatic dependent launch
    (each kernel may start while the previous one finishes) give the same
    bits as plain launches, split-K (cluster) shapes included."""
    K = 2048
    W = wl.random_matrix(256, K, 41, std=0.02).cuda()
    pk = w4.w4a8_quantize_weights(W)
    Ms = [1, 3, 16, 40, 130, 300]
    Xs = [wl.random_matrix(M, K, 50 + M).cuda() for M in Ms]
    ref = []
    for X in Xs:
        xq, s = w4.w4a8_quantize_act(X)
        ref.append(w4.w4a8_gemm(xq, s, pk).clone())
    for rep in range(3):
        outs = []
        for X in Xs:
            xq, s = w4.w4a8_quantize_act(X, flags=w4.W4A8_FLAG_PDL)
            outs.append(w4.w4a8_gemm(xq, s, pk, flags=w4.W4A8_FLAG_PDL))
        torch.cuda.synchronize()
        for a, b in zip(outs, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert w4.w4a8_get_status() == 0


@pytest.mark.parametrize("M,N,K", [(512, 4096, 4096), (1024, 8192, 2048), (48, 2048, 8192)])
def test_repeated_runs_deep_k(M, N, K):
    """Many ring rounds per CTA, repeated: every run bit-identical, and exact
    against the oracle on sampled outputs plus row/column-sum invariants over
    all outputs (guards the pipeline's barrier protocol)."""
    X = wl.random_matrix(M, K, 71 + M, std=1.0, kind="heavy")
    W = wl.random_matrix(N, K, 72 + N, std=0.02)
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    wq = _oracle_weights(W)
    W8 = oracle.dequant_weights(wq["codes"], wq["s_u8"], wq["a"])
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    first = None
    rng = np.random.default_rng(M + N + K)
    ms = rng.integers(0, M, 256)
    ns = rng.integers(0, N, 256)
    acc_s_ref, _ = oracle.w4a8_gemm_sampled(Xq_ref, sx_ref, wq, ms, ns)
    row_ref = Xq_ref.astype(np.int64) @ W8.sum(axis=0, dtype=np.int64)
    col_ref = W8.astype(np.int64) @ Xq_ref.sum(axis=0, dtype=np.int64)
    for rep in range(6):
        acc = w4.w4a8_gemm_i32(Xq, pk)
        torch.cuda.synchronize()
        assert w4.w4a8_get_status() == 0
        if first is None:
            first = acc.clone()
            assert np.array_equal(acc.cpu().numpy()[ms, ns], acc_s_ref)
            assert np.array_equal(acc.sum(dim=1, dtype=torch.int64).cpu().numpy(), row_ref)
            assert np.array_equal(acc.sum(dim=0, dtype=torch.int64).cpu().numpy(), col_ref)
        else:
            assert torch.equal(acc, first), "run %d differs from run 0" % rep
