"""The GEMM kernels' own failure path on the GPU, without a fault: with the
test wait budget set to 0 (w4a8_debug_set_wait_budget) every CTA of a launch
raises its abort flag at set-up, so each main-loop wait that does not find
its phase complete gives up at once and each CTA runs its abort path -- it records
W4A8_ERR_TIMEOUT, stores nothing, waits with the full 2 s budget for the
copies, MMAs and remote adds it already started, frees its tensor memory and
returns.  The test then restores the budget and checks that the context is
still usable: the same call is bit-exact against the oracle.

Every form of the launch is covered once: one CTA per tile, split-K with the
gather and the push reductions (thread-block clusters), the CTA pair, and
the warp-MMA decode form with one split and with split-K, and the persistent
CTA-pair form."""
import numpy as np
import pytest
import torch

import bit_block_quantized_w4a8_b200 as w4
import oracle
from bit_block_quantized_w4a8_b200 import workloads as wl
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    torch.cuda.set_device(0)
    assert w4.w4a8_get_status() == 0
    yield
    w4.w4a8_debug_set_wait_budget(-1)
    assert w4.w4a8_get_status() == 0


CASES = [
    # (M, N, K, variant, what the library runs)
    (40, 128, 256, "tensor_core", "one CTA, one split"),
    (64, 512, 2048, "tensor_core", "split-K 4, gather reduction"),
    (4, 512, 2048, "tensor_core", "split-K 8, push reduction"),
    (300, 256, 512, "cta_pair", "CTA pairs (tcgen05 cta_group::2)"),
    (2, 256, 512, "warp_mma", "decode form, one split"),
    (2, 256, 8192, "warp_mma", "decode form, split-K 2"),
    (1000, 512, 1024, "persistent", "persistent CTA pairs, several tiles per pair"),
]


@pytest.mark.parametrize("M,N,K,variant,what", CASES)
def test_abort_path_reports_timeout_stores_nothing_and_context_survives(M, N, K, variant, what):
    X = wl.random_matrix(M, K, 600 + M, std=1.0)
    W = wl.random_matrix(N, K, 601 + N, std=0.02)
    pk = w4.w4a8_quantize_weights(W.cuda())
    Xq, sx = w4.w4a8_quantize_act(X.cuda())
    out = torch.full((M, N), 7, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    def run(out=None):
        return w4.w4a8_gemm_variant(variant, Xq, None, pk, i32=True, out=out)
    w4.w4a8_debug_set_wait_budget(0)
    try:
        run(out)
        status = w4.w4a8_get_status()
    finally:
        w4.w4a8_debug_set_wait_budget(-1)
    assert status == w4.ERR_TIMEOUT, what
    assert int((out != 7).sum()) == 0, what + ": an aborted launch stored outputs"
    # the context is usable and the same call is exact again
    acc = run()
    torch.cuda.synchronize()
    assert w4.w4a8_get_status() == 0
    Xq_ref, sx_ref = oracle.quantize_act(X.numpy())
    acc_ref, _ = oracle.w4a8_gemm(Xq_ref, sx_ref, oracle.quantize_weights(W.numpy()))
    assert np.array_equal(acc.cpu().numpy(), acc_ref), what
