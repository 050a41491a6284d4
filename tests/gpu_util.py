"""Helpers shared by the GPU parity tests (comparison only; no arithmetic of
the method lives here)."""
import numpy as np
import pytest
import torch


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip("needs sm_100 (B200)")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_ordinal(bits: np.ndarray) -> np.ndarray:
    """Signed ordinal of bf16 bit patterns: neighbouring representable values
    differ by 1 and +0 / -0 both map to 0, so |ord(a) - ord(b)| is the
    distance in ulps."""
    b = bits.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def assert_bf16_within_1ulp(got_bits: np.ndarray, ref_bits: np.ndarray, what=""):
    d = np.abs(bf16_ordinal(got_bits) - bf16_ordinal(ref_bits))
    bad = np.nonzero(d > 1)
    assert d.max(initial=0) <= 1, "%s: %d outputs off by more than 1 bf16 ulp, first at %s" % (
        what, bad[0].size, tuple(int(x[0]) for x in bad))
    return d


def check_block(acc, Y, acc_ref, y_ref, what):
    """Every element of one block: INT32 bit-exact, bf16 within 1 ulp of the
    FP64 epilogue, exact zero where the accumulator is zero."""
    assert acc.shape == acc_ref.shape, what
    bad = np.nonzero(acc != acc_ref)
    assert bad[0].size == 0, "%s: %d accumulators differ, first at %s" % (
        what, bad[0].size, tuple(int(x[0]) for x in bad))
    got = bf16_bits(Y)
    assert_bf16_within_1ulp(got, y_ref, what)
    assert not np.any((acc_ref == 0) & ((got & 0x7FFF) != 0)), what + ": nonzero output for acc 0"
