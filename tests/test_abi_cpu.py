"""CPU-only checks of the boundary: the library builds for sm_100a, loads,
exports every entry point include/w4a8.h declares, and its host-only
functions (sizes, schedules, argument checks) behave as documented.  No
kernel is launched."""
import os
import re
import subprocess

import pytest

import bit_block_quantized_w4a8_b200 as w4
from bit_block_quantized_w4a8_b200 import build as wbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")


@pytest.fixture(scope="module")
def L():
    wbuild.build()
    return w4.lib()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a8_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_three_calls():
    names = _declared()
    for n in ("w4a8_quantize_weights", "w4a8_quantize_act", "w4a8_gemm"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", wbuild.LIB]).decode()
    exported = set(re.findall(r" T (w4a8_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(L, n)


def test_build_targets_sm100a_only():
    flags = " ".join(wbuild.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert len(re.findall(r"arch=", flags)) == 1


def test_packed_size(L):
    # 4096 x 4096: header 256 + s_w 16 KiB + 32 x 32 tiles of 8704 bytes
    assert w4.w4a8_packed_weight_bytes(4096, 4096) == 256 + 4 * 4096 + 32 * 32 * 8704
    # ragged N is padded to 128 channels
    n = w4.w4a8_packed_weight_bytes(200, 384)
    assert n == 1280 + 2 * 3 * 8704
    assert w4.w4a8_packed_weight_bytes(128, 200) == 0     # K % 128
    assert w4.w4a8_packed_weight_bytes(128, 256, 32) == 0  # unsupported group
    # about 0.531 bytes per weight
    assert abs(w4.w4a8_packed_weight_bytes(28672, 8192) / (28672 * 8192) - 0.53125) < 1e-3


def test_status_strings(L):
    for code in range(-7, 1):
        assert w4.w4a8_status_string(code).startswith("W4A8_")
    assert w4.w4a8_status_string(-99) == "W4A8_ERR_UNKNOWN"
    assert w4.w4a8_version() == 1


def test_argument_checks_before_any_launch(L):
    """Rejected calls return before touching the device."""
    st = None
    assert L.w4a8_gemm(None, None, None, 4, 128, 200, None, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w4a8_gemm(None, None, None, -1, 128, 256, None, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_gemm(None, None, None, 0, 128, 256, None, st) == w4.OK
    assert L.w4a8_gemm_i32(None, None, 0, 128, 256, None, st) == w4.OK
    assert L.w4a8_gemm_ex(None, None, None, 0, 128, 256, None, 4, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_gemm_ex(None, None, None, 0, 128, 256, None, 3, st) == w4.OK  # PDL | TENSOR_CORE
    assert L.w4a8_gemm(None, None, None, 4, 128, 65536 + 128, None, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w4a8_quantize_act(None, 3, 100, None, None, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w4a8_quantize_act(None, 0, 128, None, None, st) == w4.OK
    assert L.w4a8_quantize_weights(None, 128, 256, 64, None, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_unpack_weights(None, 128, 256, None, None, None, None, st) == w4.ERR_INVALID_ARG
    assert L.w4a8_debug_timeout_probe(10, st) == w4.ERR_INVALID_ARG
    # the W8A8 comparison entry points follow the same rules
    assert L.w8a8_gemm(None, None, None, None, 4, 128, 200, None, 0, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w8a8_gemm(None, None, None, None, 0, 128, 256, None, 0, st) == w4.OK
    assert L.w8a8_gemm(None, None, None, None, 0, 128, 256, None, 4, st) == w4.ERR_INVALID_ARG
    assert L.w8a8_gemm(None, None, None, None, 0, 128, 256, None, 2, st) == w4.ERR_INVALID_ARG
    assert L.w8a8_gemm(None, None, None, None, 4, 128, 256, None, 0, st) == w4.ERR_INVALID_ARG
    assert L.w8a8_gemm_i32(None, None, 0, 128, 256, None, st) == w4.OK
    assert L.w8a8_quantize_weights(None, 128, 200, None, None, st) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w8a8_quantize_weights(None, 0, 256, None, None, st) == w4.ERR_INVALID_ARG


def test_schedule_covers_the_machine(L):
    # without a device the library assumes 148 SMs; (the tensor-core
    # kernel's schedule: the dp4a form takes M <= 4, checked below)
    T, splits, ctas = w4.w4a8_gemm_schedule(16, 28672, 8192)
    assert w4.w4a8_gemm_kernel_kind(16, 28672, 8192) == w4.KERNEL_TENSOR_CORE
    assert T == 16 and ctas >= 148
    T, splits, ctas = w4.w4a8_gemm_schedule(8192, 8192, 8192)
    assert T == 256 and splits == 1 and ctas == 64 * 32
    for M in (1, 2, 16, 17, 32, 33, 64, 65, 128, 129, 256, 257, 4096):
        for N, K in ((4096, 4096), (28672, 8192), (8192, 28672), (128, 65536)):
            if w4.w4a8_gemm_kernel_kind(M, N, K) != w4.KERNEL_TENSOR_CORE:
                continue
            T, splits, ctas = w4.w4a8_gemm_schedule(M, N, K)
            assert T >= min(M, 16) and T in (16, 32, 64, 128, 256)
            assert 1 <= splits <= 8                    # one portable cluster
            kt = K // 128
            per = -(-kt // splits)
            assert -(-kt // per) == splits             # no empty split
            n_tiles, m_tiles = -(-N // 128), -(-M // T)
            assert ctas == n_tiles * m_tiles * splits


def test_w8a8_schedule_covers_the_machine(L):
    for M in (1, 8, 16, 17, 64, 65, 256, 4096):
        for N, K in ((4096, 4096), (28672, 8192), (8192, 28672)):
            T, splits, ctas = w4.w8a8_gemm_schedule(M, N, K)
            assert T >= min(M, 16) and 1 <= splits <= 8
            kt = K // 128
            per = -(-kt // splits)
            assert -(-kt // per) == splits
            assert ctas == -(-N // 128) * -(-M // T) * splits


def test_output_buffers_are_checked_before_any_launch():
    import torch
    like = torch.empty(2, 8)
    assert w4._out(None, torch.int8, (2, 8), like, "out").shape == (2, 8)
    # the kernels write every element of the output's shape: a buffer of any
    # other shape, dtype or layout, or off the inputs' device, is refused
    for bad in (torch.empty(2, 7, dtype=torch.int8), torch.empty(8, 2, dtype=torch.int8).t(),
                torch.empty(2, 8, dtype=torch.int16), torch.empty(2, 8, dtype=torch.int8), "x"):
        with pytest.raises(TypeError):
            w4._out(bad, torch.int8, (2, 8), like, "out")


def test_fused_call_shape_rules(L):
    # host-only: which decode shapes the one-launch quantize + GEMM accepts
    # (up to 16 tokens, a k range per CTA that stays resident, and the CTA's
    # slice of X within the quantizing warps' registers); everything else is
    # refused before any launch
    ok = [(1, 4096, 4096), (4, 4096, 4096), (4, 28672, 512), (16, 28672, 128),
          (8, 4096, 4096), (16, 4096, 4096)]  # (the last two: the decode form)
    refused = [(0, 4096, 4096), (17, 256, 4096), (1, 4096, 4000), (8, 4096, 8192),
               (16, 4096, 8192)]
    for sh in ok:
        assert w4.w4a8_gemm_fused_supported(*sh), sh
    for sh in refused:
        assert not w4.w4a8_gemm_fused_supported(*sh), sh


def test_kernel_kind_and_decode_schedule(L):
    """Host-only: a few tokens take the decode (warp-MMA) form with 16 output
    channels per CTA and split-K clusters of at most 8 for rows longer than
    4096; everything else the tensor-core kernel."""
    # (without a device the library assumes 148 SMs: the decode form when its
    # CTAs fit two per SM)
    assert w4.w4a8_gemm_kernel_kind(1, 4096, 4096) == w4.KERNEL_WARP_MMA      # 256 CTAs
    assert w4.w4a8_gemm_kernel_kind(16, 4096, 4096) == w4.KERNEL_WARP_MMA
    assert w4.w4a8_gemm_kernel_kind(17, 4096, 4096) == w4.KERNEL_TENSOR_CORE
    assert w4.w4a8_gemm_kernel_kind(1, 12288, 4096) == w4.KERNEL_TENSOR_CORE  # 768 CTAs
    assert w4.w4a8_gemm_kernel_kind(4, 2048, 8192) == w4.KERNEL_WARP_MMA      # 2 splits
    assert w4.w4a8_gemm_kernel_kind(64, 4096, 4096) == w4.KERNEL_TENSOR_CORE
    assert w4.w4a8_gemm_kernel_kind(1, 128, 65536) == w4.KERNEL_TENSOR_CORE  # 16 splits
    assert w4.w4a8_gemm_kernel_kind(0, 4096, 4096) == w4.KERNEL_TENSOR_CORE
    assert L.w4a8_gemm_kernel_kind(1, 4096, 200) == w4.ERR_UNSUPPORTED_SHAPE
    assert L.w4a8_gemm_kernel_kind(-1, 4096, 256) == w4.ERR_INVALID_ARG
    # schedule of the decode form: tile = all M tokens, splits, CTAs
    assert w4.w4a8_gemm_schedule(1, 4096, 4096) == (1, 1, 256)
    assert w4.w4a8_gemm_schedule(2, 1024, 11008) == (2, 3, 192)
    assert w4.w4a8_gemm_schedule(3, 200, 384) == (3, 1, 16)  # N padded to 256
    assert w4.VARIANTS["tensor_core"] == 7 and w4.VARIANTS["dp4a"] == 8
    assert w4.VARIANTS["warp_mma"] == 9


def test_debug_wait_budget_range(L):
    """Host-only: the test wait budget accepts -1 (default), 0 .. 1e10 ns."""
    assert L.w4a8_debug_set_wait_budget(-2) == w4.ERR_INVALID_ARG
    assert L.w4a8_debug_set_wait_budget(10000000001) == w4.ERR_INVALID_ARG
    assert L.w4a8_debug_set_wait_budget(0) == w4.OK
    assert L.w4a8_debug_set_wait_budget(5000) == w4.OK
    assert L.w4a8_debug_set_wait_budget(-1) == w4.OK
