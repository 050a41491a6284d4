"""B200-native block-quantized W4A8 GEMM (LiquidQuant-style INT4 weights,
per-token INT8 activations, tcgen05 INT8 tensor cores, bf16 output).

This module is the Python binding of ``libw4a8.so`` (C ABI in
``include/w4a8.h``).  It only marshals arguments: every step of the path runs
in the library's CUDA kernels.  PyTorch provides device memory and streams.
The functions carry the names of the C entry points; all tensors are CUDA
tensors on the current device and work is enqueued on the current stream
unless ``stream`` is given.

If the library has not been built, every call raises ``W4A8Error``; there is
no fallback implementation.
"""
import ctypes as _ct
import os as _os
import threading as _threading

import torch as _torch

from .build import LIB as _LIB_PATH

__all__ = [
    "W4A8Error", "lib", "w4a8_version", "w4a8_status_string",
    "w4a8_packed_weight_bytes", "w4a8_quantize_weights", "w4a8_unpack_weights",
    "w4a8_quantize_act", "w4a8_gemm", "w4a8_gemm_i32", "w4a8_gemm_schedule",
    "w4a8_get_status", "w4a8_debug_timeout_probe", "PackedWeights",
    "w8a8_quantize_weights", "w8a8_gemm", "w8a8_gemm_i32", "w8a8_gemm_schedule",
    "GroupedPackedWeights", "w4a8_quantize_grouped_weights", "w4a8_grouped_gemm",
    "w4a8_grouped_gemm_i32", "w4a8_grouped_gemm_schedule", "w4a8_gemm_variant", "VARIANTS",
    "w4a8_gemm_fused", "w4a8_gemm_fused_supported", "w4a8_gemm_kernel_kind",
    "KERNEL_TENSOR_CORE", "KERNEL_WARP_MMA", "w4a8_debug_set_wait_budget",
]

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_MISALIGNED = -3
ERR_CUDA = -5
ERR_TIMEOUT = -6
ERR_BAD_PACKED = -7
ERR_BAD_OFFSETS = -8

W4A8_FLAG_PDL = 1  # programmatic dependent launch (see include/w4a8.h)
W4A8_FLAG_TENSOR_CORE = 2  # the tcgen05 kernel even where the decode form applies

# kernel variants of the ablation study (W4A8_VARIANT_* in include/w4a8.h)
VARIANTS = {"default": 0, "baseline": 1, "naive_dequant": 2, "serial": 3, "one_group": 4,
            "group_issues_mma": 5, "cta_pair": 6, "tensor_core": 7, "dp4a": 8,
            "warp_mma": 9, "persistent": 10}

# kernels behind w4a8_gemm (W4A8_KERNEL_* in include/w4a8.h)
KERNEL_TENSOR_CORE = 0
KERNEL_WARP_MMA = 1


class W4A8Error(RuntimeError):
    def __init__(self, what, code):
        super().__init__("%s failed: %s (%d)" % (what, w4a8_status_string(code), code))
        self.code = code


_lib = None
_lock = _threading.Lock()


def lib():
    """The loaded ``libw4a8.so`` (ctypes.CDLL)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not _os.path.exists(_LIB_PATH):
            raise W4A8Error("loading %s (not built; run `python -m "
                            "bit_block_quantized_w4a8_b200.build`)" % _LIB_PATH,
                            ERR_CUDA)
        L = _ct.CDLL(_LIB_PATH)
        i32, sz, p, ll = _ct.c_int, _ct.c_size_t, _ct.c_void_p, _ct.c_longlong
        sigs = {
            "w4a8_status_string": ([i32], _ct.c_char_p),
            "w4a8_version": ([], i32),
            "w4a8_packed_weight_bytes": ([i32, i32, i32], sz),
            "w4a8_quantize_weights": ([p, i32, i32, i32, p, p], i32),
            "w4a8_unpack_weights": ([p, i32, i32, p, p, p, p, p], i32),
            "w4a8_quantize_act": ([p, i32, i32, p, p, p], i32),
            "w4a8_quantize_act_ex": ([p, i32, i32, p, p, _ct.c_uint, p], i32),
            "w4a8_gemm_ex": ([p, p, p, i32, i32, i32, p, _ct.c_uint, p], i32),
            "w4a8_gemm": ([p, p, p, i32, i32, i32, p, p], i32),
            "w4a8_gemm_i32": ([p, p, i32, i32, i32, p, p], i32),
            "w4a8_gemm_schedule": ([i32, i32, i32, p, p, p], i32),
            "w4a8_gemm_kernel_kind": ([i32, i32, i32], i32),
            "w8a8_quantize_weights": ([p, i32, i32, p, p, p], i32),
            "w8a8_gemm": ([p, p, p, p, i32, i32, i32, p, _ct.c_uint, p], i32),
            "w8a8_gemm_i32": ([p, p, i32, i32, i32, p, p], i32),
            "w8a8_gemm_schedule": ([i32, i32, i32, p, p, p], i32),
            "w4a8_grouped_gemm": ([p, p, p, i32, p, i32, i32, i32, i32, p, _ct.c_uint, p], i32),
            "w4a8_grouped_gemm_i32": ([p, p, i32, p, i32, i32, i32, i32, p, p], i32),
            "w4a8_grouped_gemm_schedule": ([i32, i32, i32, i32, i32, p, p, p], i32),
            "w4a8_gemm_variant": ([i32, p, p, p, i32, i32, i32, p, p, _ct.c_uint, p], i32),
            "w4a8_gemm_fused": ([p, p, i32, i32, i32, p, _ct.c_uint, p], i32),
            "w4a8_gemm_fused_supported": ([i32, i32, i32], i32),
            "w4a8_get_status": ([p], i32),
            "w4a8_debug_timeout_probe": ([ll, p], i32),
            "w4a8_debug_set_wait_budget": ([ll], i32),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else _ct.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = _torch.cuda.current_stream()
    return _ct.c_void_p(stream.cuda_stream)


def _check(rc, what):
    if rc != OK:
        raise W4A8Error(what, rc)


def _need(t, dtype, ndim, name):
    if not isinstance(t, _torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype or t.dim() != ndim or not t.is_contiguous():
        raise TypeError("%s must be a contiguous %dD %s tensor" % (name, ndim, dtype))


def _out(t, dtype, shape, like, name):
    """The caller's output buffer, checked (the kernels write every element
    of the given shape, so a smaller buffer would be written past), or a new
    one on ``like``'s device."""
    if t is None:
        return _torch.empty(*shape, dtype=dtype, device=like.device)
    if (not isinstance(t, _torch.Tensor) or not t.is_cuda or t.device != like.device
            or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous()):
        raise TypeError("%s must be a contiguous %s tensor of shape %s on %s" %
                        (name, dtype, tuple(shape), like.device))
    return t


def w4a8_status_string(code):
    return lib().w4a8_status_string(int(code)).decode()


def w4a8_version():
    return lib().w4a8_version()


def w4a8_packed_weight_bytes(N, K, group=64):
    return int(lib().w4a8_packed_weight_bytes(int(N), int(K), int(group)))


class PackedWeights:
    """A packed LQQ weight buffer (uint8 CUDA tensor) with its shape."""

    def __init__(self, data, N, K, group):
        self.data, self.N, self.K, self.group = data, int(N), int(K), int(group)

    def __repr__(self):
        return "PackedWeights(N=%d, K=%d, group=%d, bytes=%d)" % (
            self.N, self.K, self.group, self.data.numel())


def w4a8_quantize_weights(W, group=64, out=None, stream=None):
    """Quantize fp32 weights W [N, K] into a packed LQQ buffer."""
    _need(W, _torch.float32, 2, "W")
    N, K = W.shape
    nbytes = w4a8_packed_weight_bytes(N, K, group)
    if nbytes == 0:
        raise W4A8Error("w4a8_packed_weight_bytes", ERR_UNSUPPORTED_SHAPE)
    if out is None:
        out = _torch.empty(nbytes, dtype=_torch.uint8, device=W.device)
    elif (not isinstance(out, _torch.Tensor) or not out.is_cuda or out.device != W.device
          or out.dtype != _torch.uint8 or out.numel() < nbytes or not out.is_contiguous()):
        raise ValueError("out must be a contiguous uint8 CUDA tensor of at least %d bytes "
                         "on %s" % (nbytes, W.device))
    _check(lib().w4a8_quantize_weights(_ptr(W), N, K, group, _ptr(out), _stream(stream)),
           "w4a8_quantize_weights")
    return PackedWeights(out, N, K, group)


def w4a8_unpack_weights(packed, stream=None):
    """Canonical arrays of a packed buffer: codes [N,K], s_u8 [N,G], a [N,G], s_w [N]."""
    d = packed.data.device
    N, K, G = packed.N, packed.K, packed.K // packed.group
    codes = _torch.empty(N, K, dtype=_torch.uint8, device=d)
    s = _torch.empty(N, G, dtype=_torch.uint8, device=d)
    a = _torch.empty(N, G, dtype=_torch.uint8, device=d)
    sw = _torch.empty(N, dtype=_torch.float32, device=d)
    _check(lib().w4a8_unpack_weights(_ptr(packed.data), N, K, _ptr(codes), _ptr(s), _ptr(a),
                                     _ptr(sw), _stream(stream)), "w4a8_unpack_weights")
    return dict(codes=codes, s_u8=s, a=a, s_w=sw)


def w4a8_quantize_act(X, out=None, scale_out=None, stream=None, flags=0):
    """Per-token INT8 quantization of fp32 X [M, K]: returns (Xq int8, s_x fp32).
    ``flags`` are the launch options of w4a8_quantize_act_ex (0 = plain call)."""
    _need(X, _torch.float32, 2, "X")
    M, K = X.shape
    Xq = _out(out, _torch.int8, (M, K), X, "out")
    sx = _out(scale_out, _torch.float32, (M,), X, "scale_out")
    if flags:
        rc = lib().w4a8_quantize_act_ex(_ptr(X), M, K, _ptr(Xq), _ptr(sx), int(flags),
                                        _stream(stream))
    else:
        rc = lib().w4a8_quantize_act(_ptr(X), M, K, _ptr(Xq), _ptr(sx), _stream(stream))
    _check(rc, "w4a8_quantize_act")
    return Xq, sx


def w4a8_gemm(Xq, s_x, packed, out=None, stream=None, flags=0):
    """Y [M, N] bf16 = (s_x[m] s_w[n]) * sum_k Xq[m,k] Wdq[n,k].
    ``flags`` are the launch options of w4a8_gemm_ex (0 = plain call)."""
    _need(Xq, _torch.int8, 2, "Xq")
    _need(s_x, _torch.float32, 1, "s_x")
    M, K = Xq.shape
    if K != packed.K:
        raise ValueError("Xq has K=%d, weights have K=%d" % (K, packed.K))
    N = packed.N
    Y = _out(out, _torch.bfloat16, (M, N), Xq, "out")
    if flags:
        rc = lib().w4a8_gemm_ex(_ptr(Xq), _ptr(s_x), _ptr(packed.data), M, N, K, _ptr(Y),
                                int(flags), _stream(stream))
    else:
        rc = lib().w4a8_gemm(_ptr(Xq), _ptr(s_x), _ptr(packed.data), M, N, K, _ptr(Y),
                             _stream(stream))
    _check(rc, "w4a8_gemm")
    return Y


def w4a8_gemm_i32(Xq, packed, out=None, stream=None):
    """Exact INT32 accumulators acc [M, N] = sum_k Xq[m,k] Wdq[n,k]."""
    _need(Xq, _torch.int8, 2, "Xq")
    M, K = Xq.shape
    if K != packed.K:
        raise ValueError("Xq has K=%d, weights have K=%d" % (K, packed.K))
    N = packed.N
    acc = _out(out, _torch.int32, (M, N), Xq, "out")
    _check(lib().w4a8_gemm_i32(_ptr(Xq), _ptr(packed.data), M, N, K, _ptr(acc),
                               _stream(stream)), "w4a8_gemm_i32")
    return acc


def w4a8_gemm_schedule(M, N, K):
    """(tokens per tile, split-K factor, CTAs) the library picks for a shape."""
    t, s, c = _ct.c_int(0), _ct.c_int(0), _ct.c_int(0)
    _check(lib().w4a8_gemm_schedule(int(M), int(N), int(K), _ct.byref(t), _ct.byref(s),
                                    _ct.byref(c)), "w4a8_gemm_schedule")
    return t.value, s.value, c.value


class GroupedPackedWeights:
    """Packed LQQ weights of `groups` experts of one shape, back to back in
    one uint8 CUDA tensor (the layout w4a8_grouped_gemm reads)."""

    def __init__(self, data, groups, N, K, group):
        self.data, self.groups = data, int(groups)
        self.N, self.K, self.group = int(N), int(K), int(group)
        self.expert_bytes = w4a8_packed_weight_bytes(N, K, group)

    def expert(self, g):
        """The PackedWeights view of expert g (shares memory)."""
        b = self.expert_bytes
        return PackedWeights(self.data[g * b:(g + 1) * b], self.N, self.K, self.group)


def w4a8_quantize_grouped_weights(W, group=64, stream=None):
    """Quantize fp32 expert weights W [E, N, K] into one grouped buffer."""
    if not isinstance(W, _torch.Tensor) or W.dim() != 3:
        raise TypeError("W must be a 3D [E, N, K] CUDA tensor")
    E, N, K = W.shape
    b = w4a8_packed_weight_bytes(N, K, group)
    if b == 0:
        raise W4A8Error("w4a8_packed_weight_bytes", ERR_UNSUPPORTED_SHAPE)
    data = _torch.empty(E * b, dtype=_torch.uint8, device=W.device)
    for g in range(E):
        w4a8_quantize_weights(W[g], group=group, out=data[g * b:(g + 1) * b], stream=stream)
    return GroupedPackedWeights(data, E, N, K, group)


def _grouped_args(Xq, gw, offsets, max_rows):
    _need(Xq, _torch.int8, 2, "Xq")
    _need(offsets, _torch.int32, 1, "offsets")
    M, K = Xq.shape
    if K != gw.K or offsets.numel() != gw.groups + 1:
        raise ValueError("Xq has K=%d (weights K=%d); offsets needs %d entries"
                         % (K, gw.K, gw.groups + 1))
    max_rows = M if max_rows is None else int(max_rows)
    return M, K, max_rows


def w4a8_grouped_gemm(Xq, s_x, gw, offsets, max_rows=None, out=None, stream=None, flags=0):
    """Grouped (mixture-of-experts) W4A8 GEMM: rows offsets[g]..offsets[g+1]-1
    of Xq use expert g of ``gw``.  ``offsets`` is an int32 CUDA tensor of
    groups + 1 entries; ``max_rows`` bounds any group's rows (default M)."""
    _need(s_x, _torch.float32, 1, "s_x")
    M, K, max_rows = _grouped_args(Xq, gw, offsets, max_rows)
    Y = _out(out, _torch.bfloat16, (M, gw.N), Xq, "out")
    _check(lib().w4a8_grouped_gemm(_ptr(Xq), _ptr(s_x), _ptr(gw.data), gw.groups, _ptr(offsets),
                                   M, max_rows, gw.N, K, _ptr(Y), int(flags), _stream(stream)),
           "w4a8_grouped_gemm")
    return Y


def w4a8_grouped_gemm_i32(Xq, gw, offsets, max_rows=None, out=None, stream=None):
    """Exact INT32 accumulators of the grouped W4A8 GEMM."""
    M, K, max_rows = _grouped_args(Xq, gw, offsets, max_rows)
    acc = _out(out, _torch.int32, (M, gw.N), Xq, "out")
    _check(lib().w4a8_grouped_gemm_i32(_ptr(Xq), _ptr(gw.data), gw.groups, _ptr(offsets), M,
                                       max_rows, gw.N, K, _ptr(acc), _stream(stream)),
           "w4a8_grouped_gemm_i32")
    return acc


def w4a8_grouped_gemm_schedule(groups, M_total, max_rows, N, K):
    """(tokens per tile, split-K factor, CTAs launched) of the grouped kernel."""
    t, s, c = _ct.c_int(0), _ct.c_int(0), _ct.c_int(0)
    _check(lib().w4a8_grouped_gemm_schedule(int(groups), int(M_total), int(max_rows), int(N),
                                            int(K), _ct.byref(t), _ct.byref(s), _ct.byref(c)),
           "w4a8_grouped_gemm_schedule")
    return t.value, s.value, c.value


def w8a8_quantize_weights(W, stream=None):
    """Per-channel symmetric INT8 weights of fp32 W [N, K] for the W8A8
    comparison kernel: returns (Wq int8 [N, K], s_w fp32 [N])."""
    _need(W, _torch.float32, 2, "W")
    N, K = W.shape
    Wq = _torch.empty(N, K, dtype=_torch.int8, device=W.device)
    sw = _torch.empty(N, dtype=_torch.float32, device=W.device)
    _check(lib().w8a8_quantize_weights(_ptr(W), N, K, _ptr(Wq), _ptr(sw), _stream(stream)),
           "w8a8_quantize_weights")
    return Wq, sw


def w8a8_gemm(Xq, s_x, Wq, s_w, out=None, stream=None, flags=0):
    """W8A8 comparison GEMM: Y [M, N] bf16 = (s_x[m] s_w[n]) * sum_k Xq[m,k] Wq[n,k]."""
    _need(Xq, _torch.int8, 2, "Xq")
    _need(s_x, _torch.float32, 1, "s_x")
    _need(Wq, _torch.int8, 2, "Wq")
    _need(s_w, _torch.float32, 1, "s_w")
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_w.numel() != N or s_x.numel() != M:
        raise ValueError("shape mismatch: Xq %s, Wq %s, s_x %s, s_w %s"
                         % (tuple(Xq.shape), tuple(Wq.shape), s_x.numel(), s_w.numel()))
    Y = _out(out, _torch.bfloat16, (M, N), Xq, "out")
    _check(lib().w8a8_gemm(_ptr(Xq), _ptr(s_x), _ptr(Wq), _ptr(s_w), M, N, K, _ptr(Y),
                           int(flags), _stream(stream)), "w8a8_gemm")
    return Y


def w8a8_gemm_i32(Xq, Wq, out=None, stream=None):
    """Exact INT32 accumulators of the W8A8 comparison GEMM."""
    _need(Xq, _torch.int8, 2, "Xq")
    _need(Wq, _torch.int8, 2, "Wq")
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("Xq has K=%d, Wq has K=%d" % (K, Wq.shape[1]))
    acc = _out(out, _torch.int32, (M, N), Xq, "out")
    _check(lib().w8a8_gemm_i32(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), _stream(stream)),
           "w8a8_gemm_i32")
    return acc


def w8a8_gemm_schedule(M, N, K):
    """(tokens per tile, split-K factor, CTAs) of the W8A8 kernel for a shape."""
    t, s, c = _ct.c_int(0), _ct.c_int(0), _ct.c_int(0)
    _check(lib().w8a8_gemm_schedule(int(M), int(N), int(K), _ct.byref(t), _ct.byref(s),
                                    _ct.byref(c)), "w8a8_gemm_schedule")
    return t.value, s.value, c.value


def w4a8_gemm_variant(variant, Xq, s_x, packed, i32=False, out=None, stream=None, flags=0):
    """The W4A8 product through one of the ablation study's kernel variants
    (a name of ``VARIANTS`` or its number): bf16 Y, or with ``i32`` the exact
    INT32 accumulators."""
    v = VARIANTS[variant] if isinstance(variant, str) else int(variant)
    _need(Xq, _torch.int8, 2, "Xq")
    M, K = Xq.shape
    if K != packed.K:
        raise ValueError("Xq has K=%d, weights have K=%d" % (K, packed.K))
    N = packed.N
    if i32:
        acc = _out(out, _torch.int32, (M, N), Xq, "out")
        rc = lib().w4a8_gemm_variant(v, _ptr(Xq), None, _ptr(packed.data), M, N, K, None,
                                     _ptr(acc), int(flags), _stream(stream))
        _check(rc, "w4a8_gemm_variant")
        return acc
    _need(s_x, _torch.float32, 1, "s_x")
    Y = _out(out, _torch.bfloat16, (M, N), Xq, "out")
    rc = lib().w4a8_gemm_variant(v, _ptr(Xq), _ptr(s_x), _ptr(packed.data), M, N, K, _ptr(Y),
                                 None, int(flags), _stream(stream))
    _check(rc, "w4a8_gemm_variant")
    return Y


def w4a8_gemm_kernel_kind(M, N, K):
    """Which kernel w4a8_gemm runs for a shape: KERNEL_TENSOR_CORE or
    KERNEL_WARP_MMA (the decode form for a few tokens)."""
    k = lib().w4a8_gemm_kernel_kind(int(M), int(N), int(K))
    if k < 0:
        raise W4A8Error("w4a8_gemm_kernel_kind", k)
    return k


def w4a8_gemm_fused_supported(M, N, K):
    """Whether w4a8_gemm_fused applies to a shape (decode tiles)."""
    return bool(lib().w4a8_gemm_fused_supported(int(M), int(N), int(K)))


def w4a8_gemm_fused(X, packed, out=None, stream=None, flags=0):
    """Activation quantization and the W4A8 GEMM in one launch (decode
    shapes, see w4a8_gemm_fused_supported): Y [M, N] bf16 from fp32 X [M, K];
    bit-identical to w4a8_quantize_act followed by w4a8_gemm."""
    _need(X, _torch.float32, 2, "X")
    M, K = X.shape
    if K != packed.K:
        raise ValueError("X has K=%d, weights have K=%d" % (K, packed.K))
    Y = _out(out, _torch.bfloat16, (M, packed.N), X, "out")
    _check(lib().w4a8_gemm_fused(_ptr(X), _ptr(packed.data), M, packed.N, K, _ptr(Y),
                                 int(flags), _stream(stream)), "w4a8_gemm_fused")
    return Y


def w4a8_get_status(stream=None):
    """Synchronize the stream and return/clear the device status word."""
    return lib().w4a8_get_status(_stream(stream))


def w4a8_debug_timeout_probe(limit_ns, stream=None):
    _check(lib().w4a8_debug_timeout_probe(int(limit_ns), _stream(stream)),
           "w4a8_debug_timeout_probe")


def w4a8_debug_set_wait_budget(ns):
    """Test aid: budget of the kernels' main-loop waits for later launches
    (-1 = the default 2 s; 0 = every CTA raises its abort flag at set-up,
    so every launch aborts)."""
    _check(lib().w4a8_debug_set_wait_budget(int(ns)), "w4a8_debug_set_wait_budget")
