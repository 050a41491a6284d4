"""Seeded synthetic inputs for the W4A8 GEMM: the layer shapes and value
distributions of the LiquidGEMM evaluation (LLM decode / prefill layers),
made on the CPU in fp32 so that the CUDA library and the CPU oracle see the
same bytes.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantization, no dequantization, no GEMM), so both
the product path and the test oracle may use it.

Shapes follow the review page "LiquidGEMM" (pith.science verdict on arXiv
2509.01229): group size 64 (skeptic concrete_test), models LLaMA2-7B/70B,
LLaMA3-8B, Mistral-7B, Mixtral (skeptic concrete_test; referee minor 3),
batch sizes up to 256 for the kernel sweep (referee minor 5, paper Sec. 7.3
Fig. 12).  No model weights are used: Gaussian weights of the layer shapes
stand in for them, with a fixed fraction of activation channels scaled up as
outliers.
"""
from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import torch

GROUP = 64


@dataclass(frozen=True)
class Layer:
    name: str
    N: int  # output channels
    K: int  # reduction length


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    layers: Tuple[Layer, ...]
    Ms: Tuple[int, ...]
    w_std: float
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    description: str = ""


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny", 0, (Layer("tiny", 256, 512),), (16,), 0.02,
                 description="M=16 N=256 K=512, X~N(0,1), W~N(0,0.02)"),
        Workload("decode_sweep_4096", 1, (Layer("square", 4096, 4096),),
                 (1, 2, 4, 8, 16, 32, 64, 128, 256), 0.02, 0.01, 20.0,
                 description="N=K=4096, M in 1..256, 1% outlier channels x20"),
        Workload("llama7b_like", 2,
                 (Layer("qkv", 12288, 4096), Layer("o", 4096, 4096),
                  Layer("gate_up", 11008, 4096), Layer("down", 4096, 11008)),
                 (1, 16, 128, 1024), 0.02, 0.01, 20.0,
                 description="7B-like layers, M in {1,16,128,1024}, 1% outliers x20"),
        Workload("llama70b_like", 3,
                 (Layer("qkv", 10240, 8192), Layer("up", 28672, 8192),
                  Layer("down", 8192, 28672)),
                 (1, 32, 512, 2048), 0.015, 0.005, 50.0,
                 description="70B-like layers, M in {1,32,512,2048}, 0.5% outliers x50"),
        Workload("prefill", 4,
                 (Layer("square8k", 8192, 8192), Layer("up70b", 28672, 8192)),
                 (8192, 16384), 0.02,
                 description="M=8192 N=K=8192 and M=16384 N=28672 K=8192"),
    ]
}

# the prefill workload pairs each layer with one M, not the cross product
PREFILL_CASES = ((8192, Layer("square8k", 8192, 8192)),
                 (16384, Layer("up70b", 28672, 8192)))


def cases(name: str) -> List[Tuple[int, Layer]]:
    """(M, layer) pairs of a workload, in a fixed order."""
    w = WORKLOADS[name]
    if name == "prefill":
        return list(PREFILL_CASES)
    return [(M, L) for L in w.layers for M in w.Ms]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight_seed(w: Workload, layer_idx: int) -> int:
    return w.seed * 1_000_003 + 7919 * layer_idx + 1


def act_seed(w: Workload, layer_idx: int, M: int) -> int:
    return w.seed * 1_000_003 + 7919 * layer_idx + 104_729 * M + 2


def outlier_columns(K: int, frac: float, g: torch.Generator) -> torch.Tensor:
    n = int(frac * K)
    if n == 0:
        return torch.empty(0, dtype=torch.long)
    return torch.randperm(K, generator=g)[:n]


def make_activations(M: int, K: int, seed: int, outlier_frac: float = 0.0,
                     outlier_scale: float = 1.0) -> torch.Tensor:
    """X ~ N(0,1) fp32 [M,K]; floor(frac*K) channels (the same for every
    token, chosen by the seeded generator) scaled by ``outlier_scale``."""
    g = _gen(seed)
    X = torch.randn(M, K, generator=g, dtype=torch.float32)
    cols = outlier_columns(K, outlier_frac, g)
    if cols.numel():
        X[:, cols] *= outlier_scale
    return X


def make_weights(N: int, K: int, seed: int, std: float) -> torch.Tensor:
    """W ~ N(0, std) fp32 [N,K] (output-channel major, K contiguous)."""
    g = _gen(seed)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * std


def tiny_inputs() -> Tuple[torch.Tensor, torch.Tensor]:
    """The tiny correctness case: one generator seeded 0 draws X then W."""
    g = _gen(0)
    X = torch.randn(16, 512, generator=g, dtype=torch.float32)
    W = torch.randn(256, 512, generator=g, dtype=torch.float32) * 0.02
    return X, W


def layer_weights(name: str, layer: Layer) -> torch.Tensor:
    w = WORKLOADS[name]
    idx = [L.name for L in w.layers].index(layer.name)
    if name == "tiny":
        return tiny_inputs()[1]
    return make_weights(layer.N, layer.K, weight_seed(w, idx), w.w_std)


def layer_activations(name: str, layer: Layer, M: int) -> torch.Tensor:
    w = WORKLOADS[name]
    idx = [L.name for L in w.layers].index(layer.name)
    if name == "tiny":
        return tiny_inputs()[0][:M]
    return make_activations(M, layer.K, act_seed(w, idx, M), w.outlier_frac,
                            w.outlier_scale)


def random_matrix(rows: int, cols: int, seed: int, std: float = 1.0,
                  kind: str = "normal") -> torch.Tensor:
    """Extra seeded fp32 matrices for edge-case tests.

    kind: "normal" (N(0,std)), "zeros", "const" (every entry = std),
    "rowzero" (normal with every third row zero), "ties" (multiples of
    std/2, which put many quantizer inputs exactly on a rounding tie),
    "heavy" (normal with 2% of entries x100).
    """
    g = _gen(seed)
    if kind == "zeros":
        return torch.zeros(rows, cols)
    if kind == "const":
        return torch.full((rows, cols), float(std))
    X = torch.randn(rows, cols, generator=g, dtype=torch.float32) * std
    if kind == "rowzero":
        X[::3] = 0
    elif kind == "ties":
        X = torch.round(X / (std / 2)) * (std / 2)
    elif kind == "heavy":
        mask = torch.rand(rows, cols, generator=g) < 0.02
        X[mask] *= 100.0
    elif kind != "normal":
        raise ValueError(kind)
    return X


# ------------------------------------------------- mixture-of-experts layers
# The pages serve Mixtral-8x7B (skeptic concrete_test).  Its expert layers:
# 8 experts, hidden 4096, expert width 14336, each token routed to 2 experts.
# The gate and up projections of an expert are one GEMM (N = 2 x 14336).
# No router weights exist here: each token's two experts are drawn uniformly
# without replacement by the seeded generator.

@dataclass(frozen=True)
class MoEWorkload:
    name: str
    seed: int
    experts: int
    top_k: int
    layers: Tuple[Layer, ...]
    tokens: Tuple[int, ...]
    w_std: float
    description: str = ""


MOE_WORKLOADS: Dict[str, MoEWorkload] = {
    w.name: w for w in [
        MoEWorkload("mixtral_like", 6, 8, 2,
                    (Layer("gate_up", 28672, 4096), Layer("down", 4096, 14336)),
                    (1, 16, 64, 512), 0.02,
                    description="8 experts, top-2, tokens in {1,16,64,512}, X~N(0,1), "
                                "W~N(0,0.02)"),
    ]
}


def moe_routing(name: str, tokens: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rows grouped by expert: (offsets int32 [E+1], token index of each row
    int64 [tokens * top_k]).  Within an expert, rows keep token order."""
    w = MOE_WORKLOADS[name]
    g = _gen(w.seed * 1_000_003 + 31 * tokens + 5)
    choice = torch.stack([torch.randperm(w.experts, generator=g)[:w.top_k]
                          for _ in range(tokens)])                    # [tokens, top_k]
    rows_tok, counts = [], []
    for e in range(w.experts):
        t = torch.nonzero((choice == e).any(dim=1)).flatten()
        rows_tok.append(t)
        counts.append(t.numel())
    offsets = torch.zeros(w.experts + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(torch.tensor(counts, dtype=torch.int64), 0).to(torch.int32)
    return offsets, torch.cat(rows_tok)


def moe_expert_weights(name: str, layer: Layer, expert: int) -> torch.Tensor:
    """W_e ~ N(0, std) fp32 [N, K] of one expert."""
    w = MOE_WORKLOADS[name]
    idx = [L.name for L in w.layers].index(layer.name)
    return make_weights(layer.N, layer.K, w.seed * 1_000_003 + 7919 * idx + 613 * expert + 3,
                        w.w_std)


def moe_activations(name: str, layer: Layer, tokens: int) -> torch.Tensor:
    """X ~ N(0,1) fp32 [tokens, K], one row per token (not yet grouped)."""
    w = MOE_WORKLOADS[name]
    idx = [L.name for L in w.layers].index(layer.name)
    return make_activations(tokens, layer.K, w.seed * 1_000_003 + 7919 * idx + 104_729 * tokens + 4)
