"""Seeded synthetic inputs for the MoE expert layer (routing counts and tensors).

This module holds no MXFP8 or GEMM arithmetic: it only draws random routing
counts and bf16 tensors, so that the CUDA path and the CPU oracle can be fed
identical inputs.  The workloads mirror the model shapes on the pages:
DeepSeek-V3 16B and 671B (neurabooks.ru, "DeepSeek-V3 now trains 41% faster",
section "Что такое TorchTitan"; aifind.ru, "DeepSeek-V3 ...", section
"Параметры"), Llama 4 Scout (neurabooks.ru, "New data format speeds up
Llama 4 Scout training"), and dropless routing where each expert gets its
real, imbalanced token count (iitak.ru, "NVIDIA ... JAX", dropless paragraph).
The sizes and distributions are the pages' model shapes with synthetic
routing: no dataset is involved, so these synthetic draws stand in for real routing.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass
class Layer:
    """One grouped linear: Y[M, N] = X[M, K] W_e[N, K]^T per expert."""
    name: str
    N: int
    K: int


@dataclass
class Workload:
    name: str
    counts: np.ndarray                 # tokens per expert, int64 [E]
    layers: list = field(default_factory=list)
    x_outlier_frac: float = 0.0        # fraction of X elements scaled
    x_outlier_scale: float = 1.0
    w_std: float = 1.0
    seed: int = 0

    @property
    def E(self) -> int:
        return int(self.counts.size)

    @property
    def M(self) -> int:
        return int(self.counts.sum())

    @property
    def offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.counts)]).astype(np.int32)

    def flops_per_pass(self) -> int:
        """Algorithmic FLOPs of one of fwd/dgrad/wgrad summed over the layers."""
        return sum(2 * self.M * L.N * L.K for L in self.layers)


def _top_k_counts(logits: np.ndarray, k: int) -> np.ndarray:
    """Per-expert token counts of top-k routing (ties: lower index first)."""
    T, E = logits.shape
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    return np.bincount(order.reshape(-1), minlength=E).astype(np.int64)


def tiny() -> Workload:
    """4 experts, counts [0, 7, 21, 36]: one empty expert, none a multiple of 32."""
    return Workload("tiny", np.array([0, 7, 21, 36], dtype=np.int64), [Layer("linear", 128, 256)],
                    w_std=1.0, seed=0)


def tiny_random(seed: int, E: int = 4, M: int = 64) -> np.ndarray:
    """Seeded random counts summing to M with at least one empty expert."""
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.integers(0, M + 1, size=E - 2))
    c = np.diff(np.concatenate([[0], cuts, [M]]))
    counts = np.concatenate([[0], c]).astype(np.int64)
    rng.shuffle(counts)
    return counts


def ds_v3_16b(seed: int = 1) -> Workload:
    """hidden 2048, expert intermediate 1408, 64 experts, top-6 of 8192 tokens.
    Logits N(0,1) plus a per-expert bias N(0, 0.5); top-6 of the softmax is
    top-6 of the logits."""
    rng = np.random.default_rng(seed)
    T, E = 8192, 64
    logits = rng.standard_normal((T, E)) + rng.normal(0.0, 0.5, size=E)[None, :]
    counts = _top_k_counts(logits, 6)
    return Workload("ds-v3-16b", counts, [Layer("gate_up", 2 * 1408, 2048), Layer("down", 2048, 1408)],
                    w_std=0.02, seed=seed)


def ds_v3_671b(seed: int = 2) -> Workload:
    """One GPU's share: 32 local experts of 256, top-8 of 16384 tokens, so a
    balanced share is 16384 rows; counts ~ Multinomial(16384, p), p_j ~ j^-1.1
    (Zipf s = 1.1) with the ranks in a seeded shuffled order.  0.1 % of the
    activations are outliers x100."""
    rng = np.random.default_rng(seed)
    E, M = 32, 16384
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.1
    p = p[rng.permutation(E)]
    counts = rng.multinomial(M, p / p.sum()).astype(np.int64)
    return Workload("ds-v3-671b", counts, [Layer("gate_up", 4096, 7168), Layer("down", 7168, 2048)],
                    x_outlier_frac=1e-3, x_outlier_scale=100.0, w_std=0.02, seed=seed)


def llama4_scout(seed: int = 3) -> Workload:
    """hidden 5120, expert intermediate 8192, 16 experts, top-1 of 16384 tokens."""
    rng = np.random.default_rng(seed)
    T, E = 16384, 16
    counts = _top_k_counts(rng.standard_normal((T, E)), 1)
    return Workload("llama4-scout", counts, [Layer("gate_up", 2 * 8192, 5120), Layer("down", 5120, 8192)],
                    w_std=0.02, seed=seed)


@dataclass
class Routing:
    """Top-k routing of T tokens: expert ids idx[T, k] (int32, distinct per
    token) and combine weights w[T, k] (float32, softmax over the chosen
    logits), plus the token activations' width K."""
    name: str
    E: int
    idx: np.ndarray
    w: np.ndarray
    K: int

    @property
    def T(self) -> int:
        return int(self.idx.shape[0])

    @property
    def k(self) -> int:
        return int(self.idx.shape[1])


def _top_k_routing(name, logits: np.ndarray, k: int, K: int) -> Routing:
    T, E = logits.shape
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    w = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    return Routing(name, E, idx.astype(np.int32), w, K)


def routing(name: str, seed: int | None = None) -> Routing:
    """The routing behind a workload's counts: the same draws as the workload
    generator, kept per token (ds-v3-16b: top-6 of 64 for 8192 tokens, K =
    2048; llama4-scout: top-1 of 16 for 16384 tokens, K = 5120; tiny: top-2
    of 5 for 40 tokens, K = 256)."""
    if name == "ds-v3-16b":
        rng = np.random.default_rng(1 if seed is None else seed)
        T, E = 8192, 64
        logits = rng.standard_normal((T, E)) + rng.normal(0.0, 0.5, size=E)[None, :]
        return _top_k_routing(name, logits, 6, 2048)
    if name == "llama4-scout":
        rng = np.random.default_rng(3 if seed is None else seed)
        return _top_k_routing(name, rng.standard_normal((16384, 16)), 1, 5120)
    if name == "tiny":
        rng = np.random.default_rng(0 if seed is None else seed)
        return _top_k_routing(name, rng.standard_normal((40, 5)), 2, 256)
    raise KeyError(name)


def quantiser_sweep() -> list[tuple[int, int]]:
    return [(m, k) for m in (4096, 16384, 65536) for k in (2048, 5120, 7168)]


WORKLOADS = {"tiny": tiny, "ds-v3-16b": ds_v3_16b, "ds-v3-671b": ds_v3_671b, "llama4-scout": llama4_scout}


# ------------------------------------------------------------------ tensors
def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def with_outliers(x: torch.Tensor, frac: float, scale: float, seed: int) -> torch.Tensor:
    """Multiply a seeded uniform choice of round(frac * numel) elements by scale."""
    if frac <= 0:
        return x
    n = max(1, int(round(frac * x.numel())))
    g = _gen(seed, x.device)
    idx = torch.randint(0, x.numel(), (n,), generator=g, device=x.device)
    flat = x.reshape(-1)
    flat[idx] = (flat[idx].float() * scale).to(torch.bfloat16)
    return x


def zero_tiles(x: torch.Tensor, frac: float, seed: int, tile: int = 32) -> torch.Tensor:
    """Zero a seeded choice of aligned tile x tile blocks (both rowwise and
    colwise quantisation then meet all-zero 32-blocks)."""
    R, C = x.shape
    tr, tc = R // tile, C // tile
    n = max(1, int(round(frac * tr * tc)))
    g = _gen(seed, "cpu")
    pick = torch.randperm(tr * tc, generator=g)[:n]
    for t in pick.tolist():
        r, c = divmod(t, tc)
        x[r * tile:(r + 1) * tile, c * tile:(c + 1) * tile] = 0
    return x


def layer_tensors(w: Workload, layer: Layer, device="cpu", seed_offset: int = 0):
    """(X [M,K], W [E,N,K], dY [M,N]) bf16 for one layer of a workload.
    X and dY ~ N(0,1) (X with the workload's outliers), W ~ N(0, w_std)."""
    base = 1000 * w.seed + 17 * seed_offset + (0 if layer.name in ("gate_up", "linear") else 7)
    X = normal_bf16((w.M, layer.K), 1.0, base + 1, device)
    X = with_outliers(X, w.x_outlier_frac, w.x_outlier_scale, base + 2)
    W = normal_bf16((w.E, layer.N, layer.K), w.w_std, base + 3, device)
    dY = normal_bf16((w.M, layer.N), 1.0, base + 4, device)
    return X, W, dY


def sweep_tensor(M: int, K: int, seed: int = 4, device="cpu") -> torch.Tensor:
    """Quantiser sweep input: N(0,1), 0.1 % outliers x1000, 1 % of aligned
    32x32 tiles zeroed."""
    x = normal_bf16((M, K), 1.0, seed * 7919 + M + K, device)
    x = with_outliers(x, 1e-3, 1000.0, seed * 7919 + M + K + 1)
    if device == "cpu":
        return zero_tiles(x, 0.01, seed)
    return zero_tiles(x.cpu(), 0.01, seed).to(device)


def integer_bf16(shape, lo: int, hi: int, seed: int, device="cpu") -> torch.Tensor:
    """Uniform integers in [lo, hi] as bf16 (exact)."""
    g = _gen(seed, device)
    return torch.randint(lo, hi + 1, shape, generator=g, device=device).to(torch.bfloat16)


def offsets_from_counts(counts) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(counts, dtype=np.int64))]).astype(np.int32)
