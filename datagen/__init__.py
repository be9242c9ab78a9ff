"""Seeded synthetic inputs for the N:M-pruned linear layer.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds no arithmetic of the pruning method itself: it only draws
Gaussian tensors, scales a few outlier input channels, and stores them as bf16
bit patterns (uint16).

Workload shapes follow the pages' LLM projections:
  * SparseForge (arXiv 2605.06402), "Resultados Experimentais": LLaMA-2-7B layers;
  * SlideSparse (arXiv 2603.05232), section 4: Qwen/Llama prefill shapes and 6:8;
  * Sparse-BitNet (arXiv 2603.05168), section 2: ternary 6:8 layers.

Every tensor is drawn from N(0, sigma) in fp32 with numpy's PCG64 seeded by
(seed, tensor_id), then rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import numpy as np

# tensor ids used to derive independent streams from one seed
TID_W = 1
TID_X = 2
TID_OUTLIER_COLS = 3


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite values never overflow 32 bits here (max 0xFF7FFFFF + 0x8000)
    rounding_bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    out = ((u + rounding_bias) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tensor_id)]))


def normal_f32(shape, sigma: float, seed: int, tensor_id: int) -> np.ndarray:
    g = _rng(seed, tensor_id)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return a


def outlier_columns(K: int, count: int, seed: int) -> np.ndarray:
    """Indices of `count` outlier input channels, chosen by a seeded permutation."""
    if count <= 0:
        return np.zeros(0, dtype=np.int64)
    perm = _rng(seed, TID_OUTLIER_COLS).permutation(K)
    return np.sort(perm[:count]).astype(np.int64)


def make_weight(R: int, K: int, sigma: float, seed: int) -> np.ndarray:
    """W [R x K] (out features x in features), bf16 bits."""
    return f32_to_bf16_bits(normal_f32((R, K), sigma, seed, TID_W))


def make_activations(T: int, K: int, seed: int, n_outliers: int = 0,
                     outlier_scale: float = 20.0, sigma: float = 1.0) -> np.ndarray:
    """X [T x K] activations, N(0, sigma) with `n_outliers` channels scaled, bf16 bits."""
    x = normal_f32((T, K), sigma, seed, TID_X)
    cols = outlier_columns(K, n_outliers, seed)
    if cols.size:
        x[:, cols] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def tie_heavy_scores(R: int, K: int, seed: int, levels: int = 8) -> np.ndarray:
    """Integer-valued fp32 scores in [0, levels) (many exact ties), for tie-break tests."""
    g = _rng(seed, 17)
    return g.integers(0, levels, size=(R, K)).astype(np.float32)


def rademacher_bits(S: int, K: int, seed: int) -> np.ndarray:
    """S random sign vectors of length K as bits: uint32 [S x ceil(K/32)], bit
    k % 32 of word k / 32 set = -1, clear = +1 (bits past K are clear)."""
    g = _rng(seed, 23)
    signs = g.integers(0, 2, size=(S, K), dtype=np.uint8)
    words = np.zeros((S, (K + 31) // 32), dtype=np.uint32)
    for b in range(32):
        col = signs[:, b::32].astype(np.uint32)
        words[:, : col.shape[1]] |= col << np.uint32(b)
    return words


def small_int_bf16(shape, seed: int, tensor_id: int, lo: int = -4, hi: int = 5) -> np.ndarray:
    """Small integers stored as bf16 bits (exact), so fp64 sums of products are exact."""
    g = _rng(seed, tensor_id)
    return f32_to_bf16_bits(g.integers(lo, hi, size=shape).astype(np.float32))


# ---------------------------------------------------------------------------
# Workloads. Each names its shapes and value distributions; sizes follow the
# pages' LLM projections (Llama-7B q/k/v/o 4096x4096, gate/up 11008x4096,
# down 4096x11008; 70B gate/up 28672x8192 and down 8192x28672).
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    R: int            # out features (rows of W)
    K: int            # in features (reduction dim)
    T: int            # tokens of X (GEMM N) and of the calibration set
    n: int
    m: int
    w_sigma: float = 0.02
    x_outliers: int = 0
    score: str = "hessian"   # "hessian" (s=(H+eps)W^2) or "magnitude" (|W_latent|)
    ternary: bool = False    # quantise W to gamma*{-1,0,+1} before compression
    eps: float = 1e-8
    seed: int = 0


def _c3_layers():
    out = []
    for nm, R, K in (("q", 4096, 4096), ("gate", 11008, 4096), ("down", 4096, 11008)):
        for T in (16, 128, 2048, 8192):
            out.append(Layer(f"llama7b_{nm}_T{T}", R, K, T, 2, 4,
                             x_outliers=int(round(0.01 * K))))
    return out


def _c5_layers():
    out = []
    for nm, R, K in (("up", 28672, 8192), ("down", 8192, 28672)):
        for (n, m) in ((2, 4), (4, 6), (6, 8), (8, 10)):
            out.append(Layer(f"llama70b_{nm}_{n}of{m}", R, K, 4096, n, m, w_sigma=0.015))
    return out


WORKLOADS = {
    # small 2:4 layer with 4 outlier channels (oracle finishes in well under a second)
    "small_2of4": Layer("small_2of4", 256, 512, 128, 2, 4, x_outliers=4),
    # 6:8 via the 3-window slide, 4096x4096, 2048 tokens, scores from the same X
    "slide_6of8_4096": Layer("slide_6of8_4096", 4096, 4096, 2048, 6, 8),
    # ternary 6:8 layer, latent-magnitude score, gate/up shape 11008x4096
    "ternary_6of8_gate": Layer("ternary_6of8_gate", 11008, 4096, 4096, 6, 8,
                               score="magnitude", ternary=True),
}
for _l in _c3_layers() + _c5_layers():
    WORKLOADS[_l.name] = _l


def layer_inputs(layer: Layer, seed: int | None = None):
    """Host inputs for a workload: (X [T x K] bf16 bits, W [R x K] bf16 bits)."""
    s = layer.seed if seed is None else seed
    W = make_weight(layer.R, layer.K, layer.w_sigma, s)
    X = make_activations(layer.T, layer.K, s, n_outliers=layer.x_outliers)
    return X, W
