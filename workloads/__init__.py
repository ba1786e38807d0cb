"""Seeded synthetic BF16 weight generators shared by the tests, the benchmark
and the oracle drivers.

This module holds no part of the compression method: it only draws random
numbers and rounds them to BF16.  Real model weights are not used anywhere;
these generators stand in for them with the shapes of the models the DFloat11
pages discuss (Llama-3.1-8B / 70B) and with weight-like value distributions.

All arrays are returned as ``numpy.uint16`` BF16 bit patterns.

Recipes:

* ``normal_matrix(rows, cols, std, seed)`` -- i.i.d. N(0, std^2) float32,
  rounded to BF16.  1024x1024 / seed 0 and 4096x4096 / seed 1 are the
  single-matrix workloads.
* ``llama8b_block(seed)`` -- one Llama-3.1-8B-shaped transformer block:
  q, k, v, o, gate, up, down drawn in that order, each with its own scale
  s ~ U[0.01, 0.05] drawn just before its weights, followed by the two
  RMSNorm vectors of 4096 drawn from N(1, 0.02^2).  218,112,000 weights.
* ``heavy_tail_matrix(seed)`` -- a 28672x8192 70B-MLP-shaped matrix,
  Student-t(nu=3) * 0.015, then 0.1% of positions set to +0.0 and 0.01% to
  +-U[1, 30] (disjoint positions, drawn without replacement).
* ``adversarial(name)`` -- small fixed tensors for edge cases (every BF16 bit
  pattern, all-equal, two-valued, uniform random u16, ...).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "LLAMA8B_BLOCK_SHAPES",
    "LLAMA8B_BLOCK_NAMES",
    "round_to_bf16",
    "normal_matrix",
    "llama8b_block",
    "llama8b_block_sizes",
    "heavy_tail_matrix",
    "adversarial",
    "ADVERSARIAL_NAMES",
]

# nn.Linear weight shapes are [out_features, in_features].
LLAMA8B_BLOCK_NAMES = ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj",
                       "up_proj", "down_proj", "input_layernorm",
                       "post_attention_layernorm")
LLAMA8B_BLOCK_SHAPES = ((4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096),
                        (14336, 4096), (14336, 4096), (4096, 14336),
                        (4096,), (4096,))


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to BF16 (round to nearest, ties to even) by integer
    arithmetic and return the uint16 bit patterns.  Inputs here are finite, so
    the NaN case of the rounding rule never arises."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    # Process in slices to bound the temporary memory on very large inputs.
    flat_u = u.reshape(-1)
    flat_o = out.reshape(-1)
    step = 1 << 24
    for i in range(0, flat_u.size, step):
        s = flat_u[i:i + step]
        lsb = (s >> np.uint32(16)) & np.uint32(1)
        flat_o[i:i + step] = ((s + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    return out


def normal_matrix(rows: int, cols: int, std: float = 0.02, seed: int = 0) -> np.ndarray:
    """i.i.d. N(0, std^2) weights of shape [rows, cols], as BF16 bits."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    x *= np.float32(std)
    return round_to_bf16(x)


def llama8b_block_sizes() -> list[int]:
    return [int(np.prod(s)) for s in LLAMA8B_BLOCK_SHAPES]


def llama8b_block(seed: int = 0) -> list[np.ndarray]:
    """The nine weight tensors of one Llama-3.1-8B-shaped block, in the order
    q, k, v, o, gate, up, down, input_norm, post_attention_norm."""
    rng = np.random.default_rng(seed)
    out: list[np.ndarray] = []
    for shape in LLAMA8B_BLOCK_SHAPES[:7]:
        s = np.float32(rng.uniform(0.01, 0.05))
        x = rng.standard_normal(shape, dtype=np.float32)
        x *= s
        out.append(round_to_bf16(x))
    for shape in LLAMA8B_BLOCK_SHAPES[7:]:
        x = rng.standard_normal(shape, dtype=np.float32)
        x *= np.float32(0.02)
        x += np.float32(1.0)
        out.append(round_to_bf16(x))
    return out


def heavy_tail_matrix(seed: int = 4, rows: int = 28672, cols: int = 8192) -> np.ndarray:
    """Student-t(3) * 0.015 with 0.1% exact zeros and 0.01% outliers of
    magnitude U[1, 30] with random sign, at disjoint random positions."""
    rng = np.random.default_rng(seed)
    n = rows * cols
    x = np.empty(n, dtype=np.float32)
    step = 1 << 24
    for i in range(0, n, step):
        m = min(step, n - i)
        x[i:i + m] = (rng.standard_t(3.0, size=m) * 0.015).astype(np.float32)
    n_zero = n // 1000
    n_out = n // 10000
    pos = rng.choice(n, size=n_zero + n_out, replace=False)
    x[pos[:n_zero]] = np.float32(0.0)
    mag = rng.uniform(1.0, 30.0, size=n_out).astype(np.float32)
    sign = np.where(rng.integers(0, 2, size=n_out) == 1, np.float32(1.0), np.float32(-1.0))
    x[pos[n_zero:]] = mag * sign
    return round_to_bf16(x).reshape(rows, cols)


ADVERSARIAL_NAMES = ("all_bf16_patterns", "all_zero", "all_equal", "two_values",
                     "random_u16", "neg_zero_and_nan", "single", "empty",
                     "subnormals", "ragged_normal", "uniform_exponents",
                     "fibonacci_exponents")


def adversarial(name: str, seed: int = 7) -> np.ndarray:
    """Small edge-case tensors (BF16 bit patterns)."""
    rng = np.random.default_rng(seed)
    if name == "all_bf16_patterns":
        # Every one of the 65,536 bit patterns: +-0, subnormals, +-Inf, NaNs.
        a = np.arange(65536, dtype=np.uint32).astype(np.uint16)
        return a[rng.permutation(a.size)]
    if name == "all_zero":
        return np.zeros(100_003, dtype=np.uint16)
    if name == "all_equal":
        return np.full(77_777, 0x3F80, dtype=np.uint16)  # 1.0
    if name == "two_values":
        return np.where(rng.integers(0, 2, 50_001) == 1, 0x3C00, 0xBF00).astype(np.uint16)
    if name == "random_u16":
        return rng.integers(0, 65536, size=300_007, dtype=np.uint32).astype(np.uint16)
    if name == "neg_zero_and_nan":
        vals = np.array([0x8000, 0x0000, 0x7FC0, 0xFFC1, 0x7F80, 0xFF80, 0x7F81], dtype=np.uint16)
        return vals[rng.integers(0, vals.size, 10_000)]
    if name == "single":
        return np.array([0x3F81], dtype=np.uint16)
    if name == "empty":
        return np.zeros(0, dtype=np.uint16)
    if name == "subnormals":
        return rng.integers(0, 0x80, size=20_000, dtype=np.uint32).astype(np.uint16) | (
            rng.integers(0, 2, size=20_000, dtype=np.uint32).astype(np.uint16) << np.uint16(15))
    if name == "ragged_normal":
        # A length that is not a multiple of any tile or vector width.
        x = rng.standard_normal(1_234_567, dtype=np.float32) * np.float32(0.02)
        return round_to_bf16(x)
    if name == "uniform_exponents":
        # All 256 exponent values equally often, random sign and mantissa.
        e = np.repeat(np.arange(256, dtype=np.uint32), 1024)
        e = e[rng.permutation(e.size)]
        sm = rng.integers(0, 256, size=e.size, dtype=np.uint32)
        return (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    if name == "fibonacci_exponents":
        # Exponent frequencies 1, 1, 2, 3, 5, ... over 26 values: unlimited
        # Huffman depth 25, so a length cap below that is forced to bind.
        fib = [1, 1]
        while len(fib) < 26:
            fib.append(fib[-1] + fib[-2])
        e = np.concatenate([np.full(f, 100 + i, dtype=np.uint32) for i, f in enumerate(fib)])
        e = e[rng.permutation(e.size)]
        sm = rng.integers(0, 256, size=e.size, dtype=np.uint32)
        return (((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)).astype(np.uint16)
    raise KeyError(name)
