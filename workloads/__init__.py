"""Seeded synthetic BF16 weight tensors for the DF11 decode path.

This module serves both sides: the CPU oracle's tests and the CUDA path's
tests and benchmark.  It holds none of the codec's arithmetic: it only draws
random numbers and rounds fp32 samples to BF16 (round to nearest even, as
``torch.Tensor.to(torch.bfloat16)`` does).

The shapes stand in for a Qwen3-8B checkpoint (the model the DFloat11 pages
benchmark; real weights are not available, so values are drawn from the
distributions stated in each workload's docstring).  Every function returns a
1-D ``torch.int16`` tensor holding the BF16 bit patterns, on ``device``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

HIDDEN = 4096
INTERMEDIATE = 12288
KV_OUT = 1024
VOCAB = 151936
LAYERS = 36

# (name, out_features, in_features): one Qwen3-8B-shaped transformer block
BLOCK_SHAPES = [
    ("q_proj", HIDDEN, HIDDEN),
    ("k_proj", KV_OUT, HIDDEN),
    ("v_proj", KV_OUT, HIDDEN),
    ("o_proj", HIDDEN, HIDDEN),
    ("gate_proj", INTERMEDIATE, HIDDEN),
    ("up_proj", INTERMEDIATE, HIDDEN),
    ("down_proj", HIDDEN, INTERMEDIATE),
]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_bf16(n: int, std: float, seed: int, device="cpu",
                  mean: float = 0.0) -> torch.Tensor:
    """n samples of N(mean, std^2) in fp32, rounded to BF16 (RNE)."""
    g = _gen(seed, device)
    x = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x.to(torch.bfloat16).view(torch.int16)


def single_matrix(seed: int = 0, device="cpu", rows: int = 1024,
                  cols: int = 1024) -> torch.Tensor:
    """One 1024x1024 matrix, N(0, 0.02)."""
    return gaussian_bf16(rows * cols, 0.02, seed, device)


@dataclass
class NamedTensor:
    name: str
    shape: tuple
    bits: torch.Tensor  # int16 BF16 bit patterns, flattened


def block_tensor(seed: int, index: int, device="cpu", scale: int = 1) -> torch.Tensor:
    """Weight `index` (order of BLOCK_SHAPES) of one Qwen3-8B-shaped block,
    N(0, 1/sqrt(fan_in)) with fan_in = in_features.  `scale` > 1 divides the
    out-features (rows) for small CPU-sized variants."""
    name, rows, cols = BLOCK_SHAPES[index]
    r = max(1, rows // scale)
    return gaussian_bf16(r * cols, 1.0 / math.sqrt(cols), seed * 131 + index, device)


def block_tensors(seed: int = 0, device="cpu", scale: int = 1):
    """The seven weights of one Qwen3-8B-shaped block (see block_tensor);
    scale 1 gives the full 192,937,984-element block."""
    out = []
    for i, (name, rows, cols) in enumerate(BLOCK_SHAPES):
        r = max(1, rows // scale)
        out.append(NamedTensor(name, (r, cols), block_tensor(seed, i, device, scale)))
    return out


def adversarial_mix(n: int = 64 * 1024 * 1024, seed: int = 0,
                    device="cpu") -> torch.Tensor:
    """98.9% N(0,0.02), 0.1% N(0,2.0) outliers, 0.5% exact +0.0, 0.5% N(1,0.05)
    norm-like values; counts floor(f*n) with the remainder going to the last
    class; shuffled by seed."""
    fr = [0.989, 0.001, 0.005]
    counts = [int(math.floor(f * n)) for f in fr]
    counts.append(n - sum(counts))
    g = _gen(seed, device)
    parts = [
        torch.randn(counts[0], generator=g, device=device) * 0.02,
        torch.randn(counts[1], generator=g, device=device) * 2.0,
        torch.zeros(counts[2], device=device),
        torch.randn(counts[3], generator=g, device=device) * 0.05 + 1.0,
    ]
    x = torch.cat(parts)
    perm = torch.randperm(n, generator=g, device=device)
    return x[perm].to(torch.bfloat16).view(torch.int16)


def fibonacci_exponents(seed: int = 0, device="cpu", symbols: int = 34,
                        first_exponent: int = 100) -> torch.Tensor:
    """Exponent counts F1..F_symbols (Fibonacci numbers) over consecutive
    exponent values; random sign and mantissa bits; shuffled.  With 34
    symbols the unconstrained Huffman tree is 33 deep, so a 32-bit cap has to
    be enforced."""
    fib = [1, 1]
    while len(fib) < symbols:
        fib.append(fib[-1] + fib[-2])
    fib = fib[:symbols]
    exps = torch.cat([torch.full((c,), first_exponent + i, dtype=torch.int32)
                      for i, c in enumerate(fib)])
    n = exps.numel()
    g = _gen(seed, "cpu")
    sm = torch.randint(0, 256, (n,), generator=g, dtype=torch.int32)
    perm = torch.randperm(n, generator=g)
    exps = exps[perm]
    w = ((sm & 0x80) << 8) | (exps << 7) | (sm & 0x7F)
    w = torch.where(w >= 32768, w - 65536, w).to(torch.int16)
    return w.to(device)


def all_bf16_patterns(device="cpu") -> torch.Tensor:
    """Every one of the 65,536 BF16 bit patterns (NaNs, +-Inf, +-0,
    subnormals)."""
    w = torch.arange(65536, dtype=torch.int32)
    w = torch.where(w >= 32768, w - 65536, w).to(torch.int16)
    return w.to(device)


def embedding(seed: int = 0, device="cpu", rows: int = VOCAB,
              cols: int = HIDDEN) -> torch.Tensor:
    """151936 x 4096, N(0, 0.02)."""
    return gaussian_bf16(rows * cols, 0.02, seed, device)


def stack_units(seed: int = 0, layers: int = LAYERS):
    """The decode units of the full stack, in forward order: embedding, then
    36 blocks of seven weights (separate seeds), then the LM head.  Returns a
    list of (name, shape, generator thunk(device)) so that callers can
    materialise one unit at a time."""
    units = [("embed_tokens", (VOCAB, HIDDEN),
              lambda d, s=seed: embedding(s * 7919 + 1, d))]
    for layer in range(layers):
        for i, (name, rows, cols) in enumerate(BLOCK_SHAPES):
            def thunk(d, layer=layer, i=i, cols=cols, rows=rows):
                return gaussian_bf16(rows * cols, 1.0 / math.sqrt(cols),
                                     (seed * 1000 + layer) * 131 + i, d)
            units.append((f"layers.{layer}.{name}", (rows, cols), thunk))
    units.append(("lm_head", (VOCAB, HIDDEN),
                  lambda d, s=seed: embedding(s * 7919 + 2, d)))
    return units


def as_numpy_u16(bits: torch.Tensor):
    """Host numpy uint16 view of an int16 bit-pattern tensor."""
    return bits.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
