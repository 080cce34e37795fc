"""Seeded synthetic bf16 weight generators for the five workloads.

This module only draws inputs.  It holds none of the coding arithmetic and
imports neither the oracle nor the product; both sides are fed the same bits.

Every tensor is returned as a flat ``torch.bfloat16`` tensor on the requested
device.  Values are drawn in fp32 and rounded to bf16 with round-to-nearest-
even (``Tensor.to(torch.bfloat16)``); bit-pattern workloads (4a, 4b, 4b', 4c)
are built as integers and only reinterpreted, so NaN payloads stay raw.

Torch draws CPU tensors with mt19937 and CUDA tensors with Philox, so the same
seed gives different (identically distributed) bits on the two devices; each
test or benchmark draws once and hands the same bits to everything it checks.

Workloads (sizes in weights):
  c1   1024x1024, N(0, 0.02), seed 0
  c2   4096x4096, Student-t(4) scaled to std 0.02, plus round(0.001 n) exact
       +0.0 at seeded positions, seed 1
  c3   one Llama-2-7B-shaped block (q,k,v,o 4096x4096; gate,up 4096x11008;
       down 11008x4096), N(0, s_j) with s_j ~ U[0.01, 0.04] drawn from seed 2
  c4a  64M, two exponents (126, 127) equally likely, sign/mantissa uniform
  c4b  64M, all 256 exponents, geometric counts (ratio 1/2, floor 1)
  c4bp 64M, 34 Fibonacci counts plus 222 equal pool symbols (length cap binds)
  c4c  64M, uniform random 16-bit patterns
  c5   Llama-3-8B-shaped model: 32 blocks (q 4096x4096, k,v 1024x4096,
       o 4096x4096, gate,up 14336x4096, down 4096x14336) plus embedding and
       lm_head 128256x4096, N(0, 0.02), seed 4; one code table per block
Tensor j of a workload with seed s is drawn with seed 1000*s + j.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

N64M = 64 * 1024 * 1024


@dataclass(frozen=True)
class TensorSpec:
    name: str
    numel: int
    kind: str  # "normal", "student_t", "two_exp", "geometric", "fibonacci", "uniform_bits"
    seed: int
    std: float = 0.02
    zero_frac: float = 0.0


@dataclass
class BlockSpec:
    """Tensors that share one code table (a transformer block, or one tensor)."""
    name: str
    tensors: list = field(default_factory=list)

    @property
    def numel(self) -> int:
        return sum(t.numel for t in self.tensors)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_fp32(n: int, seed: int, device) -> torch.Tensor:
    return torch.randn(n, generator=_gen(seed, device), device=device, dtype=torch.float32)


def _bits_to_bf16(bits_i32: torch.Tensor) -> torch.Tensor:
    return bits_i32.to(torch.int16).view(torch.bfloat16)


def _uniform_int(n: int, hi: int, g: torch.Generator, device) -> torch.Tensor:
    return torch.randint(0, hi, (n,), generator=g, device=device, dtype=torch.int32)


def geometric_counts(n: int) -> np.ndarray:
    """Counts per rank r = 0..255: max(1, floor(n / 2^(r+1))), with rank 0
    absorbing the difference so the counts sum to n (needs n >= 512)."""
    c = np.array([max(1, n >> (r + 1)) for r in range(256)], dtype=np.int64)
    c[0] += n - int(c.sum())
    assert c[0] > 0 and int(c.sum()) == n
    return c


def fibonacci_counts(n: int) -> np.ndarray:
    """34 Fibonacci counts 1,1,2,...,F34 then 222 pool symbols sharing the rest."""
    fib = [1, 1]
    while len(fib) < 34:
        fib.append(fib[-1] + fib[-2])
    rest = n - sum(fib)
    assert rest >= 222, "fibonacci workload needs n > F36"
    pool = np.full(222, rest // 222, dtype=np.int64)
    pool[: rest % 222] += 1
    c = np.concatenate([np.array(fib, dtype=np.int64), pool])
    assert int(c.sum()) == n
    return c


def _exponent_bits(counts: np.ndarray, n: int, g: torch.Generator, device) -> torch.Tensor:
    """Exponent fields with exactly the given counts; ranks mapped to exponent
    values by a seeded permutation, positions shuffled by a seeded permutation."""
    perm_sym = torch.randperm(256, generator=g, device="cpu" if device == "cpu" else device).cpu()
    exps = torch.repeat_interleave(perm_sym.to(torch.int32), torch.from_numpy(counts))
    exps = exps.to(device)
    pos = torch.randperm(n, generator=g, device=device)
    return exps[pos]


def generate(spec: TensorSpec, device="cpu") -> torch.Tensor:
    """Draws one flat bf16 tensor for ``spec`` on ``device``."""
    n = spec.numel
    if spec.kind == "normal":
        return (_normal_fp32(n, spec.seed, device) * spec.std).to(torch.bfloat16)
    g = _gen(spec.seed, device)
    if spec.kind == "student_t":
        # t(4) = Z / sqrt(V/4), V = sum of four squared standard normals;
        # Var t(4) = 2, so scale by std/sqrt(2).
        z = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        v = torch.zeros(n, device=device, dtype=torch.float32)
        for _ in range(4):
            y = torch.randn(n, generator=g, device=device, dtype=torch.float32)
            v.addcmul_(y, y)
        x = z / torch.sqrt(v / 4.0) * (spec.std / math.sqrt(2.0))
        out = x.to(torch.bfloat16)
        nz = int(round(spec.zero_frac * n))
        if nz:
            pos = torch.randperm(n, generator=g, device=device)[:nz]
            out[pos] = 0.0
        return out
    if spec.kind == "two_exp":
        e = 126 + _uniform_int(n, 2, g, device)
        sm = _uniform_int(n, 256, g, device)
        bits = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)
        return _bits_to_bf16(bits)
    if spec.kind in ("geometric", "fibonacci"):
        counts = geometric_counts(n) if spec.kind == "geometric" else fibonacci_counts(n)
        e = _exponent_bits(counts, n, g, device)
        sm = _uniform_int(n, 256, g, device)
        bits = ((sm & 0x80) << 8) | (e << 7) | (sm & 0x7F)
        return _bits_to_bf16(bits)
    if spec.kind == "uniform_bits":
        return _bits_to_bf16(_uniform_int(n, 65536, g, device))
    raise ValueError(f"unknown kind {spec.kind}")


def as_u16_numpy(t: torch.Tensor) -> np.ndarray:
    """Host numpy uint16 view of a bf16 tensor's bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)


# ---------------------------------------------------------------- workloads

def c1() -> BlockSpec:
    return BlockSpec("c1", [TensorSpec("w", 1024 * 1024, "normal", 0, 0.02)])


def c2() -> BlockSpec:
    return BlockSpec("c2", [TensorSpec("w", 4096 * 4096, "student_t", 1000, 0.02, zero_frac=0.001)])


LLAMA2_7B_BLOCK = [("q", 4096 * 4096), ("k", 4096 * 4096), ("v", 4096 * 4096), ("o", 4096 * 4096),
                   ("gate", 4096 * 11008), ("up", 4096 * 11008), ("down", 11008 * 4096)]


def c3() -> BlockSpec:
    rng = np.random.default_rng(2)
    stds = rng.uniform(0.01, 0.04, size=len(LLAMA2_7B_BLOCK))
    return BlockSpec("c3", [TensorSpec(nm, sz, "normal", 2000 + j, float(stds[j]))
                            for j, (nm, sz) in enumerate(LLAMA2_7B_BLOCK)])


def c4(which: str, n: int = N64M) -> BlockSpec:
    kind, sub = {"a": ("two_exp", 30), "b": ("geometric", 31), "bp": ("fibonacci", 33),
                 "c": ("uniform_bits", 32)}[which]
    return BlockSpec(f"c4{which}", [TensorSpec("w", n, kind, 1000 * sub)])


LLAMA3_8B_BLOCK = [("q", 4096 * 4096), ("k", 1024 * 4096), ("v", 1024 * 4096), ("o", 4096 * 4096),
                   ("gate", 14336 * 4096), ("up", 14336 * 4096), ("down", 4096 * 14336)]
LLAMA3_8B_VOCAB = 128256
LLAMA3_8B_LAYERS = 32


def c5() -> list[BlockSpec]:
    """34 code-table scopes: embedding, 32 transformer blocks, lm_head."""
    blocks = [BlockSpec("embed", [TensorSpec("embed", LLAMA3_8B_VOCAB * 4096, "normal", 4000 + 224, 0.02)])]
    for layer in range(LLAMA3_8B_LAYERS):
        blocks.append(BlockSpec(f"layer{layer}", [
            TensorSpec(nm, sz, "normal", 4000 + 7 * layer + j, 0.02)
            for j, (nm, sz) in enumerate(LLAMA3_8B_BLOCK)]))
    blocks.append(BlockSpec("lm_head", [TensorSpec("lm_head", LLAMA3_8B_VOCAB * 4096, "normal", 4000 + 225, 0.02)]))
    return blocks


def c5_numel() -> int:
    return sum(b.numel for b in c5())


def scaled(block: BlockSpec, n_total: int) -> BlockSpec:
    """The same recipe with every tensor shrunk proportionally (at least one
    weight each) so the block holds about ``n_total`` weights."""
    f = n_total / block.numel
    return BlockSpec(block.name + f"@{n_total}",
                     [TensorSpec(t.name, max(1, int(t.numel * f)), t.kind, t.seed, t.std, t.zero_frac)
                      for t in block.tensors])


def generate_block(block: BlockSpec, device="cpu") -> list[torch.Tensor]:
    return [generate(t, device) for t in block.tensors]


def matrix_cols(t: TensorSpec) -> int:
    """Columns (input features) of a tensor read as a row-major [out, in]
    matrix: transformer matrices take the 4096-wide hidden state except the
    MLP down projection, which takes the intermediate state; a square test
    matrix takes its side."""
    if t.name == "down":
        return t.numel // 4096
    if t.name == "w":
        return int(round(t.numel ** 0.5))
    return 4096
