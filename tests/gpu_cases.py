"""Shared builders for the GPU parity tests: seeded inputs from synth/, expected
values from oracle/, device tensors for the library. Nothing here computes any
part of the method itself."""
from __future__ import annotations

import functools
from typing import Optional, Sequence

import numpy as np
import torch

import oracle
import synth


def bf16_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to("cuda").view(torch.bfloat16)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda")


def bf16_from_dev(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor -> fp64 NumPy values."""
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@functools.lru_cache(maxsize=16)
def quantised_stack(E: int, N: int, K: int, seed: int, which: str,
                    touched: Optional[tuple] = None):
    """Oracle-quantised N(0, 0.02) weights for the touched experts (all if None);
    untouched experts get random bytes (they are never read)."""
    packed, absmax = synth.random_packed_stack(E, N, K, seed=seed, which=which)
    experts = range(E) if touched is None else touched
    for e in experts:
        packed[e], absmax[e] = oracle.quantize_nf4(
            synth.expert_weights_f32(E, N, K, e, seed=seed, which=which))
    return packed, absmax


def groups_from_routing(w: synth.Workload, seed: int = 0):
    topk = synth.routing(w, seed)
    sorted_idx, sizes, experts, ng = oracle.moe_align(topk, w.E)
    return topk, sizes, experts, ng


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=n - 2, replace=False).tolist())
    rows.update([0, M - 1])
    return np.array(sorted(rows))


def boundaries(sizes: Sequence[int]) -> np.ndarray:
    """First and last row of every non-empty group."""
    out = []
    off = 0
    for s in sizes:
        if s > 0:
            out += [off, off + s - 1]
        off += s
    return np.unique(np.array(out, dtype=np.int64))


def tile_strata(sizes: Sequence[int], seed: int = 0, half: int = 128) -> np.ndarray:
    """One seeded row in every `half`-row slice of every group (the tensor-core
    kernel's token tiles are 256 rows of one group, split into two 128-row
    halves, one per CTA of a pair), plus the first and last row of every
    non-empty group."""
    rng = np.random.default_rng(seed)
    out = [boundaries(sizes)]
    off = 0
    for s in sizes:
        for h0 in range(0, int(s), half):
            h1 = min(int(s), h0 + half)
            out.append(np.array([off + int(rng.integers(h0, h1))]))
        off += int(s)
    return np.unique(np.concatenate(out)).astype(np.int64)
