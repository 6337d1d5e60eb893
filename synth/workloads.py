"""Workload table and seeded generators (no method arithmetic here).

Every generator takes an explicit seed and returns NumPy arrays. Streams are
split with ``numpy.random.SeedSequence.spawn`` so that the router, each GEMM's
weights and each GEMM's activations draw from independent streams, and each
expert's weights from its own child stream (so one expert can be regenerated
without drawing the others).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

# Stream indices under SeedSequence(seed).spawn(N_STREAMS).
_ROUTER, _W_GATE_UP, _W_DOWN, _X_GATE_UP, _X_DOWN, _PACKED = range(6)
N_STREAMS = 6


@dataclass(frozen=True)
class Gemm:
    """One grouped expert GEMM: x[M,K] (bf16) times W[E,N,K/2] (NF4 packed)."""
    name: str          # "gate_up" or "down"
    K: int
    N: int
    swiglu: bool = False


@dataclass(frozen=True)
class Workload:
    name: str
    E: int             # experts in the stack
    top_k: int
    T: int             # tokens; rows M = T * top_k
    gemms: Tuple[Gemm, ...]
    routing: str       # "softmax_topk_forced_empty", "uniform", "zipf1.1", "softmax_topk"
    regime: str        # "decode" or "prefill" (which kernel the shape is meant for)
    forced_empty: Tuple[int, ...] = field(default_factory=tuple)
    description: str = ""

    @property
    def M(self) -> int:
        return self.T * self.top_k


# The five shapes. K and N are the expert GEMM's reduction and output sizes;
# gate_up's N is 2 x the expert intermediate size.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        name="tiny", E=4, top_k=2, T=8,
        gemms=(Gemm("gate_up", K=256, N=128),),
        routing="softmax_topk_forced_empty", regime="decode", forced_empty=(3,),
        description="E=4, K=256, N=128, 8 tokens top-2 (16 rows), expert 3 forced empty",
    ),
    "olmoe": Workload(
        name="olmoe", E=64, top_k=8, T=1,
        gemms=(Gemm("gate_up", K=2048, N=2048), Gemm("down", K=1024, N=2048)),
        routing="uniform", regime="decode",
        description="OLMoE-shaped decode: 64 experts, top-8, 1 token (8 rows)",
    ),
    "qwen3_30b_a3b": Workload(
        name="qwen3_30b_a3b", E=128, top_k=8, T=16,
        gemms=(Gemm("gate_up", K=2048, N=1536), Gemm("down", K=768, N=2048)),
        routing="zipf1.1", regime="decode",
        description="Qwen3-30B-A3B-shaped decode batch: 128 experts, top-8, 16 tokens, Zipf(1.1) router",
    ),
    "gpt_oss_120b": Workload(
        name="gpt_oss_120b", E=128, top_k=4, T=64,
        gemms=(Gemm("gate_up", K=2880, N=5760, swiglu=True), Gemm("down", K=2880, N=2880)),
        routing="uniform", regime="decode",
        description="GPT-OSS-120B-shaped: 128 experts, top-4, 64 tokens, fused SwiGLU on gate_up",
    ),
    "mixtral_8x22b": Workload(
        name="mixtral_8x22b", E=8, top_k=2, T=4096,
        gemms=(Gemm("gate_up", K=6144, N=32768), Gemm("down", K=16384, N=6144)),
        routing="softmax_topk", regime="prefill",
        description="Mixtral-8x22B-shaped prefill: 8 experts, top-2, 4096 tokens (8192 rows)",
    ),
}


def seed_streams(seed: int) -> List[np.random.SeedSequence]:
    return np.random.SeedSequence(seed).spawn(N_STREAMS)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(seed_streams(seed)[stream])


def routing(w: Workload, seed: int = 0) -> np.ndarray:
    """topk_ids int32 [T, top_k] for the workload's router recipe.

    * softmax_topk(_forced_empty): logits ~ N(0,1) per (token, expert); the
      top-k experts by logit (softmax is monotone, so top-k of the softmax is
      top-k of the logits). Forced-empty experts get logit -inf.
    * uniform: top_k distinct experts per token, uniformly without replacement.
    * zipf1.1: expert popularity p(rank) proportional to rank^-1.1 over a seeded
      permutation of the experts; top_k distinct experts per token drawn
      without replacement with probability proportional to p (Gumbel-top-k).
    """
    rng = _rng(seed, _ROUTER)
    T, E, k = w.T, w.E, w.top_k
    if w.routing in ("softmax_topk", "softmax_topk_forced_empty"):
        logits = rng.standard_normal((T, E))
        for e in w.forced_empty:
            logits[:, e] = -np.inf
        ids = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    elif w.routing == "uniform":
        keys = rng.random((T, E))
        ids = np.argsort(keys, axis=1, kind="stable")[:, :k]
    elif w.routing == "zipf1.1":
        perm = rng.permutation(E)
        ranks = np.empty(E, dtype=np.float64)
        ranks[perm] = np.arange(1, E + 1, dtype=np.float64)
        logp = -1.1 * np.log(ranks)
        gumbel = -np.log(-np.log(rng.random((T, E))))
        ids = np.argsort(-(logp[None, :] + gumbel), axis=1, kind="stable")[:, :k]
    else:
        raise ValueError(f"unknown routing {w.routing!r}")
    return np.ascontiguousarray(ids.astype(np.int32))


def _f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest even) and return the 16-bit patterns.

    Input preparation only: activations are defined as bf16 values.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    out = ((u + rounding) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations_bf16(M: int, K: int, seed: int = 0, which: str = "gate_up") -> np.ndarray:
    """x ~ N(0,1) rounded to bf16; returned as uint16 bit patterns [M, K].

    The rows are drawn directly in sorted (grouped) order: the token gather
    that produces sorted activations happens outside the GEMM.
    """
    stream = _X_GATE_UP if which == "gate_up" else _X_DOWN
    rng = _rng(seed, stream)
    return _f32_to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))


def expert_weights_f32(E: int, N: int, K: int, expert: int, seed: int = 0,
                       which: str = "gate_up", std: float = 0.02) -> np.ndarray:
    """fp32 weights of one expert, W_e[N, K] ~ N(0, std^2), from its own stream."""
    stream = _W_GATE_UP if which == "gate_up" else _W_DOWN
    child = seed_streams(seed)[stream].spawn(E)[expert]
    rng = np.random.default_rng(child)
    return rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)


def random_packed_stack(E: int, N: int, K: int, seed: int = 0, which: str = "gate_up",
                        absmax_lo: float = 0.04, absmax_hi: float = 0.06
                        ) -> Tuple[np.ndarray, np.ndarray]:
    """A packed stack drawn directly in the packed domain (no quantiser).

    Bytes are uniform over 0..255 (both 4-bit codes uniform over 16 values) and
    each block scale is uniform on [absmax_lo, absmax_hi], the range in which
    the maximum |w| of 64 draws of N(0, 0.02) typically falls. Used where the
    values do not matter to what is measured (timing) or where a cheap stand-in
    for a multi-GB quantised stack is wanted.
    """
    child = seed_streams(seed)[_PACKED].spawn(2)[0 if which == "gate_up" else 1]
    rng = np.random.default_rng(child)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(absmax_lo, absmax_hi, size=(E, N, K // 64)).astype(np.float32)
    return packed, absmax
