"""CPU oracle for the grouped NF4 W4A16 expert GEMM -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never calls it and
shares no code with it. Every function is a thin NumPy wrapper over the plain C
in ``gnf4_oracle.c`` (fp64 accumulation, no blocking or reordering beyond the
definitions), compiled by :func:`build` with gcc.

Functions and the passages they follow (page: "grouped-nf4-gemm -- single-launch
W4A16 GEMM over fused NF4 MoE expert stacks", PyPI README of
grouped_nf4_gemm 0.1.0, opening section, unless stated):

* :func:`nf4_table` -- the NF4 code table of the bitsandbytes ``gemm_4bit``
  layout the page names (the table itself is the QLoRA-published one).
* :func:`quantize_nf4` -- blockwise fp32 absmax (64 K-elements per block),
  nearest-code quantisation; input preparation only.
* :func:`dequant_f32` / :func:`dequant_bf16` -- NF4[code] * absmax as one fp32
  multiply, optionally rounded once to bf16 (the materialised weight of the
  baseline the page says the fused kernel replaces).
* :func:`moe_align` -- the token->expert sort producing (sizes, expert_ids).
* :func:`grouped_gemm_f64` -- the grouped GEMM by definition, in fp64.
* :func:`swiglu_f64` -- silu(gate) * up on the gate_up output (package page
  "grouped-nf4-gemm", "Owns": the decode glue includes swiglu).
* :func:`baseline_bf16` -- dequantise-to-bf16 then fp32-accumulated matmul,
  the fidelity comparator of the page's "The claim" section;
  :func:`baseline_swiglu_bf16` -- that baseline's SwiGLU: silu(gate) * up in
  fp32 on its bf16 gate_up output, rounded once to bf16.
* :func:`grouped_dgrad_f64` -- the gradient of the grouped GEMM with respect
  to its activations, dx = dy . W per group, in fp64 (package page
  "grouped-nf4-gemm", header block, "Owns": the grouped packed GEMM and its
  dgrad).
* :func:`grouped_gemm_mxfp4_f64` / :func:`e2m1_table` -- the same GEMM over
  native MXFP4 (e2m1 codes, e8m0 scale per 32; package page "Direct answer");
  :func:`grouped_gemm_bf16_absmax_f64` -- NF4 with bf16 absmax (a bf16 value
  widens to fp32 exactly); :func:`swiglu_interleaved_f64` -- the gpt-oss
  gated activation on interleaved, clamped gate/up columns;
  :func:`gather_rows` -- x[i] = hidden[sorted_idx[i] // top_k].
* :func:`router_topk` / :func:`moe_combine` -- the router's top-k with softmax
  weights, and the top-k weighted combine after the down projection (package
  page "grouped-nf4-gemm", "Use this when": router softmax and top-k and the
  top-k combine among the small decode launches; "Owns": combine among the
  decode glue kernels).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gnf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-std=c99"]

_lib = None


class OracleError(RuntimeError):
    pass


_STATUS = {1: "bad shape", 2: "sizes do not sum to M (or negative)", 3: "expert id out of range",
           4: "topk id out of range", 5: "sorted_idx entry out of range"}


def build(force: bool = False) -> str:
    """Compile gnf4_oracle.c to liboracle.so (gcc, OpenMP) if it is stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", *_CFLAGS, _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_nf4_table.argtypes = [P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_f32_to_bf16.argtypes = [P, i64, P]
        lib.oracle_quantize_nf4.argtypes = [P, i64, i64, P, P]
        lib.oracle_dequant_f32.argtypes = [P, P, i64, i64, P]
        lib.oracle_dequant_bf16.argtypes = [P, P, i64, i64, P]
        lib.oracle_moe_align.argtypes = [P, i64, i32, i32, P, P, P, P]
        lib.oracle_grouped_gemm_f64.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, P, i64, P]
        lib.oracle_swiglu_f64.argtypes = [P, i64, i32, P]
        lib.oracle_baseline_bf16.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, P, i64, P]
        lib.oracle_baseline_swiglu_bf16.argtypes = [P, i64, i32, P]
        lib.oracle_e2m1_table.argtypes = [P]
        lib.oracle_grouped_gemm_mxfp4_f64.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, P,
                                                      i64, P]
        lib.oracle_swiglu_interleaved_f64.argtypes = [P, i64, i32, ctypes.c_double,
                                                      ctypes.c_double, P]
        lib.oracle_gather_rows.argtypes = [P, i64, i32, P, i64, i32, P]
        lib.oracle_router_topk.argtypes = [P, i64, i32, i32, i32, P, P]
        lib.oracle_moe_combine.argtypes = [P, P, P, i64, i32, i32, P]
        lib.oracle_grouped_dgrad_f64.argtypes = [P, P, P, P, P, i32, i64, i32, i32, i32, P]
        for name in ("oracle_quantize_nf4", "oracle_dequant_f32", "oracle_dequant_bf16",
                     "oracle_moe_align", "oracle_grouped_gemm_f64", "oracle_swiglu_f64",
                     "oracle_baseline_bf16", "oracle_baseline_swiglu_bf16", "oracle_router_topk",
                     "oracle_moe_combine", "oracle_grouped_dgrad_f64",
                     "oracle_grouped_gemm_mxfp4_f64", "oracle_swiglu_interleaved_f64",
                     "oracle_gather_rows"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(st: int):
    if st != 0:
        raise OracleError(_STATUS.get(st, f"status {st}"))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def nf4_table() -> np.ndarray:
    out = np.empty(16, dtype=np.float32)
    _load().oracle_nf4_table(_p(out))
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16(_p(a), a.size, _p(out))
    return out


def quantize_nf4(w: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """fp32 [..., K] -> (packed uint8 [..., K/2], absmax fp32 [..., K/64])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    K = w.shape[-1]
    R = w.size // K
    packed = np.empty(w.shape[:-1] + (K // 2,), dtype=np.uint8)
    absmax = np.empty(w.shape[:-1] + (K // 64,), dtype=np.float32)
    _check(_load().oracle_quantize_nf4(_p(w), R, K, _p(packed), _p(absmax)))
    return packed, absmax


def _rk(packed: np.ndarray) -> Tuple[int, int]:
    K = packed.shape[-1] * 2
    return packed.size // packed.shape[-1], K


def dequant_f32(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    R, K = _rk(packed)
    out = np.empty(packed.shape[:-1] + (K,), dtype=np.float32)
    _check(_load().oracle_dequant_f32(_p(packed), _p(absmax), R, K, _p(out)))
    return out


def dequant_bf16(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """bf16 bit patterns [..., K]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    R, K = _rk(packed)
    out = np.empty(packed.shape[:-1] + (K,), dtype=np.uint16)
    _check(_load().oracle_dequant_bf16(_p(packed), _p(absmax), R, K, _p(out)))
    return out


def moe_align(topk_ids: np.ndarray, E: int):
    """-> (sorted_idx [T*k], sizes [E], expert_ids [E], num_groups)."""
    topk_ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, k = topk_ids.shape
    sorted_idx = np.empty(T * k, dtype=np.int32)
    sizes = np.empty(E, dtype=np.int32)
    expert_ids = np.empty(E, dtype=np.int32)
    ng = np.zeros(1, dtype=np.int32)
    _check(_load().oracle_moe_align(_p(topk_ids), T, k, E, _p(sorted_idx), _p(sizes),
                                    _p(expert_ids), _p(ng)))
    return sorted_idx, sizes, expert_ids, int(ng[0])


def _gemm_args(x, w, absmax, sizes, expert_ids, rows):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    sizes = np.ascontiguousarray(sizes, dtype=np.int32)
    expert_ids = np.ascontiguousarray(expert_ids, dtype=np.int32)
    M, K = x.shape
    E, N, Kh = w.shape
    if Kh * 2 != K:
        raise OracleError("bad shape")
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
    return x, w, absmax, sizes, expert_ids, rows, M, N, K, E


def grouped_gemm_f64(x: np.ndarray, w: np.ndarray, absmax: np.ndarray, sizes: np.ndarray,
                     expert_ids: np.ndarray, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """y fp64 [len(rows) or M, N]; x as bf16 bit patterns [M, K]."""
    x, w, absmax, sizes, expert_ids, rows, M, N, K, E = _gemm_args(x, w, absmax, sizes,
                                                                   expert_ids, rows)
    nrows = M if rows is None else rows.size
    y = np.empty((nrows, N), dtype=np.float64)
    _check(_load().oracle_grouped_gemm_f64(
        _p(x), _p(w), _p(absmax), _p(sizes), _p(expert_ids), sizes.size, M, N, K, E,
        None if rows is None else _p(rows), nrows, _p(y)))
    return y


def swiglu_f64(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    M, N = y.shape
    out = np.empty((M, N // 2), dtype=np.float64)
    _check(_load().oracle_swiglu_f64(_p(y), M, N, _p(out)))
    return out


def baseline_bf16(x: np.ndarray, w: np.ndarray, absmax: np.ndarray, sizes: np.ndarray,
                  expert_ids: np.ndarray, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Dequantise-to-bf16-then-matmul emulation; bf16 bit patterns [rows, N]."""
    x, w, absmax, sizes, expert_ids, rows, M, N, K, E = _gemm_args(x, w, absmax, sizes,
                                                                   expert_ids, rows)
    nrows = M if rows is None else rows.size
    y = np.empty((nrows, N), dtype=np.uint16)
    _check(_load().oracle_baseline_bf16(
        _p(x), _p(w), _p(absmax), _p(sizes), _p(expert_ids), sizes.size, M, N, K, E,
        None if rows is None else _p(rows), nrows, _p(y)))
    return y


def baseline_swiglu_bf16(yb: np.ndarray) -> np.ndarray:
    """SwiGLU of the baseline's bf16 gate_up output (bf16 bits [M, N]) in fp32,
    rounded once: bf16 bits [M, N/2]."""
    yb = np.ascontiguousarray(yb, dtype=np.uint16)
    M, N = yb.shape
    out = np.empty((M, N // 2), dtype=np.uint16)
    _check(_load().oracle_baseline_swiglu_bf16(_p(yb), M, N, _p(out)))
    return out


def e2m1_table() -> np.ndarray:
    """The 16 e2m1 code values (fp64), index = 4-bit code."""
    out = np.empty(16, dtype=np.float64)
    _load().oracle_e2m1_table(_p(out))
    return out


def grouped_gemm_mxfp4_f64(x: np.ndarray, w: np.ndarray, scales: np.ndarray, sizes: np.ndarray,
                           expert_ids: np.ndarray, rows: Optional[np.ndarray] = None) -> np.ndarray:
    """MXFP4 grouped GEMM in fp64: w uint8 [E, N, K/2] (even k in the low
    nibble), scales e8m0 uint8 [E, N, K/32]; x bf16 bits [M, K]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    sizes = np.ascontiguousarray(sizes, dtype=np.int32)
    expert_ids = np.ascontiguousarray(expert_ids, dtype=np.int32)
    M, K = x.shape
    E, N, Kh = w.shape
    if Kh * 2 != K or scales.shape != (E, N, K // 32):
        raise OracleError("bad shape")
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
    nrows = M if rows is None else rows.size
    y = np.empty((nrows, N), dtype=np.float64)
    _check(_load().oracle_grouped_gemm_mxfp4_f64(
        _p(x), _p(w), _p(scales), _p(sizes), _p(expert_ids), sizes.size, M, N, K, E,
        None if rows is None else _p(rows), nrows, _p(y)))
    return y


def swiglu_interleaved_f64(y: np.ndarray, alpha: float, limit: float) -> np.ndarray:
    """gpt-oss gated activation on interleaved gate (even) / up (odd) columns."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    M, N = y.shape
    out = np.empty((M, N // 2), dtype=np.float64)
    _check(_load().oracle_swiglu_interleaved_f64(_p(y), M, N, float(alpha), float(limit), _p(out)))
    return out


def gather_rows(hidden: np.ndarray, sorted_idx: np.ndarray, top_k: int) -> np.ndarray:
    """x[i] = hidden[sorted_idx[i] // top_k] (bf16 bits)."""
    hidden = np.ascontiguousarray(hidden, dtype=np.uint16)
    sorted_idx = np.ascontiguousarray(sorted_idx, dtype=np.int32)
    T, K = hidden.shape
    x = np.empty((sorted_idx.size, K), dtype=np.uint16)
    _check(_load().oracle_gather_rows(_p(hidden), T, K, _p(sorted_idx), sorted_idx.size, top_k,
                                      _p(x)))
    return x


def grouped_gemm_bf16_absmax_f64(x, w, absmax_bf16_bits, sizes, expert_ids, rows=None):
    """The NF4 grouped GEMM with bf16 absmax (bit patterns [E, N, K/64]): the
    scale is the bf16 value itself, which widens to fp32 exactly."""
    wide = (np.asarray(absmax_bf16_bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)
    return grouped_gemm_f64(x, w, wide, sizes, expert_ids, rows=rows)


def quantized_stack(E: int, N: int, K: int, weights_fn) -> Tuple[np.ndarray, np.ndarray]:
    """Quantise a stack expert by expert: weights_fn(e) -> fp32 [N, K]."""
    packed = np.empty((E, N, K // 2), dtype=np.uint8)
    absmax = np.empty((E, N, K // 64), dtype=np.float32)
    for e in range(E):
        packed[e], absmax[e] = quantize_nf4(weights_fn(e))
    return packed, absmax


def router_topk(logits: np.ndarray, k: int, renormalize: bool):
    """-> (topk_ids int32 [T, k], weights fp64 [T, k]) for fp32 logits [T, E]."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    wts = np.empty((T, k), dtype=np.float64)
    _check(_load().oracle_router_topk(_p(logits), T, E, k, 1 if renormalize else 0, _p(ids),
                                      _p(wts)))
    return ids, wts


def moe_combine(y: np.ndarray, sorted_idx: np.ndarray, weights: np.ndarray) -> np.ndarray:
    """out fp64 [T, H] from y bf16 bits [T*k, H] (sorted order), sorted_idx [T*k], weights fp32 [T, k]."""
    y = np.ascontiguousarray(y, dtype=np.uint16)
    sorted_idx = np.ascontiguousarray(sorted_idx, dtype=np.int32)
    weights = np.ascontiguousarray(weights, dtype=np.float32)
    T, k = weights.shape
    H = y.shape[1]
    if y.shape[0] != T * k or sorted_idx.size != T * k:
        raise OracleError("bad shape")
    out = np.empty((T, H), dtype=np.float64)
    _check(_load().oracle_moe_combine(_p(y), _p(sorted_idx), _p(weights), T, k, H, _p(out)))
    return out


def grouped_dgrad_f64(dy: np.ndarray, w: np.ndarray, absmax: np.ndarray, sizes: np.ndarray,
                      expert_ids: np.ndarray) -> np.ndarray:
    """dx fp64 [M, K] from dy as bf16 bit patterns [M, N]."""
    dy = np.ascontiguousarray(dy, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    sizes = np.ascontiguousarray(sizes, dtype=np.int32)
    expert_ids = np.ascontiguousarray(expert_ids, dtype=np.int32)
    M, N = dy.shape
    E, Nw, Kh = w.shape
    if Nw != N:
        raise OracleError("bad shape")
    K = 2 * Kh
    dx = np.empty((M, K), dtype=np.float64)
    _check(_load().oracle_grouped_dgrad_f64(_p(dy), _p(w), _p(absmax), _p(sizes), _p(expert_ids),
                                            sizes.size, M, N, K, E, _p(dx)))
    return dx
