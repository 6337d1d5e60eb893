"""Pins for the CPU oracle (no GPU). Each test checks the oracle against
something other than itself: a closed form, a library routine, brute force
written independently here, an invariance, or a hand-derived value.

Passages (page "grouped-nf4-gemm -- single-launch W4A16 GEMM over fused NF4 MoE
expert stacks", PyPI README of grouped_nf4_gemm 0.1.0):
  opening section -- the op: [E,N,K/2] uint8 + blockwise fp32 absmax,
    (sizes, expert_ids) after the token->expert sort, LUT decode, fp32
    accumulation, bf16 epilogue, and the dequant-then-matmul baseline;
  "The claim" -- fused error below the materialise-to-bf16 baseline;
  "Cross-vendor projections" -- NF4 vs bf16 = 3.56x bytes, absmax-inclusive.
"""
import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import oracle
import synth
from conftest import frob_rel_err

NF4 = None


def table():
    global NF4
    if NF4 is None:
        NF4 = oracle.nf4_table().astype(np.float64)
    return NF4


# ------------------------------------------------------------------ table
def test_nf4_table_matches_normal_quantile_closed_form():
    # NF4 construction: 8 positive and 7 negative normal quantiles at evenly
    # spaced probabilities from delta down to 1/2, plus an exact zero, divided
    # by the largest magnitude.
    delta = 0.9677083
    pos = scipy.stats.norm.ppf(np.linspace(delta, 0.5, 9)[:-1])
    neg = -scipy.stats.norm.ppf(np.linspace(delta, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = v / np.max(np.abs(v))
    assert np.max(np.abs(v - table())) < 2e-7


def test_nf4_table_invariants():
    t = table()
    assert t.shape == (16,)
    assert t[7] == 0.0 and t[0] == -1.0 and t[15] == 1.0
    assert np.all(np.diff(t) > 0)
    # The values are the fp32 roundings of the table (exact as float32).
    assert np.array_equal(t.astype(np.float32).astype(np.float64), t)


# -------------------------------------------------------------- quantiser
def _independent_quantise(w):
    """Brute-force nearest-code quantiser written independently (NumPy)."""
    t = table().astype(np.float32)
    R, K = w.shape
    wb = w.reshape(R, K // 64, 64)
    amax = np.max(np.abs(wb), axis=2)
    with np.errstate(invalid="ignore", divide="ignore"):
        v = (wb / amax[:, :, None]).astype(np.float32)
    d = np.abs(t[None, None, None, :] - v[..., None])
    codes = np.argmin(d, axis=-1)          # argmin keeps the first (lower) index on ties
    codes[amax == 0] = 7
    codes = codes.reshape(R, K)
    packed = ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)
    return packed, amax.astype(np.float32)


def test_quantiser_matches_brute_force():
    rng = np.random.default_rng(1)
    w = (rng.standard_normal((37, 256)) * 0.02).astype(np.float32)
    w[3, 64:128] = 0.0                     # an all-zero block
    p, a = oracle.quantize_nf4(w)
    p2, a2 = _independent_quantise(w)
    assert np.array_equal(a, a2)
    assert np.array_equal(p, p2)
    assert np.all(p[3, 32:64] == 0x77) and a[3, 1] == 0.0


def test_quantiser_roundtrip_idempotent_and_error_bound():
    rng = np.random.default_rng(2)
    R, K = 64, 512
    codes = rng.integers(0, 16, size=(R, K))
    codes[:, ::64] = rng.choice([0, 15], size=(R, K // 64))   # each block reaches +-absmax
    packed = ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)
    absmax = rng.uniform(1e-3, 10.0, size=(R, K // 64)).astype(np.float32)
    deq = oracle.dequant_f32(packed, absmax)
    p2, a2 = oracle.quantize_nf4(deq)
    assert np.array_equal(a2, absmax)
    assert np.array_equal(p2, packed)
    # Reconstruction error of arbitrary weights is at most half the largest gap.
    w = (rng.standard_normal((R, K)) * 0.02).astype(np.float32)
    p, a = oracle.quantize_nf4(w)
    rec = oracle.dequant_f32(p, a).astype(np.float64)
    maxgap = np.max(np.diff(table()))
    bound = np.repeat(a.astype(np.float64), 64, axis=1) * maxgap / 2 * (1 + 1e-6)
    assert np.all(np.abs(rec - w) <= bound)
    # The largest-magnitude element of each block is reproduced exactly.
    wb = w.reshape(R, K // 64, 64)
    idx = np.argmax(np.abs(wb), axis=2)
    got = np.take_along_axis(rec.reshape(R, K // 64, 64), idx[..., None], 2)[..., 0]
    want = np.take_along_axis(wb, idx[..., None], 2)[..., 0]
    assert np.array_equal(got, want.astype(np.float64))


def test_quantiser_ties_go_to_lower_index():
    t = table().astype(np.float32)
    # Find a table midpoint exactly representable in fp32 relative to absmax 1.
    found = False
    for i in range(15):
        mid64 = (np.float64(t[i]) + np.float64(t[i + 1])) / 2
        mid = np.float32(mid64)
        if np.float64(mid) == mid64:
            w = np.zeros((1, 64), dtype=np.float32)
            w[0, 0] = 1.0
            w[0, 2] = mid
            p, _ = oracle.quantize_nf4(w)
            assert p[0, 1] >> 4 == i
            found = True
    assert found


# ---------------------------------------------------------------- dequant
def test_dequant_f32_is_single_rounded_product():
    rng = np.random.default_rng(3)
    R, K = 16, 256
    packed = rng.integers(0, 256, size=(R, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0, 1, size=(R, K // 64)).astype(np.float32)
    # Adversarial scales: zero, smallest subnormal, tiny, near fp32 max.
    absmax[0, :4] = [0.0, np.float32(1e-45), np.float32(1e-30), np.float32(3e38)]
    out = oracle.dequant_f32(packed, absmax)
    codes = np.empty((R, K), dtype=np.int64)
    codes[:, 0::2] = packed >> 4
    codes[:, 1::2] = packed & 15
    exact = table()[codes] * np.repeat(absmax.astype(np.float64), 64, axis=1)
    assert np.array_equal(out, exact.astype(np.float32))


def test_dequant_bf16_is_round_nearest_even_of_f32():
    rng = np.random.default_rng(4)
    R, K = 16, 256
    packed = rng.integers(0, 256, size=(R, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0, 3, size=(R, K // 64)).astype(np.float32)
    absmax[0, :4] = [0.0, np.float32(1e-45), np.float32(1e-30), np.float32(3e38)]
    f32 = oracle.dequant_f32(packed, absmax)
    b = oracle.dequant_bf16(packed, absmax)
    # Library routine: torch's fp32 -> bf16 conversion rounds to nearest even.
    want = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, want)
    # And by the definition: b is the nearest bf16 to f32, ties to even mantissa.
    v = f32.astype(np.float64).ravel()
    got = synth.bf16_bits_to_f32(b).astype(np.float64).ravel()
    lo = synth.bf16_bits_to_f32((f32.view(np.uint32) >> 16).astype(np.uint16)).astype(np.float64).ravel()
    step = np.abs(synth.bf16_bits_to_f32(((f32.view(np.uint32) >> 16) + 1).astype(np.uint16))
                  .astype(np.float64).ravel() - lo)
    assert np.all(np.abs(got - v) <= step / 2 + 0.0)


# ------------------------------------------------------------- moe_align
@pytest.mark.parametrize("T,k,E", [(8, 2, 4), (1, 8, 64), (16, 8, 128), (64, 4, 128), (333, 3, 7), (0, 2, 5)])
def test_moe_align_is_stable_counting_sort(T, k, E):
    rng = np.random.default_rng(T * 1000 + E)
    ids = rng.integers(0, E, size=(T, k)).astype(np.int32)
    sorted_idx, sizes, expert_ids, ng = oracle.moe_align(ids, E)
    flat = ids.ravel()
    ref = np.argsort(flat, kind="stable")
    assert np.array_equal(sorted_idx, ref.astype(np.int32))
    present = np.unique(flat)
    assert ng == present.size
    assert np.array_equal(expert_ids[:ng], present)
    assert np.array_equal(sizes[:ng], np.bincount(flat, minlength=E)[present])
    assert np.all(sizes[ng:] == 0) and np.all(expert_ids[ng:] == -1)
    assert sizes.sum() == T * k


def test_moe_align_duplicates_and_bad_ids():
    ids = np.array([[2, 2], [0, 2]], dtype=np.int32)   # duplicate expert in one token
    s, sz, ex, ng = oracle.moe_align(ids, 3)
    assert list(s) == [2, 0, 1, 3] and list(sz) == [1, 3, 0] and list(ex) == [0, 2, -1] and ng == 2
    with pytest.raises(oracle.OracleError):
        oracle.moe_align(np.array([[0, 3]], dtype=np.int32), 3)
    with pytest.raises(oracle.OracleError):
        oracle.moe_align(np.array([[-1, 0]], dtype=np.int32), 3)


# ------------------------------------------------------------ grouped GEMM
def _random_problem(rng, E, N, K, sizes, expert_ids):
    M = int(np.sum(sizes))
    x = synth.workloads._f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    return x, packed, absmax, np.array(sizes, np.int32), np.array(expert_ids, np.int32)


def _numpy_reference(x, packed, absmax, sizes, expert_ids):
    """Independent route: dequantise each expert to fp64 with NumPy, then '@'."""
    t = table()
    E, N, Kh = packed.shape
    K = 2 * Kh
    codes = np.empty((E, N, K), dtype=np.int64)
    codes[:, :, 0::2] = packed >> 4
    codes[:, :, 1::2] = packed & 15
    W = t[codes] * np.repeat(absmax.astype(np.float64), 64, axis=2)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y = np.zeros((xf.shape[0], N))
    off = 0
    for s, e in zip(sizes, expert_ids):
        if s:
            y[off:off + s] = xf[off:off + s] @ W[e].T
        off += s
    return y


@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (1, 8, 64, [3], [0]),
    (3, 8, 128, [2, 0, 4], [2, 1, 0]),
    (3, 6, 64, [1, 1, 1, 3], [0, 1, 2, 1]),
    (2, 5, 192, [0, 6], [-1, 1]),
])
def test_grouped_gemm_matches_numpy_brute_force(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 100 + N + K)
    x, w, a, s, ex = _random_problem(rng, E, N, K, sizes, experts)
    y = oracle.grouped_gemm_f64(x, w, a, s, ex)
    ref = _numpy_reference(x, w, a, s, ex)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.max(np.abs(ref)))


def test_grouped_gemm_hand_worked_values():
    # One expert, one output row, K = 64. Byte 0xF0 puts code 15 (+1.0) at k=0
    # and code 0 (-1.0) at k=1 (high nibble = even k).
    w = np.full((1, 2, 32), 0x77, dtype=np.uint8)        # all codes 7 (0.0)
    w[0, 0, 0] = 0xF0
    w[0, 1, :] = 0xFF                                      # row 1: every code +1.0
    a = np.array([[[0.5], [0.25]]], dtype=np.float32)
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, 0] = 3.0
    x[1, 1] = 2.0
    xb = synth.workloads._f32_to_bf16_bits(x)
    y = oracle.grouped_gemm_f64(xb, w, a, np.array([2], np.int32), np.array([0], np.int32))
    # row 0: 3*(+1)*0.5 = 1.5 ; 3*0.25 = 0.75.  row 1: 2*(-1)*0.5 = -1.0 ; 2*0.25 = 0.5
    assert np.array_equal(y, np.array([[1.5, 0.75], [-1.0, 0.5]]))
    # All-ones x against the all-ones row: 64 * 0.25.
    y2 = oracle.grouped_gemm_f64(synth.workloads._f32_to_bf16_bits(np.ones((1, 64), np.float32)),
                                 w, a, np.array([1], np.int32), np.array([0], np.int32))
    assert y2[0, 1] == 16.0 and y2[0, 0] == 0.5 - 0.5


def test_grouped_gemm_one_hot_reads_codes():
    rng = np.random.default_rng(7)
    E, N, K = 2, 4, 128
    w = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    a = np.ones((E, N, K // 64), dtype=np.float32)
    for k0 in (0, 1, 63, 64, 127):
        x = np.zeros((1, K), np.float32)
        x[0, k0] = 1.0
        for e in range(E):
            y = oracle.grouped_gemm_f64(synth.workloads._f32_to_bf16_bits(x), w, a,
                                        np.array([1], np.int32), np.array([e], np.int32))
            byte = w[e, :, k0 // 2]
            code = (byte >> 4) if k0 % 2 == 0 else (byte & 15)
            assert np.array_equal(y[0], table()[code])


def test_grouped_gemm_invariances():
    rng = np.random.default_rng(8)
    E, N, K = 3, 7, 128
    x, w, a, s, ex = _random_problem(rng, E, N, K, [2, 3, 1], [1, 0, 2])
    y = oracle.grouped_gemm_f64(x, w, a, s, ex)
    # zero-size groups anywhere change nothing
    y0 = oracle.grouped_gemm_f64(x, w, a, np.array([0, 2, 0, 3, 1, 0], np.int32),
                                 np.array([2, 1, 0, 0, 2, 1], np.int32))
    assert np.array_equal(y, y0)
    # permuting group order with the matching row blocks permutes the output
    perm_rows = np.r_[2:5, 5:6, 0:2]
    yp = oracle.grouped_gemm_f64(x[perm_rows], w, a, np.array([3, 1, 2], np.int32),
                                 np.array([0, 2, 1], np.int32))
    assert np.array_equal(yp, y[perm_rows])
    # splitting a group into two with the same expert changes nothing
    ys = oracle.grouped_gemm_f64(x, w, a, np.array([2, 1, 2, 1], np.int32),
                                 np.array([1, 0, 0, 2], np.int32))
    assert np.array_equal(ys, y)
    # doubling one expert's absmax doubles exactly its rows
    a2 = a.copy()
    a2[0] *= 2
    yd = oracle.grouped_gemm_f64(x, w, a2, s, ex)
    assert np.array_equal(yd[2:5], 2 * y[2:5])
    assert np.array_equal(yd[[0, 1, 5]], y[[0, 1, 5]])
    # row subset equals the same rows of the full output
    rows = np.array([5, 0, 3])
    assert np.array_equal(oracle.grouped_gemm_f64(x, w, a, s, ex, rows=rows), y[rows])


def test_grouped_gemm_rejects_bad_metadata():
    rng = np.random.default_rng(9)
    x, w, a, s, ex = _random_problem(rng, 2, 4, 64, [2, 1], [0, 1])
    with pytest.raises(oracle.OracleError):
        oracle.grouped_gemm_f64(x, w, a, np.array([2, 2], np.int32), ex)      # sum != M
    with pytest.raises(oracle.OracleError):
        oracle.grouped_gemm_f64(x, w, a, s, np.array([0, 2], np.int32))       # expert >= E
    # an out-of-range id on an empty group is ignored
    y = oracle.grouped_gemm_f64(x, w, a, np.array([2, 0, 1], np.int32), np.array([0, 99, 1], np.int32))
    assert np.array_equal(y, oracle.grouped_gemm_f64(x, w, a, s, ex))


# ---------------------------------------------------------------- SwiGLU
def test_swiglu_closed_form():
    rng = np.random.default_rng(10)
    y = rng.standard_normal((5, 12)) * 4
    y[0, 0] = 0.0
    out = oracle.swiglu_f64(y)
    g, u = y[:, :6], y[:, 6:]
    assert np.allclose(out, g * scipy.special.expit(g) * u, rtol=1e-14, atol=0)
    assert out[0, 0] == 0.0


# -------------------------------------------------------------- baseline
def test_baseline_emulation_against_fp64_of_bf16_weights():
    rng = np.random.default_rng(11)
    E, N, K = 2, 16, 256
    x, w, a, s, ex = _random_problem(rng, E, N, K, [3, 4], [1, 0])
    yb = synth.bf16_bits_to_f32(oracle.baseline_bf16(x, w, a, s, ex)).astype(np.float64)
    # Same bf16 weights, exact fp64 accumulation, one bf16 rounding: may differ
    # from the fp32-accumulated result by at most one bf16 ulp.
    wb = synth.bf16_bits_to_f32(oracle.dequant_bf16(w, a)).astype(np.float64)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.concatenate([xf[:3] @ wb[1].T, xf[3:] @ wb[0].T])
    ref_b = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)
    ulp = np.abs(ref_b) * 2.0 ** -7
    assert np.all(np.abs(yb - ref_b) <= ulp + 1e-30)


def test_baseline_swiglu_against_expit_on_its_own_bf16_values():
    # The baseline's SwiGLU works on the bf16 gate and up values its GEMM
    # materialised. Pin: the closed form g * expit(g) * u in fp64 on those same
    # values, rounded once to bf16, equals the oracle's fp32 computation except
    # where fp32 rounding crosses a bf16 rounding boundary (then one ulp).
    rng = np.random.default_rng(12)
    M, N = 64, 96
    yb = oracle.f32_to_bf16((rng.standard_normal((M, N)) * 3).astype(np.float32))
    yb[0, 0] = 0                       # g = 0 -> 0
    yb[1, 0] = oracle.f32_to_bf16(np.array([-80.0], np.float32))[0]   # silu(-80) ~ -1.4e-33
    yb[2, 0] = oracle.f32_to_bf16(np.array([40.0], np.float32))[0]     # silu(40) = 40 (to fp32)
    out = synth.bf16_bits_to_f32(oracle.baseline_swiglu_bf16(yb)).astype(np.float64)
    v = synth.bf16_bits_to_f32(yb).astype(np.float64)
    g, u = v[:, :N // 2], v[:, N // 2:]
    ref = g * scipy.special.expit(g) * u
    ref_b = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16).float().numpy()
    ref_b = ref_b.astype(np.float64)
    ulp = np.abs(ref_b) * 2.0 ** -7
    assert np.all(np.abs(out - ref_b) <= ulp + 1e-45)
    assert np.mean(out == ref_b) > 0.99
    assert out[0, 0] == 0.0
    assert out[2, 0] == ref_b[2, 0]
    # gate and up halves are not swapped: scaling the up half scales the output
    yb2 = yb.copy()
    yb2[:, N // 2:] = oracle.f32_to_bf16((v[:, N // 2:] * 2).astype(np.float32))
    out2 = synth.bf16_bits_to_f32(oracle.baseline_swiglu_bf16(yb2)).astype(np.float64)
    assert np.array_equal(out2, 2 * out)


def test_fidelity_ordering_is_achievable():
    # The fp64 result rounded once to bf16 is closer to the reference than the
    # materialise-to-bf16 baseline, as the README's "The claim" states.
    w_ = synth.WORKLOADS["tiny"]
    x = synth.activations_bf16(w_.M, 256, seed=0)
    packed, absmax = oracle.quantized_stack(w_.E, 128, 256,
                                            lambda e: synth.expert_weights_f32(w_.E, 128, 256, e))
    topk = synth.routing(w_, 0)
    _, sizes, experts, _ = oracle.moe_align(topk, w_.E)
    y = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    yb = synth.bf16_bits_to_f32(oracle.baseline_bf16(x, packed, absmax, sizes, experts))
    y_once = synth.bf16_bits_to_f32(oracle.f32_to_bf16(y.astype(np.float32)))
    assert frob_rel_err(y_once, y) < frob_rel_err(yb, y)


# ------------------------------------------------------------ byte identity
def test_nf4_bytes_vs_bf16_ratio():
    # The README's projections section: NF4 vs bf16 is a 3.56x byte reduction
    # including the fp32 absmax (0.5 + 4/64 bytes per weight vs 2).
    E, N, K = 3, 64, 256
    packed = np.zeros((E, N, K // 2), np.uint8)
    absmax = np.zeros((E, N, K // 64), np.float32)
    nbytes = packed.nbytes + absmax.nbytes
    assert nbytes == 0.5625 * E * N * K
    assert round(2 * E * N * K / nbytes, 2) == 3.56


# ---------------------------------------------------------------------------
# Router top-k and weighted combine (package page "grouped-nf4-gemm", "Use
# this when" and "Owns":
# the decode glue around the grouped GEMM)

@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 64, 8), (200, 128, 4), (16, 1000, 32), (5, 3, 3)])
@pytest.mark.parametrize("renorm", [False, True])
def test_router_topk_matches_stable_argsort_and_scipy_softmax(T, E, k, renorm):
    rng = np.random.default_rng(T * 7 + E + k)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.router_topk(logits, k, renorm)
    # ids: a library sort (stable: equal logits keep the lower expert id first)
    assert np.array_equal(ids, np.argsort(-logits, axis=1, kind="stable")[:, :k])
    lg = logits.astype(np.float64)
    if renorm:
        ref = scipy.special.softmax(np.take_along_axis(lg, ids, axis=1), axis=1)
    else:
        ref = np.take_along_axis(scipy.special.softmax(lg, axis=1), ids, axis=1)
    np.testing.assert_allclose(w, ref, rtol=1e-12, atol=0)
    if renorm:
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-12)
    else:
        assert (w.sum(axis=1) <= 1.0 + 1e-12).all()
    assert (np.diff(w, axis=1) <= 0).all()   # descending logits -> descending weights


def test_router_topk_ties_nan_and_shift():
    rng = np.random.default_rng(5)
    # many equal logits: the lower expert id goes first
    logits = rng.integers(0, 3, size=(64, 40)).astype(np.float32)
    ids, w = oracle.router_topk(logits, 6, True)
    assert np.array_equal(ids, np.argsort(-logits, axis=1, kind="stable")[:, :6])
    # all equal: the first top_k experts, equal weights
    ids, w = oracle.router_topk(np.zeros((3, 10), np.float32), 4, False)
    assert (ids == np.arange(4)).all() and np.allclose(w, 0.1)
    # a NaN logit ranks as -inf: it is chosen only after every number
    logits = rng.standard_normal((8, 12)).astype(np.float32)
    logits[:, 3] = np.nan
    ids, _ = oracle.router_topk(logits, 11, True)
    assert not (ids == 3).any()
    ids, _ = oracle.router_topk(logits, 12, True)
    assert (ids[:, -1] == 3).all()
    # shifting every logit of a token changes neither the choice nor the weights
    logits = rng.standard_normal((16, 32)).astype(np.float32)
    a_ids, a_w = oracle.router_topk(logits, 4, False)
    b_ids, b_w = oracle.router_topk(logits + np.float32(8.0), 4, False)
    assert np.array_equal(a_ids, b_ids)
    np.testing.assert_allclose(a_w, b_w, rtol=1e-6)   # the shift itself rounds in fp32


def _combine_numpy(y_bits, sorted_idx, w):
    # independent of the C oracle: inverse permutation by fancy indexing,
    # weighted sum by broadcasting
    T, k = w.shape
    yf = synth.bf16_bits_to_f32(y_bits).astype(np.float64)
    inv = np.full(T * k, -1, dtype=np.int64)
    valid = sorted_idx >= 0
    inv[sorted_idx[valid]] = np.nonzero(valid)[0]
    rows = np.where(inv >= 0, inv, 0).reshape(T, k)
    contrib = yf[rows] * w.astype(np.float64)[:, :, None] * (inv >= 0).reshape(T, k)[:, :, None]
    return contrib.sum(axis=1)


@pytest.mark.parametrize("T,E,k,H", [(1, 4, 1, 16), (37, 16, 2, 64), (64, 128, 8, 40)])
def test_moe_combine_matches_numpy_through_the_real_sort(T, E, k, H):
    rng = np.random.default_rng(T + E + k + H)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.router_topk(logits, k, True)
    sorted_idx, _, _, _ = oracle.moe_align(ids, E)
    y = synth.activations_bf16(T * k, H, seed=T + H)
    out = oracle.moe_combine(y, sorted_idx, w.astype(np.float32))
    np.testing.assert_allclose(out, _combine_numpy(y, sorted_idx, w.astype(np.float32)),
                               rtol=1e-12, atol=1e-300)


def test_moe_combine_special_cases():
    rng = np.random.default_rng(9)
    T, k, H = 12, 3, 24
    perm = rng.permutation(T * k).astype(np.int32)
    y = synth.activations_bf16(T * k, H, seed=9)
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    # one-hot weights read back exactly the row that holds slot t*k + j
    for j in range(k):
        w = np.zeros((T, k), np.float32)
        w[:, j] = 1.0
        out = oracle.moe_combine(y, perm, w)
        pos = np.argsort(perm)
        assert np.array_equal(out, yf[pos[np.arange(T) * k + j]])
    # slots left out (-1) contribute nothing
    w = rng.uniform(0.1, 1.0, size=(T, k)).astype(np.float32)
    cut = perm.copy()
    cut[::5] = -1
    full = oracle.moe_combine(y, perm, w)
    part = oracle.moe_combine(y, cut, w)
    missing = perm[::5]
    w2 = w.copy().reshape(-1)
    w2[missing] = 0.0
    assert np.allclose(part, oracle.moe_combine(y, perm, w2.reshape(T, k)), rtol=0, atol=0)
    assert not np.allclose(part, full)
    # linear in the weights
    assert np.array_equal(oracle.moe_combine(y, perm, 2 * w), 2 * full)
    # an entry outside [-1, T*k) is refused
    bad = perm.copy()
    bad[0] = T * k
    with pytest.raises(oracle.OracleError):
        oracle.moe_combine(y, bad, w)


# ---------------------------------------------------------------------------
# Grouped dgrad (package page "grouped-nf4-gemm", header block, "Owns": the
# grouped packed GEMM and its dgrad)

@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (3, 48, 128, [3, 0, 5], [2, 0, 1]),
    (2, 96, 320, [4, 4, 1], [1, 1, 0]),      # the same expert in two groups
    (1, 8, 64, [6], [0]),
])
def test_grouped_dgrad_is_the_adjoint_of_the_forward(E, N, K, sizes, experts):
    # <dy, GEMM(x)> == <dgrad(dy), x> for any x and dy, group by group: pins
    # the dgrad to the (separately pinned) forward oracle
    rng = np.random.default_rng(E + N + K)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    M = int(sum(sizes))
    x = synth.activations_bf16(M, K, seed=N)
    dy = synth.activations_bf16(M, N, seed=K)
    y = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    dx = oracle.grouped_dgrad_f64(dy, packed, absmax, sizes, experts)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
    # per row (each row has its own expert): sum_n dy y == sum_k dx x
    lhs, rhs = (dyf * y).sum(axis=1), (dx * xf).sum(axis=1)
    scale = (np.abs(dyf)[:, :, None] * 0.1).sum(axis=(1, 2)) * np.abs(xf).sum(axis=1)
    assert (np.abs(lhs - rhs) <= 1e-12 * scale + 1e-300).all()


def test_grouped_dgrad_matches_numpy_matmul():
    rng = np.random.default_rng(3)
    E, N, K = 4, 40, 192
    sizes, experts = [2, 0, 7, 3], [3, 1, 0, 3]
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    M = int(sum(sizes))
    dy = synth.activations_bf16(M, N, seed=3)
    dx = oracle.grouped_dgrad_f64(dy, packed, absmax, sizes, experts)
    W = oracle.dequant_f32(packed.reshape(E * N, K // 2),
                           absmax.reshape(E * N, K // 64)).astype(np.float64).reshape(E, N, K)
    dyf = synth.bf16_bits_to_f32(dy).astype(np.float64)
    ref = np.zeros((M, K))
    r = 0
    for s, e in zip(sizes, experts):
        ref[r:r + s] = dyf[r:r + s] @ W[e]
        r += s
    # the oracle multiplies in fp64, the library routine used here on the
    # fp32-rounded dequantised weights: within fp32 rounding of each weight
    np.testing.assert_allclose(dx, ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_grouped_dgrad_rejects_bad_metadata():
    packed = np.zeros((2, 8, 32), np.uint8)
    absmax = np.ones((2, 8, 1), np.float32)
    dy = synth.activations_bf16(4, 8, seed=0)
    with pytest.raises(oracle.OracleError):
        oracle.grouped_dgrad_f64(dy, packed, absmax, [2, 1], [0, 1])    # sizes sum 3 != 4
    with pytest.raises(oracle.OracleError):
        oracle.grouped_dgrad_f64(dy, packed, absmax, [2, 2], [0, 2])    # expert 2 of 2


# ------------------------------------------------------------------ MXFP4
# The values of the FP4 (E2M1) element type as the OCP Microscaling Formats
# (MX) v1.0 specification tabulates them: 1 sign bit, 2 exponent bits (bias
# 1), 1 mantissa bit; exponent field 0 is subnormal.
OCP_E2M1_POSITIVE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _mx_dequant_numpy(w, scales):
    """Independent NumPy decode: low nibble = even k, value from the spec's
    table above times 2^(s - 127)."""
    table = np.array(OCP_E2M1_POSITIVE + [-v for v in OCP_E2M1_POSITIVE])
    lo, hi = w & 0x0F, w >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(w.shape[:-1] + (w.shape[-1] * 2,))
    vals = table[codes]
    sc = np.ldexp(1.0, scales.astype(np.int64) - 127)
    sc = np.where(scales == 255, np.nan, sc)
    return vals * np.repeat(sc, 32, axis=-1)


def test_e2m1_table_is_the_ocp_table():
    t = oracle.e2m1_table()
    assert t[:8].tolist() == OCP_E2M1_POSITIVE
    assert t[8:].tolist() == [-v for v in OCP_E2M1_POSITIVE]
    assert np.signbit(t[8])          # code 8 is -0


@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (2, 5, 64, [3, 2], [1, 0]), (3, 7, 128, [0, 4, 1], [2, 1, 0]), (1, 3, 96, [2], [0])])
def test_mxfp4_gemm_matches_numpy_brute_force(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 100 + K)
    M = sum(sizes)
    x = synth.activations_bf16(M, K, seed=K)
    w = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    sc = rng.integers(110, 140, size=(E, N, K // 32)).astype(np.uint8)
    y = oracle.grouped_gemm_mxfp4_f64(x, w, sc, np.array(sizes, np.int32), np.array(experts, np.int32))
    wd = _mx_dequant_numpy(w, sc)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.zeros((M, N))
    off = 0
    for s_, e in zip(sizes, experts):
        ref[off:off + s_] = xf[off:off + s_] @ wd[e].T
        off += s_
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-300)


def test_mxfp4_gemm_nibble_order_and_one_hot_read_out():
    # byte 0x21: k = 0 takes the low nibble (code 1 = 0.5), k = 1 the high
    # nibble (code 2 = 1.0); scale byte 127 = 2^0, 128 = 2^1
    w = np.zeros((1, 2, 16), np.uint8)
    w[0, 0, 0] = 0x21
    w[0, 1, 0] = 0xF7                      # k = 0: code 7 = 6.0, k = 1: code 15 = -6.0
    sc = np.array([[[127], [128]]], np.uint8)
    x = np.zeros((2, 32), np.float32)
    x[0, 0] = 1.0
    x[1, 1] = 1.0
    xb = oracle.f32_to_bf16(x)
    y = oracle.grouped_gemm_mxfp4_f64(xb, w, sc, np.array([2], np.int32), np.array([0], np.int32))
    assert y.tolist() == [[0.5, 12.0], [1.0, -12.0]]


def test_mxfp4_e8m0_extremes():
    w = np.full((1, 1, 16), 0x22, np.uint8)          # every element 1.0
    x = oracle.f32_to_bf16(np.ones((1, 32), np.float32))
    for s_, want in [(0, 32.0 * 2.0 ** -127), (254, 32.0 * 2.0 ** 127)]:
        y = oracle.grouped_gemm_mxfp4_f64(x, w, np.array([[[s_]]], np.uint8),
                                          np.array([1], np.int32), np.array([0], np.int32))
        assert y[0, 0] == want
    y = oracle.grouped_gemm_mxfp4_f64(x, w, np.array([[[255]]], np.uint8),
                                      np.array([1], np.int32), np.array([0], np.int32))
    assert np.isnan(y[0, 0])


# -------------------------------------------------------- bf16 absmax
def test_bf16_absmax_equals_fp32_absmax_of_the_same_values():
    rng = np.random.default_rng(21)
    E, N, K = 2, 6, 128
    x, w, a, s, ex = _random_problem(rng, E, N, K, [3, 2], [1, 0])
    ab = oracle.f32_to_bf16(a)
    a_wide = synth.bf16_bits_to_f32(ab)
    y_b = oracle.grouped_gemm_bf16_absmax_f64(x, w, ab, s, ex)
    assert np.array_equal(y_b, oracle.grouped_gemm_f64(x, w, a_wide, s, ex))
    # and against NumPy: the scale of block b is the bf16 value (exact)
    table = oracle.nf4_table().astype(np.float64)
    codes = np.stack([w >> 4, w & 0x0F], axis=-1).reshape(E, N, K)
    wd = table[codes] * np.repeat(a_wide.astype(np.float64), 64, axis=-1)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.concatenate([xf[:3] @ wd[1].T, xf[3:] @ wd[0].T])
    assert np.allclose(y_b, ref, rtol=1e-12, atol=0)


# ------------------------------------------- interleaved, clamped SwiGLU
def test_swiglu_interleaved_closed_form_and_clamps():
    rng = np.random.default_rng(22)
    y = rng.standard_normal((4, 10)) * 6
    y[0, 0], y[0, 1] = 20.0, 3.0        # gate above the limit
    y[1, 2], y[1, 3] = 1.0, -30.0       # up below -limit
    y[2, 4], y[2, 5] = -40.0, 2.0       # very negative gate: not clamped from below
    alpha, limit = 1.702, 7.0
    out = oracle.swiglu_interleaved_f64(y, alpha, limit)
    g = np.minimum(y[:, 0::2], limit)
    u = np.clip(y[:, 1::2], -limit, limit)
    ref = g * scipy.special.expit(alpha * g) * (u + 1)
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-300)
    assert out[0, 0] == pytest.approx(7.0 * scipy.special.expit(alpha * 7.0) * 4.0, rel=1e-14)
    assert out[1, 1] == pytest.approx(1.0 * scipy.special.expit(alpha) * (-6.0), rel=1e-14)
    assert abs(out[2, 2]) < 1e-25


# ---------------------------------------------------------------- gather
def test_gather_rows_is_indexing_by_token():
    rng = np.random.default_rng(23)
    T, k, K = 5, 3, 64
    hidden = rng.integers(0, 65535, size=(T, K)).astype(np.uint16)
    topk = rng.integers(0, 4, size=(T, k)).astype(np.int32)
    sorted_idx, sizes, experts, ng = oracle.moe_align(topk, 4)
    x = oracle.gather_rows(hidden, sorted_idx, k)
    assert np.array_equal(x, hidden[sorted_idx // k])
    with pytest.raises(oracle.OracleError):
        oracle.gather_rows(hidden, np.array([T * k], np.int32), k)
