"""GPU parity for the steps either side of the grouped GEMM (package page
"grouped-nf4-gemm", "Use this when" and "Owns": the decode glue): the
router's top-k and the
top-k weighted combine, through the C ABI, against the CPU oracle.

* router top-k: expert ids bit-exact (the choice compares the fp32 logits
  themselves on both sides); weights within 2e-5 relative (fp32 exp and sum
  against fp64).
* combine: every output within one bf16 rounding of the fp64 sum plus the fp32
  accumulation error, |out - ref| <= 2^-8 |ref| + 2^-18 sum_j |w_j y_j|.
* the whole decode glue chained on the device (router -> sort -> GEMMs ->
  combine), each stage against the oracle on that stage's device input.
"""
import numpy as np
import pytest
import torch

import grouped_nf4_w4a16_b200 as gnf4
import oracle
import synth
from conftest import tolerance_violations
from gpu_cases import bf16_from_dev, bf16_to_dev, dev

pytestmark = pytest.mark.gpu


def _router(logits, k, renorm):
    ids, w = gnf4.gnf4_router_topk(dev(logits), k, renormalize=renorm)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 64, 8), (4096, 8, 2), (64, 128, 4),
                                   (16, 1000, 32), (5, 3, 3), (300, 1024, 1)])
@pytest.mark.parametrize("renorm", [False, True])
def test_router_topk_parity(T, E, k, renorm):
    rng = np.random.default_rng(T + E * 3 + k)
    logits = (rng.standard_normal((T, E)) * 2.0).astype(np.float32)
    ids, w = _router(logits, k, renorm)
    ref_ids, ref_w = oracle.router_topk(logits, k, renorm)
    assert np.array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=2e-5, atol=1e-30)


def test_router_topk_ties_and_nan():
    rng = np.random.default_rng(21)
    logits = rng.integers(0, 3, size=(500, 70)).astype(np.float32)   # many equal logits
    ids, w = _router(logits, 7, True)
    ref_ids, ref_w = oracle.router_topk(logits, 7, True)
    assert np.array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=2e-5)
    logits = rng.standard_normal((40, 30)).astype(np.float32)
    logits[:, 7] = np.nan
    logits[::3, 11] = np.nan
    for k in (4, 29, 30):   # NaN logits are chosen last (top_k <= GNF4_MAX_TOPK)
        ids, _ = _router(logits, k, True)
        ref_ids, _ = oracle.router_topk(logits, k, True)
        assert np.array_equal(ids, ref_ids)


def test_router_topk_empty():
    ids, w = gnf4.gnf4_router_topk(torch.empty((0, 16), dtype=torch.float32, device="cuda"), 2)
    assert ids.shape == (0, 2) and w.shape == (0, 2)


def _combine_abs_sum(y, sorted_idx, w):
    # sum_j |w_j y_j| per output: the scale of the fp32 accumulation error
    T, k = w.shape
    yf = synth.bf16_bits_to_f32(y).astype(np.float64)
    pos = np.full(T * k, -1, dtype=np.int64)
    ok = sorted_idx >= 0
    pos[sorted_idx[ok]] = np.nonzero(ok)[0]
    absum = np.zeros((T, y.shape[1]))
    for j in range(k):
        p = pos.reshape(T, k)[:, j]
        absum += np.where((p >= 0)[:, None], np.abs(yf[np.maximum(p, 0)]) * w[:, j:j + 1], 0.0)
    return absum


def _combine_bound(ref, absum):
    # one bf16 rounding of the sum plus the fp32 accumulation error
    return 2.0 ** -8 * np.abs(ref) + 2.0 ** -18 * absum + 1e-30


def _combine_check(T, k, H, sorted_idx, seed):
    rng = np.random.default_rng(seed)
    y = synth.activations_bf16(T * k, H, seed=seed)
    w = rng.uniform(0.0, 1.0, size=(T, k)).astype(np.float32)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_COMBINE, T * k))
    out = gnf4.gnf4_moe_combine(bf16_to_dev(y), dev(sorted_idx), dev(w), workspace=ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 0, (st, bits)
    got = bf16_from_dev(out)
    ref = oracle.moe_combine(y, sorted_idx, w)
    bad = np.abs(got - ref) > _combine_bound(ref, _combine_abs_sum(y, sorted_idx, w))
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs out of bound"


@pytest.mark.parametrize("T,E,k,H", [(1, 64, 8, 2048), (64, 128, 4, 2880), (37, 16, 2, 100),
                                     (4096, 8, 2, 512), (3, 4, 1, 8), (300, 32, 32, 64)])
def test_moe_combine_parity(T, E, k, H):
    rng = np.random.default_rng(T + E + k + H)
    ids, _ = oracle.router_topk(rng.standard_normal((T, E)).astype(np.float32), k, True)
    sorted_idx, _, _, _ = oracle.moe_align(ids, E)
    _combine_check(T, k, H, sorted_idx, seed=T + H)


def test_moe_combine_slots_left_out_and_bad_entries():
    rng = np.random.default_rng(4)
    T, k, H = 50, 4, 96
    perm = rng.permutation(T * k).astype(np.int32)
    cut = perm.copy()
    cut[::7] = -1
    _combine_check(T, k, H, cut, seed=4)
    # an entry outside [-1, T*k) sets the slot bit and is skipped
    bad = perm.copy()
    bad[3] = T * k + 5
    y = synth.activations_bf16(T * k, H, seed=5)
    w = rng.uniform(0.0, 1.0, size=(T, k)).astype(np.float32)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_MOE_COMBINE, T * k))
    gnf4.gnf4_moe_combine(bf16_to_dev(y), dev(bad), dev(w), workspace=ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 6 and bits & gnf4.DEVERR_BITS["slot"]


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_decode_glue_chain_stage_by_stage():
    # router -> moe_align -> gather -> gate_up GEMM with SwiGLU -> down GEMM ->
    # combine, all on the device through the C ABI. Each stage is checked
    # against the oracle applied to the device's own input to that stage
    # (comparing whole chains would compound one-ulp bf16 rounding flips of
    # the intermediates beyond the per-stage tolerances).
    rng = np.random.default_rng(77)
    T, E, k, Hd, F = 24, 16, 4, 256, 192   # hidden 256, expert width 192 (gate_up N = 384)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    hidden = synth.activations_bf16(T, Hd, seed=77)
    p_gu = rng.integers(0, 256, size=(E, 2 * F, Hd // 2), dtype=np.uint8)
    a_gu = rng.uniform(0.02, 0.06, size=(E, 2 * F, Hd // 64)).astype(np.float32)
    p_dn = rng.integers(0, 256, size=(E, Hd, F // 2), dtype=np.uint8)
    a_dn = rng.uniform(0.02, 0.06, size=(E, Hd, F // 64)).astype(np.float32)

    ids_d, w_d = gnf4.gnf4_router_topk(dev(logits), k, renormalize=True)
    sidx_d, sizes_d, eids_d, _ = gnf4.gnf4_moe_align(ids_d, E)
    x_d = bf16_to_dev(hidden)[(sidx_d // k).long()]
    h_d = gnf4.gnf4_grouped_gemm(x_d, dev(p_gu), dev(a_gu), sizes_d, eids_d,
                                 epilogue=gnf4.GNF4_EPI_SWIGLU)
    y_d = gnf4.gnf4_grouped_gemm(h_d, dev(p_dn), dev(a_dn), sizes_d, eids_d)
    out_d = gnf4.gnf4_moe_combine(y_d, sidx_d, w_d)
    torch.cuda.synchronize()

    ids, w = oracle.router_topk(logits, k, True)
    assert np.array_equal(ids_d.cpu().numpy(), ids)
    np.testing.assert_allclose(w_d.cpu().numpy(), w, rtol=2e-5)
    sidx, sizes, eids, _ = oracle.moe_align(ids, E)
    assert np.array_equal(sidx_d.cpu().numpy(), sidx)
    assert np.array_equal(_bits(x_d), hidden[sidx // k])
    h_ref = oracle.swiglu_f64(oracle.grouped_gemm_f64(hidden[sidx // k], p_gu, a_gu, sizes, eids))
    assert not tolerance_violations(bf16_from_dev(h_d), h_ref).any()
    h_bits = _bits(h_d)
    y_ref = oracle.grouped_gemm_f64(h_bits, p_dn, a_dn, sizes, eids)
    assert not tolerance_violations(bf16_from_dev(y_d), y_ref).any()
    y_bits, wd = _bits(y_d), w_d.cpu().numpy()
    out_ref = oracle.moe_combine(y_bits, sidx, wd)
    got = bf16_from_dev(out_d)
    assert (np.abs(got - out_ref) <= _combine_bound(out_ref, _combine_abs_sum(y_bits, sidx, wd))).all()
