"""GPU parity: libgnf4 (through its C ABI) against the CPU oracle.

* moe_align and dequant_debug: bit-exact.
* grouped GEMM: every compared element within
  |y - y_ref| <= 1e-2*|y_ref| + 1e-3*rms(y_ref) of the fp64 oracle (rms over the
  whole GEMM output), and relative Frobenius error no larger than the
  dequantise-to-bf16-then-matmul baseline's on the same rows.
"""
import numpy as np
import pytest
import torch

import grouped_nf4_w4a16_b200 as gnf4
import oracle
import synth
from conftest import frob_rel_err, tolerance_violations
from gpu_cases import (bf16_from_dev, bf16_to_dev, boundaries, dev, groups_from_routing,
                       quantised_stack, sample_rows, tile_strata)

pytestmark = pytest.mark.gpu

DECODE_WORKLOADS = ["tiny", "olmoe", "qwen3_30b_a3b", "gpt_oss_120b"]


# ------------------------------------------------------------------ dequant
@pytest.mark.parametrize("name,gi", [("tiny", 0), ("olmoe", 0), ("olmoe", 1), ("qwen3_30b_a3b", 0),
                                     ("qwen3_30b_a3b", 1), ("gpt_oss_120b", 0),
                                     ("gpt_oss_120b", 1), ("mixtral_8x22b", 0),
                                     ("mixtral_8x22b", 1)])
def test_dequant_debug_bit_exact(name, gi):
    w = synth.WORKLOADS[name]
    g = w.gemms[gi]
    if w.E * g.N * g.K <= 64 * 2048 * 2048:
        packed, absmax = quantised_stack(w.E, g.N, g.K, 0, g.name)
    else:
        packed, absmax = synth.random_packed_stack(w.E, g.N, g.K, seed=0, which=g.name)
    wd, ad = dev(packed), dev(absmax)
    rows = sample_rows(w.E * g.N, 512, seed=gi)
    flat_p = packed.reshape(-1, g.K // 2)[rows]
    flat_a = absmax.reshape(-1, g.K // 64)[rows]
    out32 = gnf4.gnf4_dequant_debug(wd, ad, gnf4.GNF4_OUT_F32).reshape(-1, g.K)
    want32 = oracle.dequant_f32(flat_p, flat_a)
    got32 = out32[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want32.view(np.uint32))
    del out32
    out16 = gnf4.gnf4_dequant_debug(wd, ad, gnf4.GNF4_OUT_BF16).reshape(-1, g.K)
    want16 = oracle.dequant_bf16(flat_p, flat_a)
    got16 = out16[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got16, want16)


def test_dequant_debug_adversarial_scales():
    rng = np.random.default_rng(5)
    packed = rng.integers(0, 256, size=(8, 128), dtype=np.uint8)
    absmax = np.array([0.0, 1e-45, 1e-30, 3e38], dtype=np.float32)[None, :].repeat(8, 0)
    got = gnf4.gnf4_dequant_debug(dev(packed), dev(absmax), gnf4.GNF4_OUT_F32).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), oracle.dequant_f32(packed, absmax).view(np.uint32))
    got16 = gnf4.gnf4_dequant_debug(dev(packed), dev(absmax), gnf4.GNF4_OUT_BF16)
    got16 = got16.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got16, oracle.dequant_bf16(packed, absmax))


# ---------------------------------------------------------------- moe_align
def _check_align(topk: np.ndarray, E: int):
    s_ref, sz_ref, ex_ref, ng_ref = oracle.moe_align(topk, E)
    s, sz, ex, ng = gnf4.gnf4_moe_align(dev(topk.astype(np.int32)), E)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(sz.cpu().numpy(), sz_ref)
    assert np.array_equal(ex.cpu().numpy(), ex_ref)
    assert int(ng.item()) == ng_ref


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_moe_align_bit_exact_on_workloads(name):
    w = synth.WORKLOADS[name]
    _check_align(synth.routing(w, 0), w.E)


@pytest.mark.parametrize("T,k,E,seed", [(0, 2, 4, 0), (1, 1, 1, 0), (5, 3, 2, 1), (37, 8, 1024, 2),
                                        (1000, 6, 256, 3), (4096, 2, 8, 4), (33, 4, 100, 5)])
def test_moe_align_bit_exact_random(T, k, E, seed):
    rng = np.random.default_rng(seed)
    _check_align(rng.integers(0, E, size=(T, k)).astype(np.int32), E)


def test_moe_align_duplicates_and_skew():
    rng = np.random.default_rng(6)
    topk = np.where(rng.random((500, 4)) < 0.7, 3, rng.integers(0, 16, size=(500, 4))).astype(np.int32)
    _check_align(topk, 16)


def test_moe_align_reports_bad_ids():
    topk = np.array([[0, 1], [7, 1], [2, -3]], dtype=np.int32)
    ws = gnf4.make_workspace(256)
    s, sz, ex, ng = gnf4.gnf4_moe_align(dev(topk), 4, workspace=ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 6 and bits & gnf4.DEVERR_BITS["topk"]
    assert s.cpu().tolist() == [0, 1, 3, 4, -1, -1]
    assert sz.cpu().tolist() == [1, 2, 1, 0] and ex.cpu().tolist() == [0, 1, 2, -1]
    assert gnf4.gnf4_read_device_status(ws)[0] == 0      # cleared


# ------------------------------------------------------------- grouped GEMM
def run_gemm(x_bits, packed, absmax, sizes, experts, swiglu=False, mode=gnf4.GNF4_MODE_AUTO,
             ws=None, y=None):
    yd = gnf4.gnf4_grouped_gemm(
        bf16_to_dev(x_bits), dev(packed), dev(absmax), dev(np.asarray(sizes, np.int32)),
        dev(np.asarray(experts, np.int32)),
        epilogue=gnf4.GNF4_EPI_SWIGLU if swiglu else gnf4.GNF4_EPI_NONE, mode=mode, workspace=ws,
        y=y)
    torch.cuda.synchronize()
    return yd


def check_gemm(x_bits, packed, absmax, sizes, experts, swiglu=False, mode=gnf4.GNF4_MODE_AUTO,
               rows=None, check_fidelity=True):
    M = x_bits.shape[0]
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(
        gnf4.GNF4_OP_GROUPED_GEMM, M, packed.shape[1], x_bits.shape[1], packed.shape[0], len(sizes)))
    yd = run_gemm(x_bits, packed, absmax, sizes, experts, swiglu, mode, ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 0, (st, bits)
    y = bf16_from_dev(yd)
    if rows is None:
        rows = np.arange(M)
    y = y[rows]
    ref = oracle.grouped_gemm_f64(x_bits, packed, absmax, sizes, experts, rows=rows)
    if swiglu:
        ref = oracle.swiglu_f64(ref)
    bad = tolerance_violations(y, ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} elements out of tolerance; worst " \
        f"{np.max(np.abs(y - ref)[bad])}"
    if check_fidelity:
        base_bits = oracle.baseline_bf16(x_bits, packed, absmax, sizes, experts, rows=rows)
        if swiglu:
            # the baseline's SwiGLU on its own bf16 gate_up output (fp32, one rounding)
            base_bits = oracle.baseline_swiglu_bf16(base_bits)
        base = synth.bf16_bits_to_f32(base_bits).astype(np.float64)
        assert frob_rel_err(y, ref) <= frob_rel_err(base, ref)
    return yd, ws


@pytest.mark.parametrize("name", DECODE_WORKLOADS)
def test_decode_gemm_parity_on_workloads(name):
    w = synth.WORKLOADS[name]
    _, sizes, experts, ng = groups_from_routing(w)
    touched = tuple(int(e) for e in experts[:ng])
    for g in w.gemms:
        packed, absmax = quantised_stack(w.E, g.N, g.K, 0, g.name, touched)
        x = synth.activations_bf16(w.M, g.K, seed=0, which=g.name)
        check_gemm(x, packed, absmax, sizes, experts, swiglu=g.swiglu, mode=gnf4.GNF4_MODE_DECODE)
        check_gemm(x, packed, absmax, sizes, experts, swiglu=g.swiglu, mode=gnf4.GNF4_MODE_AUTO)


@pytest.mark.parametrize("E,N,K,sizes,experts,swiglu", [
    (1, 8, 64, [1], [0], False),                              # smallest problem
    (3, 200, 192, [0, 1, 7, 8, 9, 17, 0], [2, 0, 1, 2, 0, 1, 1], False),   # ragged, zeros, >8 rows
    (4, 520, 2880, [3, 0, 12], [3, 1, 0], True),             # SwiGLU, N/2=260 not /128, K=2880
    (5, 300, 320, [2, 2, 2], [4, 4, 1], False),              # same expert in two groups
    (2, 1024, 4096, [5, 3], [1, 0], False),                  # K multiple of 256, descending ids
    (8, 64, 128, [1] * 8, list(range(8))[::-1], True),       # tiny N with SwiGLU (one column tile)
])
def test_decode_gemm_edge_cases(E, N, K, sizes, experts, swiglu):
    rng = np.random.default_rng(E * 7 + N)
    M = int(sum(sizes))
    x = synth.activations_bf16(M, K, seed=E + N)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    check_gemm(x, packed, absmax, sizes, experts, swiglu=swiglu, mode=gnf4.GNF4_MODE_DECODE)


def _pow2_rows_bf16(base_bits, scales):
    """bf16 bits of x * scales (exact: scaling a bf16 value by a power of two
    inside the normal range only changes its exponent)."""
    x = synth.bf16_bits_to_f32(base_bits).astype(np.float64) * scales
    return oracle.f32_to_bf16(x.astype(np.float32))


@pytest.mark.parametrize("swiglu,exps,spread", [
    (False, (-120, -60, -20, 0, 20, 60, 100), 40),
    # SwiGLU multiplies gate by up: keep both products inside bf16's normal range
    (True, (-50, -25, 0, 25, 50), 20),
])
def test_decode_gemm_activation_dynamic_range(swiglu, exps, spread):
    # The decode kernel converts activations to fp16 with one power-of-two
    # scale per (row, 64-block). Rows whose only non-zero block sits at a
    # scale from exps, and rows whose blocks each carry their own scale within
    # 2^-spread .. 2^spread, must all match the oracle, each row to the
    # tolerance taken over its own rms.
    rng = np.random.default_rng(31)
    E, N, K = 3, 96, 512
    M = len(exps) + 9
    base = synth.activations_bf16(M, K, seed=31)
    scales = np.zeros((M, K))
    for i, e in enumerate(exps):                 # one non-zero block per row
        b = i % (K // 64)
        scales[i, 64 * b:64 * b + 64] = 2.0 ** e
    for i in range(len(exps), M):                # every block its own scale
        for b in range(K // 64):
            scales[i, 64 * b:64 * b + 64] = 2.0 ** int(rng.integers(-spread, spread + 1))
    x = _pow2_rows_bf16(base, scales)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    sizes, experts = [5, 0, M - 5], [2, 0, 1]
    yd = run_gemm(x, packed, absmax, sizes, experts, swiglu=swiglu, mode=gnf4.GNF4_MODE_DECODE)
    y = bf16_from_dev(yd)
    ref = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    if swiglu:
        ref = oracle.swiglu_f64(ref)
    assert np.isfinite(y).all()
    for m in range(M):
        bad = tolerance_violations(y[m], ref[m])
        assert not bad.any(), f"row {m}: {bad.sum()} elements out of tolerance"


def test_decode_gemm_nonfinite_rows_stay_in_their_group():
    # A batch tile holds 8 activation rows; group 0 has 3, so rows 3..7 of
    # its tile belong to group 1 (another expert). NaN and Inf there must not
    # reach group 0's outputs, and all-zero rows give exact zeros.
    rng = np.random.default_rng(32)
    E, N, K = 2, 64, 256
    x = synth.activations_bf16(9, K, seed=32).copy()
    x[3] = 0x7FC0                       # NaN row (group 1)
    x[4, :64] = 0x7F80                  # +Inf block (group 1)
    x[5] = 0                            # all-zero row (group 1)
    x[1] = 0                            # all-zero row (group 0)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    sizes, experts = [3, 6], [1, 0]
    for swiglu in (False, True):
        yd = run_gemm(x, packed, absmax, sizes, experts, swiglu=swiglu, mode=gnf4.GNF4_MODE_DECODE)
        y = bf16_from_dev(yd)
        ref = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts, rows=np.arange(3))
        if swiglu:
            ref = oracle.swiglu_f64(ref)
        assert np.isfinite(y[:3]).all()
        assert not tolerance_violations(y[:3], ref).any()
        assert np.all(y[1] == 0.0) and np.all(y[5] == 0.0)
        assert np.isnan(y[3]).all()


def test_decode_gemm_large_groups_chunked():
    # Groups far above 8 rows go through the decode kernel in 8-row chunks.
    rng = np.random.default_rng(11)
    E, N, K = 4, 384, 512
    sizes, experts = [300, 1, 220, 503], [2, 0, 3, 1]
    M = sum(sizes)
    x = synth.activations_bf16(M, K, seed=11)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    rows = np.unique(np.concatenate([boundaries(sizes), sample_rows(M, 64, 1)]))
    check_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_DECODE, rows=rows)


def test_decode_gemm_deterministic_and_workspace_reusable():
    w = synth.WORKLOADS["qwen3_30b_a3b"]
    _, sizes, experts, ng = groups_from_routing(w)
    g = w.gemms[0]
    packed, absmax = synth.random_packed_stack(w.E, g.N, g.K, seed=3)
    x = synth.activations_bf16(w.M, g.K, seed=3)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, w.M, g.N, g.K,
                                                       w.E, w.E))
    outs = [run_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_DECODE, ws=ws)
            for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    # the status word is still clear: the workspace can be reused as is
    assert gnf4.gnf4_read_device_status(ws) == (0, 0)


def test_decode_gemm_bad_metadata_sets_error_and_writes_nothing():
    rng = np.random.default_rng(12)
    E, N, K = 3, 256, 256
    x = synth.activations_bf16(6, K, seed=12)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    for sizes, experts, bit in [([2, 2], [0, 1], "sizes"), ([3, 3], [0, 3], "expert"),
                                ([7, -1], [0, 1], "sizes")]:
        ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, 6, N, K, E, 2))
        y = torch.full((6, N), 7.0, dtype=torch.bfloat16, device="cuda")
        run_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_DECODE, ws=ws, y=y)
        st, bits = gnf4.gnf4_read_device_status(ws)
        assert st == 6 and bits & gnf4.DEVERR_BITS[bit]
        assert bool((y == 7.0).all())


def test_prefill_gemm_bad_metadata_sets_error_and_writes_nothing():
    rng = np.random.default_rng(13)
    E, N, K = 3, 256, 256
    M = 300
    x = synth.activations_bf16(M, K, seed=13)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    for sizes, experts, bit in [([100, 100], [0, 1], "sizes"), ([150, 150], [0, 3], "expert"),
                                ([301, -1], [0, 1], "sizes")]:
        ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, M, N, K, E, 2))
        y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
        run_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_PREFILL, ws=ws, y=y)
        st, bits = gnf4.gnf4_read_device_status(ws)
        assert st == 6 and bits & gnf4.DEVERR_BITS[bit]
        assert bool((y == 7.0).all())


def test_host_tensors_are_refused_on_gpu_box():
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    w = torch.zeros((1, 8, 32), dtype=torch.uint8)
    a = torch.zeros((1, 8, 1), dtype=torch.float32)
    s = torch.tensor([4], dtype=torch.int32)
    e = torch.tensor([0], dtype=torch.int32)
    with pytest.raises(gnf4.Gnf4Error) as ei:
        gnf4.gnf4_grouped_gemm(x, w, a, s, e, y=torch.zeros((4, 8), dtype=torch.bfloat16),
                               workspace=torch.zeros(1 << 20, dtype=torch.uint8))
    assert ei.value.status == 2


# ----------------------------------------------------- prefill (tensor cores)
@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (3, 200, 192, [300, 0, 513, 7], [2, 0, 1, 1]),     # ragged groups, N % 128 != 0
    (2, 384, 2048, [256, 255, 257], [1, 0, 1]),        # token-tile edges
    (4, 128, 64, [1, 1000], [3, 0]),                   # one K stage, a one-row group
    (1, 136, 640, [70], [0]),                          # a single partial tile
    (2, 100, 128, [300, 40], [1, 0]),                  # rows of y not a multiple of 16 bytes
    (2, 264, 256, [512, 64], [0, 1]),                  # whole 32-token chunks only, N % 256 = 8
])
def test_prefill_gemm_edge_cases(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 13 + N + K)
    M = int(sum(sizes))
    x = synth.activations_bf16(M, K, seed=E + N + K)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    # every row: these problems are small enough for the oracle to take whole
    check_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_PREFILL)


@pytest.mark.parametrize("exps,spread", [
    ((-120, -60, -20, 0, 20, 60, 100), 40),
    ((-8, 0, 8, 16, 24), 6),
])
def test_prefill_gemm_activation_dynamic_range(exps, spread):
    # The tensor-core kernel scales each activation row by a power of two
    # before its bf16 and e5m2 operands are made (e5m2 alone saturates above
    # 57344 and flushes below 2^-16). Rows whose only non-zero block sits at a
    # scale from exps, and rows whose blocks each carry their own scale within
    # 2^-spread .. 2^spread, must all match the oracle, each row to the
    # tolerance taken over its own rms.
    rng = np.random.default_rng(37)
    E, N, K = 3, 160, 512
    M = len(exps) + 9
    base = synth.activations_bf16(M, K, seed=37)
    scales = np.zeros((M, K))
    for i, e in enumerate(exps):                 # one non-zero block per row
        b = i % (K // 64)
        scales[i, 64 * b:64 * b + 64] = 2.0 ** e
    for i in range(len(exps), M):                # every block its own scale
        for b in range(K // 64):
            scales[i, 64 * b:64 * b + 64] = 2.0 ** int(rng.integers(-spread, spread + 1))
    x = _pow2_rows_bf16(base, scales)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    sizes, experts = [5, 0, M - 5], [2, 0, 1]
    yd = run_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_PREFILL)
    y = bf16_from_dev(yd)
    ref = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    assert np.isfinite(y).all()
    for m in range(M):
        bad = tolerance_violations(y[m], ref[m])
        assert not bad.any(), f"row {m}: {bad.sum()} elements out of tolerance"


@pytest.mark.parametrize("gi", [0, 1])
def test_prefill_gemm_full_size_mixtral(gi):
    # Full Mixtral-8x22B-shaped GEMMs in the launch configuration the benchmark
    # times (AUTO -> tensor-core kernel), checked on a stratified row sample:
    # one seeded row in each 128-row half of every 256-row token tile of every
    # group (each CTA of every tile pair), plus every group boundary; all
    # columns of each sampled row (every 256-row weight tile). The packed stack
    # is drawn directly (uniform codes, absmax in the quantised-N(0,0.02)
    # range): a multi-GB quantiser run adds nothing to this check.
    w = synth.WORKLOADS["mixtral_8x22b"]
    g = w.gemms[gi]
    _, sizes, experts, ng = groups_from_routing(w)
    packed, absmax = synth.random_packed_stack(w.E, g.N, g.K, seed=0, which=g.name)
    x = synth.activations_bf16(w.M, g.K, seed=0, which=g.name)
    rows = tile_strata(sizes[:ng], seed=3 + gi)
    assert rows.size >= 64
    check_gemm(x, packed, absmax, sizes, experts, mode=gnf4.GNF4_MODE_AUTO, rows=rows)


@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (3, 520, 192, [300, 0, 513, 7], [2, 0, 1, 1]),     # ragged groups, N/2 = 260 not /128
    (2, 512, 2048, [256, 255, 257], [1, 0, 1]),        # token-tile edges
    (2, 200, 128, [300, 40], [1, 0]),                  # rows of y (N/2 = 100) not /16 bytes
])
def test_prefill_gemm_fused_swiglu(E, N, K, sizes, experts):
    # The tensor-core kernel pairs gate row j and up row N/2 + j in the same
    # warp's TMEM lanes and combines them in the epilogue.
    rng = np.random.default_rng(E * 17 + N + K)
    M = int(sum(sizes))
    x = synth.activations_bf16(M, K, seed=E + N)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    check_gemm(x, packed, absmax, sizes, experts, swiglu=True, mode=gnf4.GNF4_MODE_PREFILL)


def test_prefill_gemm_full_size_mixtral_swiglu_through_auto():
    # Mixtral-8x22B-shaped gate_up with the fused SwiGLU: AUTO now takes the
    # tensor-core kernel (8192 rows over 8 experts); stratified rows.
    w = synth.WORKLOADS["mixtral_8x22b"]
    g = w.gemms[0]
    _, sizes, experts, ng = groups_from_routing(w)
    packed, absmax = synth.random_packed_stack(w.E, g.N, g.K, seed=0, which=g.name)
    x = synth.activations_bf16(w.M, g.K, seed=0, which=g.name)
    rows = tile_strata(sizes[:ng], seed=9)
    check_gemm(x, packed, absmax, sizes, experts, swiglu=True, mode=gnf4.GNF4_MODE_AUTO, rows=rows)
