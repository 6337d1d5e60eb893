"""GPU parity of gnf4_grouped_gemm_ex against the CPU oracle: native MXFP4
weights, NF4 with bf16 absmax, the interleaved clamped SwiGLU of gpt-oss, the
activation gather through the sort's permutation, the stream-K split of
starved grids, and the bounded waits' timeout path.

Every GEMM output is compared element by element with the fp64 oracle at
|y - y_ref| <= 1e-2*|y_ref| + 1e-3*rms(y_ref) (rms over the compared output).
"""
import numpy as np
import pytest
import torch

import grouped_nf4_w4a16_b200 as gnf4
import oracle
import synth
from conftest import frob_rel_err, tolerance_violations
from gpu_cases import bf16_from_dev, bf16_to_dev, dev, groups_from_routing, quantised_stack

pytestmark = pytest.mark.gpu

ALPHA, LIMIT = 1.702, 7.0


def _mx_stack(E, N, K, seed, lo=118, hi=124):
    """Random e2m1 codes and e8m0 scales 2^-9 .. 2^-4: values of the size of
    N(0, 0.02) weights (the released gpt-oss experts are of this kind)."""
    rng = np.random.default_rng(seed)
    w = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    sc = rng.integers(lo, hi, size=(E, N, K // 32)).astype(np.uint8)
    return w, sc


def _ex(w, scales, sizes, experts, **kw):
    ws = kw.pop("workspace", None)
    y = gnf4.gnf4_grouped_gemm_ex(dev(w), scales, dev(np.asarray(sizes, np.int32)),
                                  dev(np.asarray(experts, np.int32)), workspace=ws, **kw)
    torch.cuda.synchronize()
    return y


def _check(y_dev, ref, what=""):
    y = bf16_from_dev(y_dev)
    bad = tolerance_violations(y, ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} out of tolerance"


def _epi_ref(y, epi):
    if epi == gnf4.GNF4_EPI_SWIGLU:
        return oracle.swiglu_f64(y)
    if epi == gnf4.GNF4_EPI_SWIGLU_INTERLEAVED:
        return oracle.swiglu_interleaved_f64(y, ALPHA, LIMIT)
    return y


# ------------------------------------------------------------------ MXFP4
@pytest.mark.parametrize("E,N,K,sizes,experts,epi", [
    (1, 16, 64, [1], [0], gnf4.GNF4_EPI_NONE),
    (3, 200, 192, [0, 1, 7, 8, 9, 17, 0], [2, 0, 1, 2, 0, 1, 1], gnf4.GNF4_EPI_NONE),
    (4, 520, 2880, [3, 0, 12], [3, 1, 0], gnf4.GNF4_EPI_SWIGLU),
    (4, 520, 2880, [3, 0, 12], [3, 1, 0], gnf4.GNF4_EPI_SWIGLU_INTERLEAVED),
    (2, 1024, 4096, [5, 3], [1, 0], gnf4.GNF4_EPI_NONE),
])
def test_mxfp4_decode_parity(E, N, K, sizes, experts, epi):
    w, sc = _mx_stack(E, N, K, seed=E * 31 + N)
    x = synth.activations_bf16(int(sum(sizes)), K, seed=E + N)
    y = _ex(w, dev(sc), sizes, experts, x=bf16_to_dev(x), fmt=gnf4.GNF4_FMT_MXFP4, epilogue=epi,
            mode=gnf4.GNF4_MODE_DECODE)
    ref = _epi_ref(oracle.grouped_gemm_mxfp4_f64(x, w, sc, sizes, experts), epi)
    _check(y, ref, "mxfp4")


def test_mxfp4_extreme_scales():
    # e8m0 bytes across most of their range, a block of NaN scale (255) and
    # the smallest (0): each output row is checked against its own rms
    E, N, K = 2, 64, 256
    rng = np.random.default_rng(41)
    w = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    sc = rng.integers(60, 190, size=(E, N, K // 32)).astype(np.uint8)
    sc[1, 5, 3] = 255
    sc[0, 7, :] = 0
    x = synth.activations_bf16(6, K, seed=41)
    sizes, experts = [2, 4], [0, 1]
    y = bf16_from_dev(_ex(w, dev(sc), sizes, experts, x=bf16_to_dev(x), fmt=gnf4.GNF4_FMT_MXFP4,
                          mode=gnf4.GNF4_MODE_DECODE))
    ref = oracle.grouped_gemm_mxfp4_f64(x, w, sc, sizes, experts)
    assert np.isnan(y[2:, 5]).all() and np.isnan(ref[2:, 5]).all()
    ok = ~np.isnan(ref)
    for m in range(6):
        r = ref[m][ok[m]]
        rel = np.abs(y[m][ok[m]] - r) <= 1e-2 * np.abs(r) + 1e-3 * np.sqrt(np.mean(r ** 2))
        assert rel.all(), f"row {m}"


def test_mxfp4_full_size_gpt_oss_shape():
    # The GPT-OSS-120B-shaped expert GEMMs on native MXFP4 stacks (its released
    # format), the gate_up one with the interleaved clamped SwiGLU.
    w_ = synth.WORKLOADS["gpt_oss_120b"]
    _, sizes, experts, ng = groups_from_routing(w_)
    for g, epi in zip(w_.gemms, (gnf4.GNF4_EPI_SWIGLU_INTERLEAVED, gnf4.GNF4_EPI_NONE)):
        w, sc = _mx_stack(w_.E, g.N, g.K, seed=7 + g.K + g.N)
        x = synth.activations_bf16(w_.M, g.K, seed=0, which=g.name)
        y = _ex(w, dev(sc), sizes, experts, x=bf16_to_dev(x), fmt=gnf4.GNF4_FMT_MXFP4, epilogue=epi)
        ref = _epi_ref(oracle.grouped_gemm_mxfp4_f64(x, w, sc, sizes, experts), epi)
        _check(y, ref, f"gpt-oss {g.name}")


# ---------------------------------------------------------- bf16 absmax
@pytest.mark.parametrize("name", ["olmoe", "qwen3_30b_a3b", "gpt_oss_120b"])
def test_nf4_bf16_absmax_on_workloads(name):
    w_ = synth.WORKLOADS[name]
    _, sizes, experts, ng = groups_from_routing(w_)
    touched = tuple(int(e) for e in experts[:ng])
    for g in w_.gemms:
        packed, absmax = quantised_stack(w_.E, g.N, g.K, 0, g.name, touched)
        ab = oracle.f32_to_bf16(absmax)
        x = synth.activations_bf16(w_.M, g.K, seed=0, which=g.name)
        epi = gnf4.GNF4_EPI_SWIGLU if g.swiglu else gnf4.GNF4_EPI_NONE
        y = _ex(packed, dev(ab).view(torch.bfloat16), sizes, experts, x=bf16_to_dev(x),
                epilogue=epi)
        ref = _epi_ref(oracle.grouped_gemm_bf16_absmax_f64(x, packed, ab, sizes, experts), epi)
        _check(y, ref, f"{name} {g.name}")


def test_bf16_absmax_odd_row_lengths():
    # K / 64 odd: consecutive rows' bf16 absmax start at alternating 2-byte
    # offsets, and the last element of the stack sits at a word boundary
    E, N, K = 3, 40, 192
    rng = np.random.default_rng(43)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    ab = oracle.f32_to_bf16(rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32))
    sizes, experts = [4, 0, 9], [2, 0, 1]
    x = synth.activations_bf16(13, K, seed=43)
    for mode in (gnf4.GNF4_MODE_DECODE, gnf4.GNF4_MODE_AUTO):
        y = _ex(packed, dev(ab).view(torch.bfloat16), sizes, experts, x=bf16_to_dev(x), mode=mode)
        _check(y, oracle.grouped_gemm_bf16_absmax_f64(x, packed, ab, sizes, experts), "bf16 absmax")


# ------------------------------------------ fp32 absmax copy paths
@pytest.mark.parametrize("epi", [gnf4.GNF4_EPI_NONE, gnf4.GNF4_EPI_SWIGLU])
def test_fp32_absmax_unaligned_base_matches_aligned(epi):
    # K % 256 == 0 with a 16-byte aligned absmax takes one 16-byte scale copy
    # per row and stage; the same absmax 4 bytes past a 16-byte boundary
    # takes 4-byte copies. Same values, same arithmetic: bit-identical output.
    E, N, K = 3, 272, 1024
    rng = np.random.default_rng(77 + epi)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    sizes, experts = [5, 0, 8, 3], [2, 0, 1, 0]
    x = synth.activations_bf16(int(sum(sizes)), K, seed=78)
    aligned = dev(absmax)
    assert aligned.data_ptr() % 16 == 0
    buf = torch.zeros(absmax.size + 4, dtype=torch.float32, device="cuda")
    shifted = buf[1:1 + absmax.size].view(absmax.shape)
    shifted.copy_(aligned)
    assert shifted.data_ptr() % 16 == 4
    ys = [_ex(packed, a, sizes, experts, x=bf16_to_dev(x), epilogue=epi, mode=gnf4.GNF4_MODE_DECODE)
          for a in (aligned, shifted)]
    assert torch.equal(ys[0], ys[1])
    _check(ys[1], _epi_ref(oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts), epi),
           "fp32 absmax, 4-byte copies")


# ------------------------------------------ interleaved clamped SwiGLU
@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (4, 520, 2880, [3, 0, 12], [3, 1, 0]),
    (8, 64, 128, [1] * 8, list(range(8))[::-1]),
    (2, 272, 512, [9, 17], [0, 1]),
])
def test_nf4_swiglu_interleaved_parity(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 5 + N)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    # large enough scales that some gates and ups pass the clamp limit
    absmax = rng.uniform(0.05, 0.6, size=(E, N, K // 64)).astype(np.float32)
    x = synth.activations_bf16(int(sum(sizes)), K, seed=E + K)
    y = _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x),
            epilogue=gnf4.GNF4_EPI_SWIGLU_INTERLEAVED, swiglu_alpha=ALPHA, swiglu_limit=LIMIT)
    pre = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    assert (pre[:, 0::2] > LIMIT).any() or K <= 512
    ref = oracle.swiglu_interleaved_f64(pre, ALPHA, LIMIT)
    _check(y, ref, "interleaved swiglu")
    # no worse than the same activation on the dequantise-to-bf16 baseline's output
    base = synth.bf16_bits_to_f32(oracle.baseline_bf16(x, packed, absmax, sizes, experts))
    base_act = oracle.swiglu_interleaved_f64(base.astype(np.float64), ALPHA, LIMIT)
    assert frob_rel_err(bf16_from_dev(y), ref) <= frob_rel_err(base_act, ref)


# ---------------------------------------------------------------- gather
@pytest.mark.parametrize("name", ["tiny", "olmoe", "qwen3_30b_a3b", "gpt_oss_120b"])
def test_gather_through_sorted_idx_on_workloads(name):
    # the whole chain on the device: moe_align's permutation feeds the GEMM,
    # which reads hidden[sorted_idx[i] / top_k] itself (no sorted copy of x)
    w_ = synth.WORKLOADS[name]
    topk = synth.routing(w_, 0)
    s_d, sz_d, ex_d, ng_d = gnf4.gnf4_moe_align(dev(topk), w_.E)
    sorted_idx, sizes, experts, ng = oracle.moe_align(topk, w_.E)
    g = w_.gemms[0]
    hidden = synth.activations_bf16(w_.T, g.K, seed=5)
    packed, absmax = synth.random_packed_stack(w_.E, g.N, g.K, seed=5)
    epi = gnf4.GNF4_EPI_SWIGLU if g.swiglu else gnf4.GNF4_EPI_NONE
    y = gnf4.gnf4_grouped_gemm_ex(dev(packed), dev(absmax), sz_d, ex_d, hidden=bf16_to_dev(hidden),
                                  sorted_idx=s_d, top_k=w_.top_k, M=w_.M, epilogue=epi)
    torch.cuda.synchronize()
    x = oracle.gather_rows(hidden, sorted_idx, w_.top_k)
    ref = _epi_ref(oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts), epi)
    _check(y, ref, f"gather {name}")
    # and identical bits to the same GEMM on the gathered copy
    y2 = _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), epilogue=epi)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_gather_bad_slot_sets_error_and_writes_nothing():
    E, N, K, T, k = 3, 64, 256, 4, 2
    rng = np.random.default_rng(44)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    hidden = synth.activations_bf16(T, K, seed=44)
    sidx = np.array([0, 1, 2, 3, 4, 5, 6, T * k], np.int32)     # last entry out of range
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, 8, N, K, E, 2))
    y = torch.full((8, N), 5.0, dtype=torch.bfloat16, device="cuda")
    gnf4.gnf4_grouped_gemm_ex(dev(packed), dev(absmax), dev(np.array([4, 4], np.int32)),
                              dev(np.array([0, 2], np.int32)), hidden=bf16_to_dev(hidden),
                              sorted_idx=dev(sidx), top_k=k, y=y, workspace=ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 6 and bits & gnf4.DEVERR_BITS["slot"]
    assert bool((y == 5.0).all())


# ------------------------------------------------------ stream-K split
@pytest.mark.parametrize("N,K,sizes", [
    (16, 8192, [1]),                 # one tile of 32 stages across many SMs
    (128, 4096, [3, 5]),             # two tiles
    (2048, 2048, [1] * 8),           # the OLMoE-shaped gate_up: 128 tiles on more SMs
])
def test_starved_grid_split_is_exact_and_deterministic(N, K, sizes):
    E = len(sizes)
    rng = np.random.default_rng(N + K)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    experts = list(range(E))
    x = synth.activations_bf16(int(sum(sizes)), K, seed=N)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, int(sum(sizes)),
                                                       N, K, E, E))
    outs = [_ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), workspace=ws,
                mode=gnf4.GNF4_MODE_DECODE) for _ in range(3)]
    _check(outs[0], oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts), "split")
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    # every tile counter is back at zero: the workspace is reusable as is
    assert gnf4.gnf4_read_device_status(ws) == (0, 0)
    n_counters = torch.cuda.get_device_properties(0).multi_processor_count * 4
    assert int(ws[256:256 + 4 * n_counters].count_nonzero().item()) == 0


# ------------------------------------------------------- bounded waits
def test_decode_wait_limit_runs_out_cleanly():
    # The workspace header's word 2 shortens every bounded wait of the decode
    # kernel (0: the 2 s default). At 1 ns the activation warp's first wait
    # runs out before the first stage's copies can land: the kernel records
    # GNF4_DEVERR_TIMEOUT, lets its copies land, returns without writing y,
    # and the context stays usable.
    E, N, K = 2, 256, 1024
    rng = np.random.default_rng(45)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    x = synth.activations_bf16(6, K, seed=45)
    sizes, experts = [2, 4], [1, 0]
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, 6, N, K, E, 2))
    ws[8:12] = torch.tensor([1, 0, 0, 0], dtype=torch.uint8)       # limit 1 ns
    y = torch.full((6, N), 9.0, dtype=torch.bfloat16, device="cuda")
    _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), y=y, workspace=ws,
        mode=gnf4.GNF4_MODE_DECODE)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 7 and bits == gnf4.DEVERR_BITS["timeout"]
    assert bool((y == 9.0).all())
    # a fresh workspace: the same call completes and is right
    y = _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), mode=gnf4.GNF4_MODE_DECODE)
    _check(y, oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts), "after timeout")


# ------------------------------------------------ tensor-core kernel variants
PREFILL_CASES = [
    (3, 520, 192, [300, 0, 513, 7], [2, 0, 1, 1]),     # ragged groups, partial weight tiles
    (2, 512, 2048, [256, 255, 257], [1, 0, 1]),        # token-tile edges
]


@pytest.mark.parametrize("E,N,K,sizes,experts", PREFILL_CASES)
@pytest.mark.parametrize("epi", [gnf4.GNF4_EPI_NONE, gnf4.GNF4_EPI_SWIGLU,
                                 gnf4.GNF4_EPI_SWIGLU_INTERLEAVED])
def test_prefill_mxfp4(E, N, K, sizes, experts, epi):
    # MXFP4 code values times their e8m0 scales are exact in bf16: one bf16
    # pass, no remainder pass
    w, sc = _mx_stack(E, N, K, seed=E * 7 + K)
    x = synth.activations_bf16(int(sum(sizes)), K, seed=N)
    y = _ex(w, dev(sc), sizes, experts, x=bf16_to_dev(x), fmt=gnf4.GNF4_FMT_MXFP4, epilogue=epi,
            mode=gnf4.GNF4_MODE_PREFILL)
    ref = _epi_ref(oracle.grouped_gemm_mxfp4_f64(x, w, sc, sizes, experts), epi)
    _check(y, ref, "prefill mxfp4")


@pytest.mark.parametrize("E,N,K,sizes,experts", PREFILL_CASES)
def test_prefill_bf16_absmax(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 3 + N)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    ab = oracle.f32_to_bf16(rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32))
    x = synth.activations_bf16(int(sum(sizes)), K, seed=K)
    y = _ex(packed, dev(ab).view(torch.bfloat16), sizes, experts, x=bf16_to_dev(x),
            mode=gnf4.GNF4_MODE_PREFILL)
    _check(y, oracle.grouped_gemm_bf16_absmax_f64(x, packed, ab, sizes, experts), "prefill bf16")


@pytest.mark.parametrize("E,N,K,sizes,experts", PREFILL_CASES)
def test_prefill_swiglu_interleaved(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 11 + N)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.05, 0.6, size=(E, N, K // 64)).astype(np.float32)
    x = synth.activations_bf16(int(sum(sizes)), K, seed=K + 1)
    y = _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), mode=gnf4.GNF4_MODE_PREFILL,
            epilogue=gnf4.GNF4_EPI_SWIGLU_INTERLEAVED, swiglu_alpha=ALPHA, swiglu_limit=LIMIT)
    ref = oracle.swiglu_interleaved_f64(oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts),
                                        ALPHA, LIMIT)
    _check(y, ref, "prefill interleaved swiglu")


def test_prefill_gather_chain_mixtral_shape():
    # Mixtral-shaped routing: moe_align on the device, then the tensor-core
    # GEMM reading hidden[sorted_idx[i] / top_k] itself; the output must be
    # bit-identical to the same GEMM on the gathered copy, and match the
    # oracle on a stratified row sample
    from gpu_cases import tile_strata
    w_ = synth.WORKLOADS["mixtral_8x22b"]
    topk = synth.routing(w_, 0)
    s_d, sz_d, ex_d, ng_d = gnf4.gnf4_moe_align(dev(topk), w_.E)
    sorted_idx, sizes, experts, ng = oracle.moe_align(topk, w_.E)
    K, N = 1024, 768
    hidden = synth.activations_bf16(w_.T, K, seed=6)
    packed, absmax = synth.random_packed_stack(w_.E, N, K, seed=6)
    y = gnf4.gnf4_grouped_gemm_ex(dev(packed), dev(absmax), sz_d, ex_d, hidden=bf16_to_dev(hidden),
                                  sorted_idx=s_d, top_k=w_.top_k, M=w_.M,
                                  mode=gnf4.GNF4_MODE_PREFILL)
    torch.cuda.synchronize()
    x = oracle.gather_rows(hidden, sorted_idx, w_.top_k)
    y2 = _ex(packed, dev(absmax), sizes, experts, x=bf16_to_dev(x), mode=gnf4.GNF4_MODE_PREFILL)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    rows = tile_strata(sizes[:ng], seed=4)
    ref = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts, rows=rows)
    bad = tolerance_violations(bf16_from_dev(y)[rows], ref)
    assert not bad.any()


def test_prefill_gather_bad_slot_writes_nothing():
    E, N, K, T, k = 2, 256, 256, 300, 2
    rng = np.random.default_rng(46)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    hidden = synth.activations_bf16(T, K, seed=46)
    sidx = np.arange(T * k, dtype=np.int32)
    sidx[377] = -5
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_GEMM, T * k, N, K, E, 2))
    y = torch.full((T * k, N), 5.0, dtype=torch.bfloat16, device="cuda")
    gnf4.gnf4_grouped_gemm_ex(dev(packed), dev(absmax), dev(np.array([300, 300], np.int32)),
                              dev(np.array([1, 0], np.int32)), hidden=bf16_to_dev(hidden),
                              sorted_idx=dev(sidx), top_k=k, y=y, workspace=ws,
                              mode=gnf4.GNF4_MODE_PREFILL)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 6 and bits & gnf4.DEVERR_BITS["slot"]
    assert bool((y == 5.0).all())
