"""GPU parity for the grouped dgrad (package page "grouped-nf4-gemm", header
block, "Owns": the grouped packed GEMM and its dgrad), through the C ABI,
against the fp64 oracle: every element of dx within
|dx - dx_ref| <= 1e-2 |dx_ref| + 1e-3 rms(dx_ref) (the GEMM tolerance; the
kernel's fp32 weight products and fp32 sums are far inside it), and the
device error word for bad group metadata, with nothing written.
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


@pytest.mark.parametrize("E,N,K,sizes,experts", [
    (1, 8, 64, [1], [0]),                                    # smallest problem
    (3, 200, 192, [0, 1, 7, 8, 9, 17, 0], [2, 0, 1, 2, 0, 1, 1]),   # ragged, empty groups
    (4, 2048, 1024, [2, 3, 0, 3], [3, 1, 0, 0]),             # OLMoE-like down shapes
    (2, 96, 2880, [5, 4], [1, 1]),                           # K = 2880 (not a multiple of 256)
    (3, 1024, 2048, [1, 1, 1, 1, 1, 1, 1, 1], [0, 1, 2, 0, 1, 2, 0, 1]),  # 8 one-row groups: a starved grid
    (2, 5760, 2880, [37, 3], [1, 0]),                        # GPT-OSS-like gate_up rows, > 8 rows a group
    (8, 64, 320, [1] * 8, list(range(8))[::-1]),
])
def test_grouped_dgrad_parity(E, N, K, sizes, experts):
    rng = np.random.default_rng(E * 7 + N + K)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    M = int(sum(sizes))
    dy = synth.activations_bf16(M, N, seed=N + K)
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_DGRAD, M, N, K, E,
                                                       len(sizes)))
    dx = gnf4.gnf4_grouped_dgrad(bf16_to_dev(dy), dev(packed), dev(absmax),
                                 dev(np.asarray(sizes, np.int32)), dev(np.asarray(experts, np.int32)),
                                 workspace=ws)
    st, bits = gnf4.gnf4_read_device_status(ws)
    assert st == 0, (st, bits)
    ref = oracle.grouped_dgrad_f64(dy, packed, absmax, sizes, experts)
    bad = tolerance_violations(bf16_from_dev(dx), ref)
    assert not bad.any(), f"{bad.sum()} of {bad.size} elements out of tolerance"


def test_grouped_dgrad_bad_metadata_sets_error_and_writes_nothing():
    rng = np.random.default_rng(12)
    E, N, K = 3, 64, 128
    dy = synth.activations_bf16(6, N, seed=12)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    for sizes, experts, bit in [([2, 2], [0, 1], "sizes"), ([3, 3], [0, 3], "expert"),
                                ([7, -1], [0, 1], "sizes")]:
        ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(gnf4.GNF4_OP_GROUPED_DGRAD, 6, N, K, E, 2))
        dx = torch.full((6, K), 7.0, dtype=torch.bfloat16, device="cuda")
        gnf4.gnf4_grouped_dgrad(bf16_to_dev(dy), dev(packed), dev(absmax),
                                dev(np.asarray(sizes, np.int32)),
                                dev(np.asarray(experts, np.int32)), dx=dx, workspace=ws)
        st, bits = gnf4.gnf4_read_device_status(ws)
        assert st == 6 and bits & gnf4.DEVERR_BITS[bit]
        assert bool((dx == 7.0).all())
