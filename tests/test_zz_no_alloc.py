"""gnf4_grouped_gemm_noalloc: the decode grouped GEMM for callers that cannot
allocate device memory (for example a plugin whose host application owns all
device memory through its own pool, or a latency-critical path that cannot
accept the implicit synchronisation of an allocation). Instead of a caller
workspace it uses a fixed scratch array inside the library.

This file is named so that pytest collects it last: a failure here leaves
every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import grouped_nf4_w4a16_b200 as gnf4
import synth
from gpu_cases import bf16_to_dev, dev


def _problem(seed, E, N, K, sizes, experts):
    rng = np.random.default_rng(seed)
    M = int(sum(sizes))
    x = synth.activations_bf16(M, K, seed=seed)
    packed = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    absmax = rng.uniform(0.01, 0.1, size=(E, N, K // 64)).astype(np.float32)
    return (bf16_to_dev(x), dev(packed), dev(absmax), dev(np.asarray(sizes, np.int32)),
            dev(np.asarray(experts, np.int32)))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # Two different problems back to back: the second call must not see
    # anything the first one left in the shared scratch array. Both entry
    # points run the same kernel on the same inputs, so the outputs must be
    # bit-identical (a tolerance could hide stale scratch that perturbs a few
    # values slightly).
    cases = [
        (dict(seed=1, E=16, N=1536, K=2048, sizes=[3, 0, 12, 1, 9, 8, 2], experts=[5, 0, 2, 15, 7, 1, 9]),
         gnf4.GNF4_EPI_NONE),
        (dict(seed=2, E=8, N=520, K=2880, sizes=[1, 4, 0, 7], experts=[3, 0, 6, 2]),
         gnf4.GNF4_EPI_SWIGLU),
    ]
    for kw, epi in cases:
        x, w, a, s, e = _problem(**kw)
        ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(
            gnf4.GNF4_OP_GROUPED_GEMM, x.shape[0], w.shape[1], x.shape[1], w.shape[0], s.numel()))
        want = gnf4.gnf4_grouped_gemm(x, w, a, s, e, epilogue=epi, mode=gnf4.GNF4_MODE_DECODE,
                                      workspace=ws)
        got = gnf4.gnf4_grouped_gemm_noalloc(x, w, a, s, e, epilogue=epi)
        torch.cuda.synchronize()
        assert gnf4.gnf4_read_device_status(ws) == (0, 0)
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))


@pytest.mark.gpu
def test_noalloc_good_call_after_bad_metadata_call():
    # A call whose device-side metadata is wrong (sizes do not sum to M) sets
    # the error word inside the scratch array and writes nothing to y. The
    # next good call clears that word first, so it runs normally and returns
    # the same bits as the workspace entry point.
    x, w, a, s, e = _problem(seed=3, E=6, N=384, K=1024, sizes=[2, 5, 3], experts=[4, 0, 5])
    bad_sizes = dev(np.asarray([2, 5, 4], np.int32))      # sums to 11, M is 10
    y_bad = torch.full((x.shape[0], w.shape[1]), 3.0, dtype=torch.bfloat16, device="cuda")
    gnf4.gnf4_grouped_gemm_noalloc(x, w, a, bad_sizes, e, y=y_bad)
    torch.cuda.synchronize()
    assert bool((y_bad == 3.0).all())
    ws = gnf4.make_workspace(gnf4.gnf4_workspace_bytes(
        gnf4.GNF4_OP_GROUPED_GEMM, x.shape[0], w.shape[1], x.shape[1], w.shape[0], s.numel()))
    want = gnf4.gnf4_grouped_gemm(x, w, a, s, e, mode=gnf4.GNF4_MODE_DECODE, workspace=ws)
    for _ in range(2):
        got = gnf4.gnf4_grouped_gemm_noalloc(x, w, a, s, e)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_noalloc_scratch_limit_follows_the_decode_workspace():
    # The entry point sizes its scratch need from the decode kernel (the
    # 256-byte status header): even a huge problem passes the scratch check
    # and is refused further on for its fake pointers, never for scratch.
    lib = gnf4.load_library()
    st = lib.gnf4_grouped_gemm_noalloc(1, 1, 1, 1, 1, 8, 1 << 24, 32768, 6144, 8, 64, 0, 1, None)
    assert st not in (0, 9)
    assert "SCRATCH_LIMIT" in gnf4.gnf4_status_string(9)
    assert gnf4.GNF4_NOALLOC_SCRATCH_BYTES == 8 << 20
