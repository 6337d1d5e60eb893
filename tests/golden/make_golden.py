"""Writes the stored oracle outputs under tests/golden/.

Calls only the CPU oracle (oracle/) and the seeded input generators (synth/).
Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def tiny_case(seed=0):
    w = synth.WORKLOADS["tiny"]
    g = w.gemms[0]
    topk = synth.routing(w, seed)
    sorted_idx, sizes, experts, ng = oracle.moe_align(topk, w.E)
    x = synth.activations_bf16(w.M, g.K, seed)
    packed, absmax = oracle.quantized_stack(
        w.E, g.N, g.K, lambda e: synth.expert_weights_f32(w.E, g.N, g.K, e, seed))
    y = oracle.grouped_gemm_f64(x, packed, absmax, sizes, experts)
    yb = oracle.baseline_bf16(x, packed, absmax, sizes, experts)
    return dict(topk=topk, sorted_idx=sorted_idx, sizes=sizes, expert_ids=experts,
                num_groups=np.int32(ng), x=x, packed=packed, absmax=absmax, y_ref=y,
                y_baseline=yb)


if __name__ == "__main__":
    out = os.path.join(HERE, "tiny_seed0.npz")
    np.savez_compressed(out, **tiny_case(0))
    print("wrote", out)
