"""The N > 1 host logic of bench.py on CPU, world size 2 over gloo: the
max-over-ranks timing reduction, and the reference arm (rank 0 runs and
prints one line, the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _torchrun(args, timeout=600):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=timeout)


def test_max_over_ranks_world_size_2():
    r = _torchrun([os.path.join("tests", "multirank_worker.py")])
    assert r.returncode == 0, r.stdout + r.stderr
    assert "rank 0 max 2.5" in r.stdout and "rank 1 max 2.5" in r.stdout


def test_reference_arm_world_size_2_prints_one_line():
    r = _torchrun(["bench.py", "--impl", "reference", "--workload", "tiny", "--gpus", "2",
                   "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_counter_key_ignores_comments_but_not_code(tmp_path):
    # bench.py keys the committed ncu counters by a hash of a kernel source's
    # code: editing a comment keeps them, editing code drops them
    import sys
    sys.path.insert(0, ROOT)
    import bench
    base = "int f(int a) {\n  return a + 1;   // one\n}\n/* block\n comment */\n"
    p = tmp_path / "k.cu"
    p.write_text(base)
    h0 = bench.source_hash(str(p))
    p.write_text(base.replace("// one", "// the successor").replace("block", "other block") + "\n\n")
    assert bench.source_hash(str(p)) == h0
    p.write_text(base.replace("a + 1", "a + 2"))
    assert bench.source_hash(str(p)) != h0


def test_reference_arm_never_loads_the_product_library():
    # The reference arm is the oracle on the host cores: its inputs are built
    # on the host and the product package (and so libgnf4.so) is never loaded.
    code = ("import sys, types; sys.argv = ['bench.py']; import bench; "
            "a = types.SimpleNamespace(workload='tiny', steps=1, warmup=3); "
            "line = bench.run_reference(a, 0, 1); "
            "print('LOADED' if 'grouped_nf4_w4a16_b200' in sys.modules else 'CLEAN', line['impl'])")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "CLEAN reference" in r.stdout
