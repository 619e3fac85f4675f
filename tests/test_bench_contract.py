"""bench.py on the host: the reference arm's JSON line, and the hash that
keys the DRAM-traffic figures to the kernel code they were captured from.

`bench.py --impl reference` times the fp64 oracle on the host cores (no GPU
needed), so its line can be checked here: the same metric, unit and
config keys as the CUDA arm, its own `cpu_baseline` and a zero-copy `e2e`.
Under torchrun only rank 0 prints; the other ranks exit 0 without work.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["--impl", "reference", "--workload", "tiny_fp32", "--steps", "2", "--warmup", "3"]


def _json_lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_line(d, n_gpus):
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == n_gpus and d["steps"] == 2 and d["warmup"] == 3
    assert d["ms_per_step"] > 0 and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"].startswith("tiny_fp32")
    # the same config object as the CUDA arm's line
    assert set(d["config"]) == {"workload", "global_batch_tokens", "parallelism", "l2"}
    assert d["config"]["global_batch_tokens"] == 256 * n_gpus
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, "bench.py"] + ARGS, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1)


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29613", "bench.py", "--gpus", "2"] + ARGS
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 2)


def test_capture_validity_ignores_comments_and_layout_only():
    """A DRAM-traffic figure in the bench line stays valid while the code of
    the captured kernel is unchanged (otherwise the line reports null):
    comments and whitespace do not count, any token of code does."""
    sys.path.insert(0, ROOT)
    import bench

    src = ("// header comment\n__global__ void k(int *p) {\n"
           "  /* block\n comment */ p[0] = 1;  // trailing\n}\n")
    same = "__global__ void k(int *p) {\n\n    p[0] = 1;\n}\n// another note\n"
    assert bench.code_text(src) == bench.code_text(same)
    assert bench.code_text(src) != bench.code_text(src.replace("p[0] = 1", "p[0] = 2"))
    assert bench.code_text(src) != bench.code_text(src.replace("int *p", "int *q"))
    for entry in bench.NCU_TRAFFIC.values():
        assert len(bench.source_hash(entry["source"])) == 16
