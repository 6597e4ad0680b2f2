"""The reference arm of bench.py (the CPU oracle, timed on the host cores)
keeps the JSON-line contract: one line from rank 0 with the metric, the
workload, the e2e object and the cpu_baseline object, and nothing from the
other ranks.  Runs on the CPU, on the small workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "0", "--workload", "linear_512_n256"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_json_line():
    p = _run({"RANK": "0"})
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"] == "linear_512_n256"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert "sample" in cb
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    p = _run({"RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_bench_jobs_cover_each_workload():
    """One bench step covers every linear of the workload: the 70B-shaped
    block's seven linears on four distinct inputs (q/k/v share one, gate/up
    another), the sweep's two activation variants under three quantiser
    settings on one weight; the flops the roofline divides by are
    n_alpha x 2 N D_in D_out summed over the searches."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    sys.modules["bench_mod"] = bench          # the dataclasses look their module up
    spec.loader.exec_module(bench)
    block = bench.make_job("llama70b_block")
    assert len(block.xs) == 4 and len(block.ws) == 7 and len(block.searches) == 7 and block.A == 21
    assert [s.x for s in block.searches] == [0, 0, 0, 1, 2, 2, 3]
    assert block.flops() == 21 * 2.0 * 4096 * (2 * 8192 * 8192 + 2 * 8192 * 1024 + 2 * 8192 * 28672 + 28672 * 8192)
    assert block.units() == 7 * 21
    sweep = bench.make_job("sweep_4096x11008_n16k")
    assert len(sweep.xs) == 2 and len(sweep.ws) == 1 and sweep.A == 41
    assert sorted((s.bits, s.group, s.x) for s in sweep.searches) == sorted(
        (b, g, x) for b, g in ((4, 128), (4, 64), (3, 128)) for x in (0, 1))
    other = bench.make_job("llama70b_block", rank=2)
    assert [x[2].seed for x in other.xs] == [2000, 2001, 2002, 2003]     # another rank, another block
