"""The reference arm of bench.py (the CPU oracle timed on the host) prints one JSON line with
the keys the benchmark contract asks for; under a multi-rank launch only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ, **(extra_env or {}))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_prints_the_contract_line():
    lines = _run()
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["n_gpus"] == 1 and d["warmup"] >= 3 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"]


def test_reference_arm_other_ranks_exit_quietly():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_cpu_baseline_takes_a_checkpoint_layout_case():
    """The batch workload draws its weights in the checkpoint layout; the baseline repacks them."""
    import bench
    import synth
    c = synth.make_case(4, 256, 64, 64, sym=False, seed=5, ckpt_layout=True)
    assert c.get("b") is None
    r = bench.cpu_baseline(c, seconds=0.01)
    assert r["kind"] == "oracle" and r["value"] > 0 and "M=4 K=256 N=64" in r["sample"]


def test_source_hash_ignores_comments_and_layout_only():
    """The traffic record is tied to the kernel's code: comments and whitespace do not change the
    hash, a change inside a string literal or of a token does."""
    import bench
    base = 'int a = 1; // one\n/* two\n lines */ const char* s = "x // y"; char c = \'"\';\n'
    assert bench.code_only(base) == bench.code_only('int a = 1;\nconst char* s = "x // y";  char c = \'"\'; // z\n')
    assert bench.code_only(base) != bench.code_only(base.replace('"x // y"', '"x //  y"'))
    assert bench.code_only(base) != bench.code_only(base.replace("a = 1", "a = 2"))
