"""The bench's oracle-timing legs on the host (no GPU needed).

`cpu_baseline`, the side lines' `cpu_oracle` and the `--impl reference` arm all
time the CPU oracle on a sample of a workload's queries and extrapolate to the
whole batch.  Checked here on small workloads: the sample covers every query
when the budget allows, slot subsampling reports what it timed, the reference
arm prints one well-formed JSON line, and the size overrides parse.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from block_sparse_attention_22_b200 import synth  # noqa: E402


def test_parse_overrides():
    assert bench.parse_overrides("n_seqs=2,ctx=262144") == {"n_seqs": 2, "ctx": 262144}
    assert bench.parse_overrides("drift=0.5") == {"drift": 0.5}
    assert bench.parse_overrides("") == {}


def test_oracle_side_lines_name_workloads():
    for name, (slots, budget) in bench.ORACLE_SIDE.items():
        assert synth.make_workload(name).name == name       # a recipe (no tensors are drawn)
        assert slots >= 0 and budget > 0


def test_oracle_sample_times_every_query_of_a_small_batch():
    wl = synth.make_workload("tiny_fp32")
    x = synth.make_inputs(wl)
    v, threads, desc = bench.oracle_sample(wl, x, target_s=2.0)
    assert v > 0
    assert threads == len(os.sched_getaffinity(0))
    assert f"{wl.n_tokens} of {wl.n_tokens} queries (all)" in desc


def test_oracle_sample_times_a_subset_of_slots():
    wl = synth.make_workload("decode_256k", ctx=2001, n_seqs=4)
    x = synth.make_inputs(wl)
    v, _, desc = bench.oracle_sample(wl, x, target_s=1.0, max_slots=2)
    assert v > 0
    assert desc.startswith("2 of 4 sequences timed")


def test_reference_arm_prints_one_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_fp32",
         "--steps", "2", "--warmup", "1", "--ref-seconds", "1"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
