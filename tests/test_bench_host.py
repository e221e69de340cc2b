"""Host-side pieces of bench.py that need no GPU.

The union-tile bench line reports the distinct kept blocks of every tile of
neighbouring queries; it computes them with a sort, independently of the
library's union lists.  Here that count is checked against Python sets on
small ragged batches, including rows shorter than the budget (padding -1
past nsel must not count) and tiles cut at segment ends.
"""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _reference(sel, nsel, segl, mq):
    out = []
    for off, q_len, _, _ in segl:
        for q0 in range(0, q_len, mq):
            rows = range(off + q0, off + min(q_len, q0 + mq))
            out.append(len({int(b) for i in rows for b in sel[i, :int(nsel[i])].tolist()}))
    return out


def test_union_lengths_match_sets_on_ragged_batches():
    g = torch.Generator().manual_seed(11)
    S = 16
    segl = [(0, 23, 40, 0), (23, 1, 900, 1), (24, 10, 0, 2)]       # 23 = 2 tiles of 10 + 3
    T = 34
    sel = torch.full((T, S), -1, dtype=torch.int32)
    nsel = torch.zeros(T, dtype=torch.int32)
    for t in range(T):
        n = int(torch.randint(1, S + 1, (1,), generator=g))
        blocks = torch.randperm(40, generator=g)[:n].sort().values
        sel[t, :n] = blocks.to(torch.int32)
        sel[t, n:] = 7 if t % 2 else -1        # stale entries past nsel are ignored
        nsel[t] = n
    for mq in (1, 3, 10, 32):
        got = bench.union_lengths(sel, nsel, segl, mq).tolist()
        assert got == _reference(sel, nsel, segl, mq), mq


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1000, 2.0, 1) == 500000.0
    assert bench.job_throughput(1000, 2.0, 4) == 2000000.0


def test_algorithmic_work_matches_the_per_unit_figures():
    """The bench's algorithmic work against the per-unit figures of the method:
    a 1M-context decode query streams its sequence's k^ (262143 blocks x 128
    dims x 2 B = 67.1 MB) and gathers 512 kept blocks of K and V in both groups
    (4.19 MB); the 128K prefill does 2.20 TFLOP of indexer and 6.54 TFLOP of
    attention contractions and gathers 545 GB at zero reuse."""
    from block_sparse_attention_22_b200 import synth
    w = bench.algorithmic_work(synth.make_workload("decode_1m"))
    assert w["index"]["khat_bytes"] == 8 * 262143 * 128 * 2
    assert w["attn"]["gathered_bytes"] == 8 * 512 * 4 * 2 * 256 * 2 * 2
    per_query = w["algorithmic_bytes"] / 8
    assert 71.3e6 < per_query < 71.5e6, per_query
    assert w["actual_bytes"] - w["algorithmic_bytes"] == 2 * w["index"]["score_bytes"]
    p = bench.algorithmic_work(synth.make_workload("prefill_128k"))
    assert abs(p["index"]["flops"] - 2.20e12) < 0.01e12
    assert abs(p["attn"]["flops"] - 6.54e12) < 0.01e12
    assert abs(p["attn"]["gathered_bytes"] - 545.5e9) < 0.5e9
    assert p["index"]["khat_bytes"] == 0            # a prefill's k^ is L2-resident


def test_step_tensor_roofline_arithmetic():
    work = {"flops": 8.0e12, "compress": {"bytes": 1e6},
            "index": {"flops": 2.0e12, "khat_bytes": 0.0, "query_bytes": 1e6},
            "attn": {"flops": 6.0e12, "bytes": 500e9}}
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0, "source": "test"}
    r = bench.step_tensor_roofline(work, 80.0, [0.1, 4.0, 5.0, 70.0], peaks)
    assert abs(r["achieved"] - 100.0) < 1e-9          # 8e12 flop / 80 ms
    assert abs(r["frac"] - 0.1) < 1e-12
    assert abs(r["index_stage"]["frac"] - 0.5) < 1e-12
    # attainable: 1e6/5e12 + 2e12/1e15 + 0 + 500e9/5e12 seconds
    assert abs(r["attainable"]["ms_per_step"] - (0.0002 + 2.0 + 100.0)) < 1e-9


def test_shared_prefix_work_counts_the_prefix_once():
    """8 decode queries on a 943716-token shared prefix: the prefix's pooled
    keys are streamed once (8 sharing queries fit one 16-query tile), each
    sequence's own blocks once per sequence."""
    import dataclasses
    from block_sparse_attention_22_b200 import synth
    wl = synth.make_workload("shared_prefix_1m")
    P = wl.prefix[0][1]
    own = ((1 << 20) - 1) // 4 - P
    w = bench.algorithmic_work(wl)
    assert w["index"]["khat_bytes"] == (P + 8 * own) * 128 * 2
    alone = bench.algorithmic_work(dataclasses.replace(wl, prefix=[]))
    assert alone["index"]["khat_bytes"] == 8 * (((1 << 20) - 1) // 4) * 128 * 2
