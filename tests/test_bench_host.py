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
