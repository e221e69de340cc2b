"""The seeded input generator: the drifting-query (locality) input.

The AR(1) recursion is evaluated block by block in synth; these checks pin it
to the recursion written out step by step, to its stationary statistics, and
check that workloads without drift draw exactly the inputs they drew before
(drift only transforms the indexer queries and weights, after every tensor is
drawn from the same generator stream).
"""
import math

import torch

from block_sparse_attention_22_b200 import synth


def test_block_evaluation_equals_the_stepwise_recursion():
    g = torch.Generator().manual_seed(3)
    x = torch.randn(700, 5, generator=g)            # 700: two full blocks of 256 and a ragged one
    rho, innov = 0.97, math.sqrt(1 - 0.97 ** 2)
    ref = x.clone().double()
    for t in range(1, ref.shape[0]):
        ref[t] = rho * ref[t - 1] + innov * x[t].double()
    y = x.clone()
    synth._ar1_(y, rho, innov)
    assert torch.allclose(y.double(), ref, atol=1e-5, rtol=1e-5)
    assert torch.equal(y[0], x[0])


def test_drifting_queries_are_stationary_with_the_stated_correlation():
    wl = synth.make_workload("prefill_8k", n=4000, n_seqs=1, drift=0.99)
    x = synth.make_inputs(wl)
    q = x["q_idx"].float().reshape(4000, -1)
    assert abs(q.mean().item()) < 0.05
    assert abs(q.std().item() - 1.0) < 0.05
    for lag in (1, 10, 50):
        c = ((q[lag:] * q[:-lag]).sum() / (q * q).sum()).item()
        assert abs(c - 0.99 ** lag) < 0.03, (lag, c)
    w = x["w"]
    assert (w > 0).all() and (w < 1).all()
    assert abs(w.mean().item() - 0.5) < 0.05


def test_drift_leaves_every_other_tensor_and_the_default_inputs_unchanged():
    plain = synth.make_inputs(synth.make_workload("prefill_8k", n=600, n_seqs=2))
    drift = synth.make_inputs(synth.make_workload("prefill_8k", n=600, n_seqs=2, drift=0.9))
    for k in ("q", "k", "v"):
        assert torch.equal(plain[k], drift[k]), k
    assert not torch.equal(plain["q_idx"], drift["q_idx"])
    # each segment drifts on its own: its first token keeps its draw
    assert torch.equal(plain["q_idx"][0], drift["q_idx"][0])
    assert torch.equal(plain["q_idx"][600], drift["q_idx"][600])
    local = synth.make_workload("prefill_128k_local")
    assert local.drift == 0.99 and synth.make_workload("prefill_128k").drift == 0.0
    assert [s.q_len for s in local.segments] == [131072]


def test_mixed_tail_variant_puts_the_chunk_at_the_end_of_its_sequence():
    tail = synth.make_workload("mixed_1m_tail")
    base = synth.make_workload("mixed_1m")
    assert [(s.slot, s.pos0, s.q_len) for s in tail.segments[:8]] == \
        [(s.slot, s.pos0, s.q_len) for s in base.segments[:8]]
    chunk = tail.segments[8]
    assert (chunk.pos0, chunk.q_len) == ((1 << 20) - 4096, 4096)
    assert tail.fill[8] == 1 << 20 and tail.cached_blocks[8] == chunk.pos0 // 4
    assert (base.segments[8].pos0, base.fill[8]) == (942080, 946176)
