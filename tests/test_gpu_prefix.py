"""Decode sequences that share one cached prefix (qsa_forward_prefixed).

The release article's section "GDN+QSA" quotes the 1M-context throughput at
a 90 % prefix-cache hit: many requests on one cached prefix.  Here the
prefix's indexer keys, pooled keys, K and V live once, in their own cache
slot; each sequence's suffix lives in its slot.  As the oracle sees it, every
sequence is still one whole cache (its prefix rows, then its suffix rows),
and the forward pass of each query must be exactly the method on that cache:

  * selections exact (outside the tie band) and outputs within the forward's
    bf16 tolerances, against the oracle on the whole caches;
  * the same selections and outputs, bit for bit, as qsa_forward on a copy of
    the batch in which every sequence's whole cache sits in its own slot (the
    shared prefix's scores come from the same tensor-core products, whatever
    the tile of queries);
  * the sequences' own slots hold zeros below the prefix's end, so a kernel
    that read a prefix block from the wrong slot would change the result.
Cases: decode (one query per sequence), speculative decode (4 consecutive
queries per sequence; 20 queries sharing, more than one 16-query tile), two
prefixes of different lengths and a sequence that shares nothing in one
batch, a prefix that ends inside a 128-block tile, the full 1M-context
workload on sampled sequences, and the argument checks.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth
from qsa_testlib import compare_forward, gpu_forward, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def unshared_copy(wl, x):
    """The same sequences with every whole cache in its own slot (no prefix)."""
    n = len(wl.segments)
    fills = [wl.fill[s.slot] for s in wl.segments]
    cap = wl.n_cap
    sh = wl.shape
    kx = torch.zeros((n, cap, sh.idx_dim), dtype=x["k_idx"].dtype, device=x["k_idx"].device)
    k = torch.zeros((n, sh.n_groups, cap, sh.head_dim), dtype=x["k"].dtype, device=x["k"].device)
    v = torch.zeros_like(k)
    for i, seg in enumerate(wl.segments):
        a, b, c = synth.sequence_cache(wl, x, seg.slot, fills[i])
        kx[i, :fills[i]] = a
        k[i, :, :fills[i]] = b
        v[i, :, :fills[i]] = c
    segs = [synth.Segment(i, s.pos0, s.q_len) for i, s in enumerate(wl.segments)]
    cached = [wl.cached_blocks[s.slot] for s in wl.segments]
    wl2 = synth.Workload(wl.name + "-unshared", sh, segs, n, cap, fills, cached, [], wl.seed)
    x2 = {"q": x["q"], "q_idx": x["q_idx"], "w": x["w"], "k_idx": kx, "k": k, "v": v}
    return wl2, x2


@pytest.mark.parametrize("over", [
    dict(ctx=30001, n_seqs=3),                   # decode; the prefix (6750 blocks) ends inside a 128-block tile
    dict(ctx=20004, n_seqs=5, q_len=4),          # speculative decode: 20 sharing queries, two 16-query tiles
    dict(ctx=40001, n_seqs=2, prefix=32768),     # a prefix that ends on a tile boundary (8192 blocks)
])
def test_shared_prefix_matches_oracle_and_unshared_forward(over):
    wl = synth.make_workload("shared_prefix_1m", **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    res = compare_forward(wl, x, run, min_exact=1.0)
    assert res["verdicts"]["band"] == 0
    wl2, x2 = unshared_copy(wl, x)
    ref = gpu_forward(wl2, x2)
    assert torch.equal(run.nsel, ref.nsel)
    assert torch.equal(run.sel, ref.sel)
    assert torch.equal(run.o, ref.o)
    assert torch.equal(run.lse, ref.lse)


def test_two_prefixes_and_an_unshared_sequence_in_one_batch():
    """Sequences 0-1 share prefix A (slot 5, 5000 blocks), sequences 2-3
    prefix B (slot 6, 3000 blocks), sequence 4 shares nothing; decode
    queries at different positions."""
    sh = synth.Shape()
    ctxs = [24001, 22003, 25000, 21999, 18001]
    pA, pB = 5000, 3000
    prefix = [(5, pA), (5, pA), (6, pB), (6, pB), (0, 0)]
    segs = [synth.Segment(i, c - 1, 1) for i, c in enumerate(ctxs)]
    fills = ctxs + [pA * 4, pB * 4]
    starts = [p * 4 for _, p in prefix] + [0, 0]
    cached = [(c - 1) // 4 for c in ctxs] + [pA, pB]
    g = torch.Generator().manual_seed(3)
    needles = []
    for i, c in enumerate(ctxs):
        for b in torch.randperm(min(pA, pB), generator=g)[:2].tolist():
            needles.append((i, c - 1, b))
    wl = synth.Workload("two-prefixes", sh, segs, 7, 25004, fills, cached, needles, 21, prefix=prefix,
                        start=starts)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, min_exact=1.0)
    wl2, x2 = unshared_copy(wl, x)
    ref = gpu_forward(wl2, x2)
    assert torch.equal(run.sel, ref.sel)
    assert torch.equal(run.o, ref.o)


@pytest.mark.slow
def test_shared_prefix_full_size_sampled():
    """The 1M-context workload: 8 sequences on a 943716-token shared prefix
    (two sequences compared with the oracle), and invariants on all."""
    wl = synth.make_workload("shared_prefix_1m")
    x = synth.make_inputs(wl, device="cuda")
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, [0, 7])
    pos = wl.token_positions()
    assert torch.equal(run.nsel.cpu(), torch.clamp(pos // 4 + 1, max=wl.shape.budget_blocks).int())
    # the needles of every sequence, in its prefix and in its suffix, are kept
    sel = run.sel.cpu().numpy()
    for (slot, t, b) in wl.needles:
        assert b in set(sel[slot].tolist()), (slot, b)


def test_prefix_argument_checks():
    wl = synth.make_workload("shared_prefix_1m", ctx=8001, n_seqs=2)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    cfg = qsa.make_config(sh)
    khat = torch.zeros((wl.n_slots, wl.n_cap // 4, sh.idx_dim), dtype=sh.torch_dtype, device="cuda")
    cache = qsa.make_cache(x["k_idx"], khat, x["k"], x["v"])
    segs = qsa.make_segments([(i, s.q_len, s.pos0, s.slot) for i, s in enumerate(wl.segments)])
    T = wl.n_tokens
    o = torch.empty((T, sh.n_heads, sh.head_dim), dtype=sh.torch_dtype, device="cuda")
    ws = torch.empty(qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_FORWARD_PREFIXED), dtype=torch.uint8, device="cuda")
    P = wl.prefix[0][1]
    bad = [
        [(2, P), (9, P)],              # prefix slot out of range
        [(2, P), (2, -1)],             # negative length
        [(2, P), (2, 2001)],           # prefix past the queries (8000 < 2001 * 4)
    ]
    for pre in bad:
        with pytest.raises(qsa.QSAError) as e:
            qsa.qsa_forward_prefixed(cfg, cache, segs, qsa.make_prefixes(pre), T, x["q"], x["q_idx"], x["w"], o,
                                     workspace=ws)
        assert e.value.status == qsa.QSA_ERR_INVALID_ARG, pre
    n0 = qsa.launch_count()
    long_seg = qsa.make_segments([(0, 16, 7984, 0), (16, 1, 8000, 1)])     # 16 queries on a prefix: unsupported
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_forward_prefixed(cfg, cache, long_seg, qsa.make_prefixes(wl.prefix), 17, x["q"], x["q_idx"],
                                 x["w"], o, workspace=ws)
    assert e.value.status == qsa.QSA_ERR_UNSUPPORTED
    assert qsa.launch_count() == n0
