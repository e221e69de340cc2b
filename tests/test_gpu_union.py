"""Union-tile attention (qsa_sparse_attn_fwd_union) against the oracle.

The union path gathers, per tile of neighbouring query tokens, the union of
their kept blocks once and masks each query row to its own selection and
causal limit, so every query must get exactly the attention the oracle
computes over its own kept tokens (Miles docs "Qwen3.8-Flash-Next",
section 1).  Cases: inputs with and without locality (drifting indexer
queries), ragged tiles at segment ends, decode and speculative-decode
segments (tiles of 1 and 4 queries), tiles whose union spans the whole
context (hundreds of 64-key chunks, so the running maximum moves and O is
rescaled), layer shapes that fill 128, 96, 64 and 32 query rows of a tile,
hand-made selections, and more than 128 segments (several launches sharing
one workspace).  Tolerances are the forward's (bf16 I/O).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth

from qsa_testlib import check_outputs, gpu_forward, gpu_prepare_cache, sample_tokens, segments_of, to_np

pytestmark = pytest.mark.gpu


def union_attn(wl, x, sel, nsel):
    sh = wl.shape
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    T = wl.n_tokens
    o = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), dtype=sh.torch_dtype, device="cuda")
    lse = torch.full((T, sh.n_heads), float("nan"), device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_ATTN_UNION)), dtype=torch.uint8,
                     device="cuda")
    n0 = qsa.launch_count()
    qsa.qsa_sparse_attn_fwd_union(cfg, cache, segs, T, x["q"], sel, nsel, o, lse, ws)
    torch.cuda.synchronize()
    qsa.qsa_device_status()
    # per launch table of at most 128 non-empty segments: the union lists, then the attention
    tables = -(-sum(1 for s in wl.segments if s.q_len > 0) // 128)
    assert qsa.launch_count() - n0 == 2 * tables
    return o, lse


def oracle_check(wl, x, sel, nsel, o, lse, tokens, what):
    rc = oracle.config_from_shape(wl.shape)
    pos = wl.token_positions().numpy()
    slots = wl.token_slots().numpy()
    o_ref, lse_ref = [], []
    for i in tokens:
        s = int(slots[i])
        fill = wl.fill[s]
        r, l = oracle.attend(rc, to_np(x["q"][i]), to_np(x["k"][s, :, :fill]), to_np(x["v"][s, :, :fill]),
                             int(pos[i]), to_np(sel[i]).astype(np.int32), int(nsel[i]))
        o_ref.append(r)
        lse_ref.append(l)
    check_outputs(to_np(o[tokens]), np.stack(o_ref), to_np(lse[tokens]), np.stack(lse_ref), wl.shape.dtype, what)


def union_sizes(wl, sel, nsel, mq):
    """Union length of every tile, from the selection on the host."""
    sel, nsel = sel.cpu().numpy(), nsel.cpu().numpy()
    out = []
    for off, seg in zip(wl.token_offsets(), wl.segments):
        for q0 in range(0, seg.q_len, mq):
            rows = range(off + q0, off + min(seg.q_len, q0 + mq))
            out.append(len(set(int(b) for i in rows for b in sel[i, :nsel[i]])))
    return np.array(out)


CASES = [
    ("prefill_8k", dict(n=3000, n_seqs=2, drift=0.99), 7),     # locality: tiles share most blocks
    ("prefill_8k", dict(n=1237, n_seqs=2), 5),                 # no locality; 1237 = 123 tiles of 10 + 7
    ("chunk_128k", dict(n=24000, chunk=203), 1),               # unions of ~5000 blocks (80 chunks)
    ("decode_256k", dict(ctx=20001, n_seqs=3), 1),             # one-query tiles
    ("spec_decode_1m", dict(ctx=30001, n_seqs=2), 1),          # four-query tiles near the end of a long cache
]


@pytest.mark.parametrize("name,over,every", CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(CASES)])
def test_union_attention_matches_the_oracle(name, over, every):
    wl = synth.make_workload(name, **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    o, lse = union_attn(wl, x, run.sel, run.nsel)
    oracle_check(wl, x, run.sel, run.nsel, o, lse, sample_tokens(wl, every), name)
    # every token against the per-query tensor-core path (both bf16; P rounded against other maxima)
    check_outputs(to_np(o), to_np(run.o).astype(np.float64), to_np(lse), to_np(run.lse).astype(np.float64),
                  "bf16", name + " vs per-query")


def test_locality_shrinks_the_unions():
    """With drifting indexer queries, a tile of 10 neighbours keeps far fewer
    distinct blocks than 10 x 512; with independent queries it does not."""
    sizes = {}
    for drift in (0.0, 0.99):
        wl = synth.make_workload("chunk_128k", n=60000, chunk=200)
        wl.drift = drift
        x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
        run = gpu_forward(wl, x)
        sizes[drift] = union_sizes(wl, run.sel, run.nsel, 10).mean()
        o, lse = union_attn(wl, x, run.sel, run.nsel)
        oracle_check(wl, x, run.sel, run.nsel, o, lse, sample_tokens(wl, 9), f"drift {drift}")
    assert sizes[0.0] > 3800
    assert sizes[0.99] < 0.4 * sizes[0.0], sizes


@pytest.mark.parametrize("shape", [
    dict(n_heads=32, n_groups=2),      # 16 heads per group: 8 queries fill 128 rows
    dict(n_heads=8, n_groups=4),       # 2 heads per group: 32 queries, 64 rows
    dict(n_heads=16, n_groups=16),     # 1 head per group: 32 queries, 32 rows
    dict(idx_dim=64),                  # default heads, 64-dim indexer
], ids=lambda d: "-".join(f"{k}{v}" for k, v in d.items()))
def test_union_attention_on_layer_shapes(shape):
    wl = synth.make_workload("prefill_8k", n=2300, n_seqs=1, shape=shape, drift=0.99)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    o, lse = union_attn(wl, x, run.sel, run.nsel)
    oracle_check(wl, x, run.sel, run.nsel, o, lse, sample_tokens(wl, 13), str(shape))


def test_tiles_with_hand_made_selections():
    """Members whose selections are disjoint, nested, or short (early
    positions), and a member that keeps only its own block: each row must see
    exactly its own keys."""
    wl = synth.make_workload("prefill_8k", n=40, n_seqs=1)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    T, S = wl.n_tokens, wl.shape.budget_blocks
    sel = torch.full((T, S), -1, dtype=torch.int32)
    nsel = torch.zeros(T, dtype=torch.int32)
    g = torch.Generator().manual_seed(5)
    for t in range(T):
        own = t // 4
        if t % 3 == 0:
            keep = [own]
        else:
            pool = torch.randperm(own, generator=g)[: min(own, 1 + t % 5)].tolist() if own else []
            keep = sorted(pool) + [own]
        sel[t, :len(keep)] = torch.tensor(keep, dtype=torch.int32)
        nsel[t] = len(keep)
    sel, nsel = sel.cuda(), nsel.cuda()
    o, lse = union_attn(wl, x, sel, nsel)
    oracle_check(wl, x, sel, nsel, o, lse, list(range(T)), "hand-made")


def test_union_attention_over_several_launch_tables():
    """More than 128 segments (several launches sharing one workspace through
    their tile offsets), out of slot order, with 1- to 3-query segments."""
    sh = synth.Shape()
    n_seq, ctx = 150, 700
    wl = synth.Workload("many", sh, [], n_seq, 1024, [ctx] * n_seq, [0] * n_seq, [], 11)
    wl.segments = [synth.Segment(s, ctx - 3 - (s % 3), 1 + (s % 3)) for s in reversed(range(n_seq))]
    wl.cached_blocks = [sg.pos0 // 4 for sg in sorted(wl.segments, key=lambda sg: sg.slot)]
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    o, lse = union_attn(wl, x, run.sel, run.nsel)
    oracle_check(wl, x, run.sel, run.nsel, o, lse, list(range(0, wl.n_tokens, 7)), "many segments")
    check_outputs(to_np(o), to_np(run.o).astype(np.float64), to_np(lse), to_np(run.lse).astype(np.float64),
                  "bf16", "many segments vs per-query")
