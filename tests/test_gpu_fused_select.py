"""Fused prefill selection (qsa_forward_lowmem) on rows long enough for its
sampled threshold.

For bf16 segments of 16 or more queries, qsa_forward_lowmem scores an evenly spaced
sample of the pooled blocks, takes a threshold per query from it, keeps only
the (score, block) pairs at or above it in a second scoring pass, and selects
exactly among them; a query whose list holds fewer than S-1 or more than 4096
pairs is selected exactly over all of its blocks with recomputed scores.
Rows of more than 4096 candidate blocks (contexts past 16K tokens) take the
sampled threshold, so these cases use a 1024-query chunk at 23.5K-24.5K
tokens of a cached prefix.  Every selection is compared with the oracle's
(design report, QSA item: top-k over micro-block scores; ties toward the
lower block index), or with a closed form.
"""
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth

from qsa_testlib import compare_forward, gpu_forward, sample_tokens

pytestmark = pytest.mark.gpu


def _chunk():
    return synth.make_workload("chunk_128k", n=24576, chunk=1024)


def test_sampled_threshold_rows_match_oracle():
    wl = _chunk()
    x = synth.make_inputs(wl, device="cuda")
    qsa.select_fallbacks()                          # clear the counter
    run = gpu_forward(wl, x, lowmem=True)
    # on random inputs every list holds between S-1 and 4096 pairs
    assert qsa.select_fallbacks() == 0
    res = compare_forward(wl, x, run, sample_tokens(wl, 13))
    assert res["n"] > 80


def test_all_zero_scores_overflow_into_the_exact_fallback():
    """w = 0 makes every score of a query exactly 0: its threshold admits all
    of its ~6K blocks, more than a list holds, and the exact fallback keeps
    blocks 0..S-2 (ties toward the lower index) plus the own block."""
    wl = _chunk()
    x = synth.make_inputs(wl, device="cuda")
    zero = list(range(0, wl.n_tokens, 5))
    x["w"][zero] = 0.0
    qsa.select_fallbacks()
    run = gpu_forward(wl, x, lowmem=True)
    assert qsa.select_fallbacks() == len(zero)
    S = wl.shape.budget_blocks
    pos = wl.token_positions()
    sel = run.sel.cpu()
    nsel = run.nsel.cpu()
    for i in zero:
        bt = int(pos[i]) // wl.shape.r
        assert int(nsel[i]) == S
        assert sel[i].tolist() == list(range(S - 1)) + [bt], i
    others = [i for i in sample_tokens(wl, 13) if i % 5 != 0]
    compare_forward(wl, x, run, others)


def test_dominant_sampled_blocks_underflow_into_the_exact_fallback():
    """Indexer keys of every 16th block scaled by 8: those blocks score far
    above the rest, so the threshold taken from the sample (which holds only
    them) admits ~100 pairs, fewer than S-1, and the exact fallback selects
    over all blocks.  The answer (all of the scaled blocks and the best of
    the others) is checked against the oracle."""
    wl = _chunk()
    x = synth.make_inputs(wl, device="cuda")
    nb = wl.fill[0] // wl.shape.r
    blocks = torch.arange(0, nb, 16)
    rows = (blocks.unsqueeze(1) * wl.shape.r + torch.arange(wl.shape.r)).flatten().cuda()
    x["k_idx"][0, rows] *= 8                     # a power of two: exact in bf16
    qsa.select_fallbacks()
    run = gpu_forward(wl, x, lowmem=True)
    assert qsa.select_fallbacks() > wl.n_tokens // 2
    compare_forward(wl, x, run, sample_tokens(wl, 13))
    # most of the scaled blocks are kept (a scaled block whose four head dots
    # are all negative scores 0 and may lose)
    sel = run.sel.cpu()
    pos = wl.token_positions()
    S = wl.shape.budget_blocks
    for i in range(0, wl.n_tokens, 97):
        bt = int(pos[i]) // wl.shape.r
        kept = set(sel[i, :S - 1].tolist())
        scaled = list(range(0, bt, 16))
        assert 2 * sum(b in kept for b in scaled) > len(scaled), i


@pytest.mark.parametrize("name,over,every", [
    ("prefill_8k", dict(n=2500, n_seqs=2), 7),
    ("mixed_1m", dict(ctx=16384, n_decode=3, chunk=300, chunk_pos0=5001), 3),
    ("prefill_128k", {}, 1021),
])
def test_lowmem_forward_matches_oracle(name, over, every):
    wl = synth.make_workload(name, **over)
    x = synth.make_inputs(wl, device="cuda")
    run = gpu_forward(wl, x, lowmem=True)
    compare_forward(wl, x, run, sample_tokens(wl, every))


def test_lowmem_selection_equals_the_score_matrix_path():
    """Both paths take every score from the same MMA and epilogue arithmetic
    and select exactly, so without a fallback their selections and outputs
    are identical."""
    wl = _chunk()
    x = synth.make_inputs(wl, device="cuda")
    ref = gpu_forward(wl, x)
    qsa.select_fallbacks()
    low = gpu_forward(wl, x, lowmem=True)
    assert qsa.select_fallbacks() == 0
    assert torch.equal(ref.nsel, low.nsel)
    assert torch.equal(ref.sel, low.sel)
    assert torch.equal(ref.o, low.o)
    assert torch.equal(ref.lse, low.lse)
