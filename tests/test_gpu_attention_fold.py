"""The attention's late fold of the last chunk's maximum, on the rescale path.

The tensor-core attention takes the per-head maximum over every chunk of a
unit but the last, writes the first P chunks with it, and folds the last
chunk's maximum in before the third; when that maximum exceeds the running
one by more than 8 (log2 units), O and the row sums so far are rescaled in
TMEM.  Kept blocks are in ascending order, so the block just before a query's
own block lands in the query's last chunk; planting a key there that matches
the query (main K rows = the query's head-0 row: score |q|^2 tau ~ 16, against
~3 for random keys) forces the rescale for head 0 of each group.  The block is
made the query's best indexer candidate the same way synth plants needles
(indexer key rows = sum_h w_h q_idx_h with the rotary dims zeroed), so it is
selected.  Design report QSA item and Miles docs section 1 define the
selection and the attention the oracle computes.
"""
import pytest
import torch

from block_sparse_attention_22_b200 import synth

from qsa_testlib import compare_forward, gpu_forward

pytestmark = pytest.mark.gpu


def test_last_chunk_dominant_keys_take_the_rescale_path():
    wl = synth.make_workload("prefill_8k", n=3000, n_seqs=1)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    rho = sh.rope_dims
    targets = [2301, 2502, 2703, 2904, 2999]
    for t in targets:
        b = t // sh.r - 1                          # the block before the own block
        u = (x["w"][t].float().unsqueeze(1) * x["q_idx"][t].float()).sum(0)
        u[:rho] = 0
        rows = torch.arange(b * sh.r, (b + 1) * sh.r, device="cuda")
        x["k_idx"][0, rows] = (4.0 * u).to(x["k_idx"].dtype)
        for g in range(sh.n_groups):
            x["k"][0, g, rows] = x["q"][t, g * (sh.n_heads // sh.n_groups)].unsqueeze(0).expand(sh.r, -1)
    run = gpu_forward(wl, x)
    sel = run.sel.cpu()
    for t in targets:
        assert t // sh.r - 1 in sel[t, 480:511].tolist(), t     # kept, in the last chunk
    res = compare_forward(wl, x, run, targets + list(range(2048, 3000, 37)))
    assert res["n"] >= len(targets)
