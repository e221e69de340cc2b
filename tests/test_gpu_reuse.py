"""Selection reuse across layers (multi-token-prediction style): a second
QSA layer attends with the selection a first layer's qsa_forward produced,
skipping its own pooling, scoring and selection.  The reuse path is
qsa_sparse_attn_fwd fed with the first layer's sel/nsel; the oracle attends
the second layer's q/K/V over exactly that selection."""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth
from qsa_testlib import check_outputs, gpu_forward, gpu_prepare_cache, sample_tokens, segments_of, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name,over,every", [
    ("prefill_8k", dict(n=3000, n_seqs=2), 11),
    ("decode_256k", dict(ctx=20001, n_seqs=3), 1),
])
def test_second_layer_attends_with_the_first_layers_selection(name, over, every):
    wl = synth.make_workload(name, **over)
    x1 = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    wl2 = synth.make_workload(name, seed=77, **over)          # the second layer: other q/K/V
    x2 = {k: v.cuda() for k, v in synth.make_inputs(wl2).items()}
    sh = wl.shape
    run1 = gpu_forward(wl, x1)                                 # layer 1: full forward, keeps sel/nsel
    cfg, cache2, _ = gpu_prepare_cache(wl2, x2)
    segs = segments_of(wl)
    T = wl.n_tokens
    o = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), dtype=sh.torch_dtype, device="cuda")
    lse = torch.empty((T, sh.n_heads), device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_ATTN)), dtype=torch.uint8, device="cuda")
    n0 = qsa.launch_count()
    qsa.qsa_sparse_attn_fwd(cfg, cache2, segs, T, x2["q"], run1.sel, run1.nsel, o, lse, ws)
    torch.cuda.synchronize()
    assert qsa.launch_count() - n0 <= 2                        # attention (+ split-K combine): no index/select
    rc = oracle.config_from_shape(sh)
    pos = wl.token_positions().numpy()
    slots = wl.token_slots().numpy()
    tokens = sample_tokens(wl, every)
    o_ref, lse_ref = [], []
    for i in tokens:
        s = int(slots[i])
        fill = wl.fill[s]
        r, l = oracle.attend(rc, to_np(x2["q"][i]), to_np(x2["k"][s, :, :fill]), to_np(x2["v"][s, :, :fill]),
                             int(pos[i]), to_np(run1.sel[i]).astype(np.int32), int(run1.nsel[i]))
        o_ref.append(r)
        lse_ref.append(l)
    check_outputs(to_np(o[tokens]), np.stack(o_ref), to_np(lse[tokens]), np.stack(lse_ref), sh.dtype, name)
