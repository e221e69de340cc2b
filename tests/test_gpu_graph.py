"""qsa_forward inside a CUDA graph.

The fused driver enqueues every step on one stream with no host
synchronisation (its kernels, and for few long selection rows one memset),
so a caller can capture a decode step once and replay it; a decode loop
replaces the inputs in place between replays.  Replays must give exactly the
results of direct calls on the same inputs, for a decode batch (few long
rows: the histogram selection and split-K attention), a prefill batch (many
rows) and the shared-prefix forward.
"""
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth
from qsa_testlib import gpu_prepare_cache, segments_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name,over", [
    ("decode_256k", dict(ctx=140001, n_seqs=3)),        # rows past 32K blocks: histogram selection
    ("prefill_8k", dict(n=1500, n_seqs=1)),
    ("shared_prefix_1m", dict(ctx=30001, n_seqs=3)),
])
def test_captured_forward_replays_like_direct_calls(name, over):
    wl = synth.make_workload(name, **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    T = wl.n_tokens
    pre = qsa.make_prefixes(wl.prefix) if wl.prefix else None
    op = qsa.QSA_OP_FORWARD_PREFIXED if pre is not None else qsa.QSA_OP_FORWARD
    ws = torch.empty(qsa.workspace_size(cfg, segs, T, op), dtype=torch.uint8, device="cuda")
    q, qi, w = x["q"].clone(), x["q_idx"].clone(), x["w"].clone()
    o = torch.empty((T, sh.n_heads, sh.head_dim), dtype=sh.torch_dtype, device="cuda")
    lse = torch.empty((T, sh.n_heads), device="cuda")
    sel = torch.empty((T, sh.budget_blocks), dtype=torch.int32, device="cuda")
    nsel = torch.empty((T,), dtype=torch.int32, device="cuda")

    def step():
        if pre is not None:
            qsa.qsa_forward_prefixed(cfg, cache, segs, pre, T, q, qi, w, o, lse, sel, nsel, ws)
        else:
            qsa.qsa_forward(cfg, cache, segs, T, q, qi, w, o, lse, sel, nsel, ws)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    g = torch.Generator(device="cuda").manual_seed(7)
    for it in range(2):                                  # two replays, new queries in place each time
        q.copy_(torch.randn(q.shape, generator=g, device="cuda").to(q.dtype))
        qi.copy_(torch.randn(qi.shape, generator=g, device="cuda").to(qi.dtype))
        graph.replay()
        torch.cuda.synchronize()
        got = (o.clone(), lse.clone(), sel.clone(), nsel.clone())
        step()
        torch.cuda.synchronize()
        assert torch.equal(got[2], sel) and torch.equal(got[3], nsel), it
        assert torch.equal(got[0], o) and torch.equal(got[1], lse), it
    assert qsa.device_status() == qsa.QSA_OK
