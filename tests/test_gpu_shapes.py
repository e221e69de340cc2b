"""Forward and backward parity on layer shapes other than the default.

The library takes any n_q_heads / n_kv_groups <= 16 heads per group and an
indexer dim of 64 or 128 (include/qsa.h).  The default layer (24 heads in 2
groups, indexer dim 128; Miles docs "Qwen3.8-Flash-Next", section 1) fills 12
of the 16 head rows of a tensor-core tile; these cases fill all 16, a few, one,
four groups, and the 64-dim indexer (a single 64-dim slab, 16 rotated dims)
on the bf16 tensor-core path, each on a ragged prefill against the oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth

from qsa_testlib import compare_forward, gpu_forward, gpu_prepare_cache, sample_tokens, segments_of, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    dict(n_heads=32, n_groups=2),                 # 16 heads per group: a full tile
    dict(n_heads=8, n_groups=4),                  # 2 heads per group, 4 groups
    dict(n_heads=12, n_groups=1),                 # one group
    dict(n_heads=16, n_groups=16),                # 1 head per group (MHA)
    dict(idx_dim=64),                             # 64-dim indexer in bf16
]


def _workload(shape):
    return synth.make_workload("prefill_8k", n=2300, n_seqs=1, shape=shape)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda d: "-".join(f"{k}{v}" for k, v in d.items()))
def test_forward_parity_on_layer_shapes(shape):
    wl = _workload(shape)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    res = compare_forward(wl, x, run, sample_tokens(wl, 11))
    assert res["n"] > 100


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda d: "-".join(f"{k}{v}" for k, v in d.items()))
def test_backward_parity_on_layer_shapes(shape):
    wl = synth.make_workload("prefill_8k", n=700, n_seqs=1, shape=shape)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    fwd = gpu_forward(wl, x)
    T = wl.n_tokens
    g = torch.Generator().manual_seed(37)
    dout = torch.randn((T, sh.n_heads, sh.head_dim), generator=g).to(sh.torch_dtype).cuda()
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    dq = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), device="cuda")
    dk = torch.zeros(x["k"].shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(x["v"].shape, dtype=torch.float32, device="cuda")
    qsa.qsa_sparse_attn_bwd(cfg, cache, segs, T, x["q"], fwd.o, fwd.lse, dout, fwd.sel, fwd.nsel, dq, dk, dv)
    torch.cuda.synchronize()
    qsa.qsa_device_status()
    rc = oracle.config_from_shape(sh)
    pos = wl.token_positions().numpy()
    fill = wl.fill[0]
    k = to_np(x["k"][0, :, :fill])
    v = to_np(x["v"][0, :, :fill])
    dks, dvs = np.zeros(k.shape), np.zeros(v.shape)
    dq_ref = np.zeros((T, sh.n_heads, sh.head_dim))
    for i in range(T):
        dq_ref[i], dks, dvs = oracle.attend_bwd(rc, to_np(x["q"][i]), k, v, int(pos[i]),
                                                to_np(fwd.sel[i]).astype(np.int32), int(fwd.nsel[i]),
                                                to_np(dout[i]), dks, dvs)
    for name, got, ref in (("dq", to_np(dq), dq_ref), ("dk", to_np(dk[0, :, :fill]), dks),
                           ("dv", to_np(dv[0, :, :fill]), dvs)):
        scale = max(float(np.abs(ref).max()), 1e-30)
        err = np.abs(got.astype(np.float64) - ref)
        assert np.isfinite(got).all(), name
        assert err.max() <= 1e-2 * scale, (name, float(err.max()), scale)
        assert err.mean() <= 1e-3 * scale, (name, float(err.mean()), scale)


@pytest.mark.parametrize("name,shape", [
    ("decode_256k", dict(n_heads=32, n_groups=2)),
    ("decode_256k", dict(idx_dim=64)),
    ("spec_decode_1m", dict(n_heads=8, n_groups=4)),
], ids=lambda x: x if isinstance(x, str) else "-".join(f"{k}{v}" for k, v in x.items()))
def test_decode_parity_on_layer_shapes(name, shape):
    """Decode-like segments: 4-query index tiles, the few-rows selection and
    split-K attention with its combine, on the same shape variants."""
    wl = synth.make_workload(name, ctx=20001, n_seqs=3, shape=shape)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    run = gpu_forward(wl, x)
    res = compare_forward(wl, x, run, range(wl.n_tokens))
    assert res["n"] == wl.n_tokens
