"""Backward of the sparse attention (qsa_sparse_attn_bwd) against the oracle.

The GPU forward (qsa_forward) provides o, lse and the selection; the GPU
backward then takes a seeded upstream gradient dout.  The oracle computes the
gradients of sum(dout * o) over the same kept tokens (qsa_ref_attend_bwd,
pinned against finite differences of the forward oracle), accumulating the
key gradients over every query of the batch.

Acceptance (from the arithmetic): the GPU recomputes probabilities from the
forward's fp32 lse and takes delta = dout . o from the forward's output, in
fp32 with fp32 atomic accumulation of dk/dv; the oracle works in fp64 from
the same rounded inputs.  fp32 I/O: max |err| <= 1e-4 * max |ref|; bf16 I/O
(o rounded to bf16 feeds delta): max |err| <= 1e-2 * max |ref| and mean
|err| <= 1e-3 * max |ref|."""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth
from qsa_testlib import gpu_forward, gpu_prepare_cache, segments_of, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": (1e-4, 1e-5), "bf16": (1e-2, 1e-3)}


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(name, got, ref, dtype):
    mx, mean = TOL[dtype]
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), name
    assert err.max() <= mx * scale, (name, "max", float(err.max()), scale)
    assert err.mean() <= mean * scale, (name, "mean", float(err.mean()), scale)


@pytest.mark.parametrize("name,over", [
    ("tiny_fp32", {}),
    ("prefill_8k", dict(n=600, n_seqs=1)),
    ("prefill_8k", dict(n=1200, n_seqs=2)),     # tensor-core path: several units per SM, 10 chunks
    ("decode_256k", dict(ctx=20001, n_seqs=3)),
])
def test_backward_matches_oracle_gradients(name, over):
    wl = synth.make_workload(name, **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    fwd = gpu_forward(wl, x)
    T = wl.n_tokens
    g = torch.Generator().manual_seed(31)
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
    slots = wl.token_slots().numpy()
    caches = {}
    dq_ref = np.zeros((T, sh.n_heads, sh.head_dim))
    for i in range(T):
        s = int(slots[i])
        if s not in caches:
            fill = wl.fill[s]
            k = to_np(x["k"][s, :, :fill])
            v = to_np(x["v"][s, :, :fill])
            caches[s] = [k, v, np.zeros(k.shape), np.zeros(v.shape)]
        k, v, dks, dvs = caches[s]
        dq_ref[i], caches[s][2], caches[s][3] = oracle.attend_bwd(
            rc, to_np(x["q"][i]), k, v, int(pos[i]), to_np(fwd.sel[i]).astype(np.int32), int(fwd.nsel[i]),
            to_np(dout[i]), dks, dvs)
    _check(name + " dq", to_np(dq), dq_ref, sh.dtype)
    for s, (k, v, dks, dvs) in caches.items():
        fill = k.shape[1]
        _check(name + f" dk slot {s}", to_np(dk[s, :, :fill]), dks, sh.dtype)
        _check(name + f" dv slot {s}", to_np(dv[s, :, :fill]), dvs, sh.dtype)
        # rows no query of the batch attends keep their zero
        assert torch.count_nonzero(dk[s, :, fill:]) == 0 and torch.count_nonzero(dv[s, :, fill:]) == 0


@pytest.mark.parametrize("name,over", [("tiny_fp32", {}), ("prefill_8k", dict(n=600, n_seqs=1))])
def test_backward_accumulates_key_gradients(name, over):
    wl = synth.make_workload(name, **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    fwd = gpu_forward(wl, x)
    T = wl.n_tokens
    dout = torch.ones((T, sh.n_heads, sh.head_dim), device="cuda").to(sh.torch_dtype)
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    dq = torch.empty((T, sh.n_heads, sh.head_dim), device="cuda")
    dk1 = torch.zeros(x["k"].shape, device="cuda")
    dv1 = torch.zeros(x["v"].shape, device="cuda")
    qsa.qsa_sparse_attn_bwd(cfg, cache, segs, T, x["q"], fwd.o, fwd.lse, dout, fwd.sel, fwd.nsel, dq, dk1, dv1)
    dk2, dv2 = dk1.clone(), dv1.clone()
    qsa.qsa_sparse_attn_bwd(cfg, cache, segs, T, x["q"], fwd.o, fwd.lse, dout, fwd.sel, fwd.nsel, dq, dk2, dv2)
    torch.cuda.synchronize()
    # the second call adds the same contributions in another atomic order: equal up to
    # fp32 rounding of sums of a few hundred terms, relative to each tensor's scale
    torch.testing.assert_close(dk2, 2 * dk1, rtol=0, atol=1e-5 * float(dk1.abs().max()))
    torch.testing.assert_close(dv2, 2 * dv1, rtol=0, atol=1e-5 * float(dv1.abs().max()))
