"""Caller-supplied selections with entries out of range.

The attention entry points take `sel`/`nsel` from the caller (a layer that
reuses another layer's selection passes them in, Miles docs
"Qwen3.8-Flash-Next", section 1: selection rows are built outside the
attention kernel).  Every kept block goes through one bounds check on the
device: an entry outside [0, n_cap/r) other than the -1 padding is skipped
(it contributes no key), recorded in the device error word, and reported by
qsa_device_status() as QSA_ERR_BAD_INDEX.  A count above the budget is
clamped to the row.  The rest of each row must be attended exactly as the
oracle attends the valid entries alone.

The bad entries are planted on the host in a copy of a real selection; the
kernels read only the rows' in-bounds words and never dereference a
rejected entry, so nothing here can fault.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth
from qsa_testlib import check_outputs, gpu_forward, gpu_prepare_cache, segments_of, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def plant_bad_entries(sel, nsel, n_blocks, S):
    """Replace one non-own entry of every third row by an out-of-range block
    (n_blocks, n_blocks + 3, 2^30, -2, -2^30 in turn) and give every seventh
    row a count above the budget.  Returns the corrupted rows and, per row,
    the valid entries the oracle attends."""
    sel = sel.cpu().clone()
    nsel = nsel.cpu().clone()
    bad_values = [n_blocks, n_blocks + 3, 1 << 30, -2, -(1 << 30)]
    valid, planted = [], 0
    for i in range(sel.shape[0]):
        n = int(nsel[i])
        row = sel[i, :n].tolist()
        valid.append(np.array(row, dtype=np.int32))
        if i % 3 == 0 and n > 1:
            sel[i, (7 * i) % (n - 1)] = bad_values[planted % len(bad_values)]
            planted += 1
            keep = [b for j, b in enumerate(row) if j != (7 * i) % (n - 1)]
            valid[-1] = np.array(keep, dtype=np.int32)
        if i % 7 == 1:
            nsel[i] = S + 100             # clamped to the row; the -1 padding is skipped silently
    assert planted > 0
    return sel.cuda(), nsel.cuda(), valid


def oracle_on_valid(wl, x, valid, tokens):
    rc = oracle.config_from_shape(wl.shape)
    pos = wl.token_positions().numpy()
    slots = wl.token_slots().numpy()
    o_ref, lse_ref = [], []
    for i in tokens:
        s = int(slots[i])
        fill = wl.fill[s]
        sel = np.full(wl.shape.budget_blocks, -1, np.int32)
        sel[:len(valid[i])] = valid[i]
        r, l = oracle.attend(rc, to_np(x["q"][i]), to_np(x["k"][s, :, :fill]), to_np(x["v"][s, :, :fill]),
                             int(pos[i]), sel, len(valid[i]))
        o_ref.append(r)
        lse_ref.append(l)
    return np.stack(o_ref), np.stack(lse_ref)


@pytest.mark.parametrize("name,over,union", [
    ("tiny_fp32", {}, False),                                 # CUDA-core attention (fp32 I/O)
    ("prefill_8k", dict(n=1500, n_seqs=1), False),            # tensor-core attention
    ("decode_256k", dict(ctx=20001, n_seqs=3), False),        # split rows, combined afterwards
    ("prefill_8k", dict(n=1500, n_seqs=1), True),             # union-tile attention
])
def test_out_of_range_entries_are_skipped_and_reported(name, over, union):
    wl = synth.make_workload(name, **over)
    x = {k: v.cuda() for k, v in synth.make_inputs(wl).items()}
    sh = wl.shape
    run = gpu_forward(wl, x)
    assert qsa.device_status() == qsa.QSA_OK                  # a clean forward records nothing
    sel, nsel, valid = plant_bad_entries(run.sel, run.nsel, wl.n_cap // sh.r, sh.budget_blocks)
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    T = wl.n_tokens
    o = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), dtype=sh.torch_dtype, device="cuda")
    lse = torch.full((T, sh.n_heads), float("nan"), device="cuda")
    op = qsa.QSA_OP_ATTN_UNION if union else qsa.QSA_OP_ATTN
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, op)), dtype=torch.uint8, device="cuda")
    attn = qsa.qsa_sparse_attn_fwd_union if union else qsa.qsa_sparse_attn_fwd
    attn(cfg, cache, segs, T, x["q"], sel, nsel, o, lse, ws)
    assert qsa.device_status() == qsa.QSA_ERR_BAD_INDEX
    assert qsa.device_status() == qsa.QSA_OK                  # read and cleared
    tokens = list(range(T)) if T <= 600 else list(range(0, T, 3)) + list(range(1, T, 7))
    tokens = sorted(set(tokens))
    o_ref, lse_ref = oracle_on_valid(wl, x, valid, tokens)
    check_outputs(to_np(o[tokens]), o_ref, to_np(lse[tokens]), lse_ref, sh.dtype, name)


def test_status_string_names_the_bad_index():
    assert "out of range" in qsa.status_string(qsa.QSA_ERR_BAD_INDEX)
