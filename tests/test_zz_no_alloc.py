"""qsa_select_topk_noalloc: the selection entry point for callers that cannot
allocate device memory (its few-long-rows scratch is a static device array in the
library).  It must give the same selection as qsa_select_topk with a caller
workspace, call after call.  Selections are integer results, so the
comparison is exact, as in the other selection tests.

This file is collected last on purpose: it is the only test that touches the
library's shared static scratch array.
"""
import ctypes

import pytest
import torch

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _rows(seed, lengths):
    g = torch.Generator().manual_seed(seed)
    rows = torch.randn((len(lengths), max(lengths)), generator=g).abs() * 5
    rows[:, ::7] = torch.randint(0, 3, rows[:, ::7].shape, generator=g).float()   # exact ties
    return rows.cuda()


def _noalloc(cfg, segs, T, scores, sel, nsel):
    arr, n = segs
    return qsa.get_lib().qsa_select_topk_noalloc(ctypes.byref(cfg), arr, n, T, scores.data_ptr(), scores.shape[1],
                                                 sel.data_ptr(), nsel.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream)


def test_noalloc_selection_matches_workspace_entry_point_on_consecutive_calls():
    sh = synth.Shape()
    cfg = qsa.make_config(sh)
    S = sh.budget_blocks
    # few long rows: their histograms, counters and candidate lists live in
    # the scratch (cleared at the start of every call); the short row keeps
    # every block
    lengths = [300001, 65535, 300, 40000, 524287]
    segs = qsa.make_segments([(i, 1, 4 * n + 3, 0) for i, n in enumerate(lengths)])
    T = len(lengths)
    assert qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT) > 0
    for call, seed in enumerate([1, 2]):
        scores = _rows(seed, lengths)
        sel_ref = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
        nsel_ref = torch.full((T,), -7, dtype=torch.int32, device="cuda")
        ws = torch.empty(qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT), dtype=torch.uint8, device="cuda")
        qsa.qsa_select_topk(cfg, segs, T, scores, scores.shape[1], sel_ref, nsel_ref, ws)
        sel = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
        nsel = torch.full((T,), -7, dtype=torch.int32, device="cuda")
        assert _noalloc(cfg, segs, T, scores, sel, nsel) == qsa.QSA_OK
        torch.cuda.synchronize()
        assert torch.equal(nsel, nsel_ref), call
        assert torch.equal(sel, sel_ref), call


def test_noalloc_rejects_a_batch_larger_than_its_scratch():
    sh = synth.Shape()
    cfg = qsa.make_config(sh)
    T = 500         # 500 decode rows at 2M context: 48 KiB of histogram and candidate list each
    segs = qsa.make_segments([(i, 1, (1 << 21) - 1, 0) for i in range(T)])
    assert qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT) > (16 << 20)
    scores = torch.zeros((1, 1), device="cuda")   # never read: rejected before any launch
    sel = torch.zeros((1, 512), dtype=torch.int32, device="cuda")
    n0 = qsa.launch_count()
    assert _noalloc(cfg, segs, T, scores.expand(T, 524288), sel, sel[0]) == qsa.QSA_ERR_WORKSPACE
    assert qsa.launch_count() == n0
