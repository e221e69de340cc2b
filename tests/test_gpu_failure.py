"""Failure path of the bounded device-side waits, exercised without faulting
the GPU: a diagnostic kernel waits on an mbarrier phase that nothing
completes; the wait must give up, record QSA_ERR_TIMEOUT in the device error
word (reported and cleared by qsa_device_status), and leave the context
usable for ordinary calls."""
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_times_out_reports_and_recovers():
    assert qsa.device_status() == qsa.QSA_OK            # nothing pending from earlier tests
    qsa.qsa_selftest_wait_timeout()
    assert qsa.device_status() == qsa.QSA_ERR_TIMEOUT
    assert qsa.device_status() == qsa.QSA_OK            # the word was cleared
    # the context still runs real work: a selection over seeded rows
    sh = synth.Shape()
    cfg = qsa.make_config(sh)
    lengths = [600, 3000]
    segs = qsa.make_segments([(i, 1, 4 * n + 3, 0) for i, n in enumerate(lengths)])
    g = torch.Generator().manual_seed(3)
    rows = torch.randn((len(lengths), max(lengths)), generator=g).cuda()
    sel = torch.full((2, sh.budget_blocks), -7, dtype=torch.int32, device="cuda")
    nsel = torch.zeros((2,), dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, 2, qsa.QSA_OP_SELECT)), dtype=torch.uint8, device="cuda")
    qsa.qsa_select_topk(cfg, segs, 2, rows, rows.shape[1], sel, nsel, ws)
    torch.cuda.synchronize()
    assert nsel.tolist() == [sh.budget_blocks, sh.budget_blocks]
    assert qsa.device_status() == qsa.QSA_OK
