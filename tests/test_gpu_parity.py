"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Stage by stage (pooled keys, scores, selection on seeded score rows, attention
on the oracle's selection) and end to end (qsa_forward) on the workloads the
pages describe, at sizes the oracle finishes in seconds (several tiles and a
ragged tail) and at full size on sampled queries.  Tolerances are in
tests/qsa_testlib.py.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth
from qsa_testlib import (OracleSeq, check_outputs, compare_forward, gpu_forward, gpu_prepare_cache,
                         sample_tokens, segments_of, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _cuda_inputs(wl, gen_device="cpu"):
    x = synth.make_inputs(wl, device=gen_device)
    return {k: v.cuda() for k, v in x.items()}


# --------------------------------------------------------------------------- stage: pooling
@pytest.mark.parametrize("dtype,idx_dim,rope_fraction", [
    ("bf16", 128, 0.25), ("f32", 64, 0.25), ("bf16", 64, 0.25), ("f32", 128, 0.25),
    ("bf16", 128, 0.3),      # 19 rotated pairs: a pair's partner sits in another 16-byte chunk
    ("f32", 64, 0.3),        # 9 pairs
    ("f32", 64, 1.0),        # every dim rotates
])
def test_compress_keys_bit_exact_including_large_positions(dtype, idx_dim, rope_fraction):
    sh = synth.Shape(dtype=dtype, idx_dim=idx_dim, rope_fraction=rope_fraction)
    n_cap = 1 << 20
    g = torch.Generator().manual_seed(5)
    k_idx = torch.randn((1, n_cap, sh.idx_dim), generator=g).to(sh.torch_dtype).cuda()
    khat = torch.zeros((1, n_cap // 4, sh.idx_dim), dtype=sh.torch_dtype, device="cuda")
    dummy = torch.zeros((1, 2, n_cap, 256), dtype=sh.torch_dtype, device="cuda")
    cfg = qsa.make_config(sh)
    cache = qsa.make_cache(k_idx, khat, dummy, dummy)
    ranges = [(0, 0, 37), (0, 1000, 1001), (0, 262000, 262144)]
    qsa.qsa_compress_keys(cfg, cache, [r[0] for r in ranges], [r[1] for r in ranges], [r[2] for r in ranges])
    torch.cuda.synchronize()
    rc = oracle.config_from_shape(sh)
    for _, b0, b1 in ranges:
        ref = oracle.compress_keys(rc, to_np(k_idx[0, :4 * b1]), b0, b1)
        got = to_np(khat[0, b0:b1])
        np.testing.assert_array_equal(got, ref)
    untouched = torch.count_nonzero(khat[0, 37:1000]).item()
    assert untouched == 0


# --------------------------------------------------------------------------- stage: scores
@pytest.mark.parametrize("name,over", [("tiny_fp32", {}), ("prefill_8k", dict(n=3001, n_seqs=1))])
def test_index_scores_parity(name, over):
    wl = synth.make_workload(name, **over)
    x = _cuda_inputs(wl)
    sh = wl.shape
    cfg, cache, khat = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    # pool every complete block first
    qsa.qsa_compress_keys(cfg, cache, [0], [0], [wl.fill[0] // 4])
    T = wl.n_tokens
    ld = max(1, (wl.segments[-1].pos0 + wl.segments[-1].q_len - 1) // 4)
    scores = torch.full((T, ld), float("nan"), device="cuda")
    qsa.qsa_index_scores(cfg, cache, segs, T, x["q_idx"], x["w"], scores, ld)
    torch.cuda.synchronize()
    seq = OracleSeq(wl, x, 0)
    pos = wl.token_positions().numpy()
    for i in sample_tokens(wl, 97):
        t = int(pos[i])
        ref = oracle.index_scores(seq.cfg, to_np(x["q_idx"][i]), to_np(x["w"][i]), t, seq.khat)
        got = to_np(scores[i, :t // 4])
        tol = 2e-5 * (np.abs(ref).max() if ref.size else 0) + 1e-6
        assert np.abs(got - ref).max(initial=0) <= tol, (i, t)
        if t // 4 < ld:
            assert torch.isnan(scores[i, t // 4:]).all()   # nothing written past the causal edge


# --------------------------------------------------------------------------- stage: selection
def _score_rows(seed, lengths, tie_levels=None):
    g = torch.Generator().manual_seed(seed)
    ld = max(lengths)
    rows = torch.randn((len(lengths), ld), generator=g).abs() * 7
    if tie_levels:
        rows = torch.randint(0, tie_levels, (len(lengths), ld), generator=g).float()
        rows[rows == 0] = -0.0                       # -0 and +0 must tie
        rows[:, ::3] = torch.where(rows[:, ::3] == -0.0, torch.zeros(()), rows[:, ::3])
    return rows


@pytest.mark.parametrize("lengths,ties", [
    ([1, 3, 511, 512, 513, 600, 2047, 2048, 4096, 32767], None),
    ([600, 3000, 32767], 3),
    ([20000, 32768, 3000], None),         # few rows: one wide CTA per row
    ([32769, 40000, 65535], None),        # few long rows: 4096-score chunks sharing a row histogram
    ([65535, 262143], 5),
    ([300001, 70000], 2),                 # ties everywhere: candidate list too long, exact fallback
    ([40961, 4097, 4096, 8191, 600, 511, 1], None),   # one-element last chunks, single-chunk rows, short rows
])
def test_select_topk_matches_oracle_on_seeded_rows(lengths, ties):
    S = 512
    cfg_sh = synth.Shape()
    cfg = qsa.make_config(cfg_sh)
    rows = _score_rows(len(lengths) + (ties or 0), lengths, ties)
    # one decode-like segment per row at position t = 4*len + 3
    segs_l = [(i, 1, 4 * n + 3, 0) for i, n in enumerate(lengths)]
    segs = qsa.make_segments(segs_l)
    T = len(lengths)
    sc = rows.cuda().contiguous()
    sel = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT)), dtype=torch.uint8, device="cuda")
    qsa.qsa_select_topk(cfg, segs, T, sc, sc.shape[1], sel, nsel, ws)
    torch.cuda.synchronize()
    rc = oracle.config_from_shape(cfg_sh)
    for i, n in enumerate(lengths):
        t = 4 * n + 3
        ref, rn = oracle.select(rc, rows[i, :n].double().numpy(), t)
        assert int(nsel[i]) == rn
        np.testing.assert_array_equal(sel[i].cpu().numpy(), ref)


@pytest.mark.parametrize("case", ["odd_ld", "negative", "needles", "one_hot", "dense_bin", "mid_bin", "tied_bin"])
def test_select_few_long_rows_edge_cases(case):
    """The few-long-rows path (a row histogram of the top 12 key bits, then a
    filter at the bin holding the 511th largest): rows whose start is not
    16-byte aligned (odd row pitch), negative scores, a few dominant needles
    far above the rest, a row that is zero but for one element, scores
    packed into a narrow range so that the threshold bin holds thousands of
    elements (near and over the candidate list's capacity: the exact
    fallback), a threshold bin of about 2000 elements (radix select over the
    bin), and 600 equal scores in the threshold bin of which the lowest
    indices must win (selection by counting)."""
    S = 512
    cfg_sh = synth.Shape()
    cfg = qsa.make_config(cfg_sh)
    lengths = [65535, 100003, 40000, 262143]
    g = torch.Generator().manual_seed(23)
    ld = max(lengths) + (1 if case == "odd_ld" else 0)
    rows = torch.randn((len(lengths), ld), generator=g) * 7
    if case != "negative":
        rows = rows.abs()
    if case == "needles":
        for i, n in enumerate(lengths):
            rows[i, torch.randint(0, n, (40,), generator=g)] = 1e6 + torch.arange(40).float()
    if case == "one_hot":
        rows.zero_()
        rows[:, 12345] = 1.0
    if case == "dense_bin":
        rows = 100.0 + torch.rand((len(lengths), ld), generator=g) * 0.5   # one bin of the top bits holds ~all
        rows[0] = 100.0 + torch.rand((ld,), generator=g) * 12.5 * 8        # ~5000 per bin near the top: fits or not
    if case in ("mid_bin", "tied_bin"):
        rows = torch.rand((len(lengths), ld), generator=g)                 # below the threshold bin
        for i, n in enumerate(lengths):
            pos = torch.randperm(n, generator=g)
            rows[i, pos[:300]] = 200.0 + torch.rand(300, generator=g) * 50   # 300 above the bin
            if case == "mid_bin":
                rows[i, pos[300:2300]] = 96.0 + torch.rand(2000, generator=g) * 7.9   # one bin of the top bits
            else:
                rows[i, pos[300:900]] = 100.0                                  # 600 equal keys, 211 kept
    segs = qsa.make_segments([(i, 1, 4 * n + 3, 0) for i, n in enumerate(lengths)])
    T = len(lengths)
    sc = rows.cuda().contiguous()
    sel = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT)), dtype=torch.uint8, device="cuda")
    qsa.qsa_select_topk(cfg, segs, T, sc, ld, sel, nsel, ws)
    torch.cuda.synchronize()
    rc = oracle.config_from_shape(cfg_sh)
    for i, n in enumerate(lengths):
        ref, rn = oracle.select(rc, rows[i, :n].double().numpy(), 4 * n + 3)
        assert int(nsel[i]) == rn
        np.testing.assert_array_equal(sel[i].cpu().numpy(), ref, err_msg=f"{case} row {i}")
    # the same call again on the same workspace: the histograms and counters restart from zero
    sel2 = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
    qsa.qsa_select_topk(cfg, segs, T, sc, ld, sel2, nsel, ws)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2)


@pytest.mark.parametrize("tie_levels", [None, 2, 1000])
def test_select_many_rows_matches_oracle(tie_levels):
    """700 rows, enough for the many-rows kernel (one warp per row): lengths on
    both sides of every threshold it has (S, the list capacity 1024, the
    sampled threshold, 64K blocks for the bitmap ordering), random keys, two
    tie levels (every list overflows: the exact fallback) or a thousand levels
    (many ties at the K-th key)."""
    S = 512
    cfg_sh = synth.Shape()
    cfg = qsa.make_config(cfg_sh)
    base = [1, 3, 511, 512, 513, 600, 1023, 1024, 1025, 1536, 2047, 4096, 16384, 32767, 65535, 65536, 70001]
    lengths = [base[i % len(base)] for i in range(700)]
    rows = _score_rows(11 + (tie_levels or 0), lengths, tie_levels)
    segs = qsa.make_segments([(i, 1, 4 * n + 3, 0) for i, n in enumerate(lengths)])
    T = len(lengths)
    sc = rows.cuda().contiguous()
    sel = torch.full((T, S), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_SELECT)), dtype=torch.uint8, device="cuda")
    qsa.select_fallbacks()
    qsa.qsa_select_topk(cfg, segs, T, sc, sc.shape[1], sel, nsel, ws)
    torch.cuda.synchronize()
    fallbacks = qsa.select_fallbacks()
    if tie_levels == 2:
        assert fallbacks > 0
    rc = oracle.config_from_shape(cfg_sh)
    sel_c, nsel_c = sel.cpu().numpy(), nsel.cpu().numpy()
    for i, n in enumerate(lengths):
        ref, rn = oracle.select(rc, rows[i, :n].double().numpy(), 4 * n + 3)
        assert int(nsel_c[i]) == rn, i
        np.testing.assert_array_equal(sel_c[i], ref, err_msg=f"row {i} length {n}")


# --------------------------------------------------------------------------- stage: attention
@pytest.mark.parametrize("name,over,every", [
    ("tiny_fp32", {}, 1),
    ("prefill_8k", dict(n=2600, n_seqs=1), 13),
    ("decode_256k", dict(ctx=9001, n_seqs=3), 1),           # split-K + combine path
])
def test_attention_parity_on_oracle_selection(name, over, every):
    wl = synth.make_workload(name, **over)
    x = _cuda_inputs(wl)
    sh = wl.shape
    tokens = sample_tokens(wl, every)
    pos = wl.token_positions().numpy()
    slots = wl.token_slots().numpy()
    seqs = {}
    S = sh.budget_blocks
    T = wl.n_tokens
    sel = torch.full((T, S), -1, dtype=torch.int32)
    nsel = torch.ones((T,), dtype=torch.int32)
    refs = {}
    for i in tokens:
        s = int(slots[i])
        seqs.setdefault(s, OracleSeq(wl, x, s))
        r = seqs[s].query(to_np(x["q"][i]), to_np(x["q_idx"][i]), to_np(x["w"][i]), int(pos[i]))
        sel[i] = torch.from_numpy(r["sel"])
        nsel[i] = r["nsel"]
        refs[i] = r
    # untested tokens attend only to their own block
    for i in range(T):
        if i not in refs:
            sel[i, 0] = int(pos[i]) // 4
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    o = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), dtype=sh.torch_dtype, device="cuda")
    lse = torch.empty((T, sh.n_heads), device="cuda")
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_ATTN)), dtype=torch.uint8, device="cuda")
    qsa.qsa_sparse_attn_fwd(cfg, cache, segs, T, x["q"], sel.cuda(), nsel.cuda(), o, lse, ws)
    torch.cuda.synchronize()
    o_ref = np.stack([refs[i]["o"] for i in tokens])
    lse_ref = np.stack([refs[i]["lse"] for i in tokens])
    check_outputs(to_np(o[tokens]), o_ref, to_np(lse[tokens]), lse_ref, sh.dtype, name)


# --------------------------------------------------------------------------- end to end
@pytest.mark.parametrize("name,over,every,min_exact", [
    ("tiny_fp32", {}, 1, 0.99),
    ("prefill_8k", dict(n=2500, n_seqs=2), 7, 0.99),
    ("decode_256k", dict(ctx=20001, n_seqs=4), 1, 0.99),
    ("spec_decode_1m", dict(ctx=20001, n_seqs=3), 1, 0.99),     # 4 queries share a k^ stream
    ("decode_256k", dict(ctx=140001, n_seqs=3), 1, 0.99),      # rows past 32K blocks: histogram selection
    ("spec_decode_1m", dict(ctx=140001, n_seqs=2), 1, 0.99),
    ("mixed_1m", dict(ctx=16384, n_decode=3, chunk=300, chunk_pos0=5001), 3, 0.99),
])
def test_forward_parity_small(name, over, every, min_exact):
    wl = synth.make_workload(name, **over)
    x = _cuda_inputs(wl)
    run = gpu_forward(wl, x)
    res = compare_forward(wl, x, run, sample_tokens(wl, every), min_exact)
    assert res["n"] > 0


def test_forward_short_budget_selection_active_everywhere():
    """A 256-token budget on a ragged 2500-token prefill: every query past t=255 selects."""
    wl = synth.make_workload("prefill_8k", n=2500, n_seqs=1, shape=dict(budget_tokens=256))
    x = _cuda_inputs(wl)
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, range(wl.n_tokens))


@pytest.mark.parametrize("name,every,max_seqs", [
    ("prefill_8k", 61, None),
    ("prefill_128k", 1021, None),
    ("decode_256k", 1, 6),
    ("mixed_1m", 97, 3),
])
def test_forward_parity_full_size_sampled(name, every, max_seqs):
    wl = synth.make_workload(name)
    x = synth.make_inputs(wl, device="cuda")
    run = gpu_forward(wl, x)
    toks = sample_tokens(wl, every)
    if max_seqs is not None:
        slots = wl.token_slots().numpy()
        keep = sorted(set(slots[toks]))[:max_seqs - 1] + [int(slots[-1])]
        toks = [i for i in toks if slots[i] in keep]
    compare_forward(wl, x, run, toks)
    # invariants on every query: counts, own block last, sorted, padding
    pos = wl.token_positions()
    nsel = run.nsel.cpu()
    S = wl.shape.budget_blocks
    assert torch.equal(nsel, torch.clamp(pos // 4 + 1, max=S).int())
    sel = run.sel.cpu()
    last = sel.gather(1, (nsel.long() - 1).unsqueeze(1)).squeeze(1)
    assert torch.equal(last.long(), pos // 4)
    ar = torch.arange(S).unsqueeze(0)
    assert bool(((sel == -1) == (ar >= nsel.unsqueeze(1))).all())
    d = sel[:, 1:] - sel[:, :-1]
    valid = ar[:, 1:] < nsel.unsqueeze(1)
    assert bool((d[valid] > 0).all())


def test_needles_kept_and_retrieved_on_gpu():
    wl = synth.make_workload("prefill_8k")
    x = synth.make_inputs(wl, device="cuda")
    run = gpu_forward(wl, x)
    offs = wl.token_offsets()
    for (slot, t, b) in wl.needles:
        i = offs[slot] + t
        n = int(run.nsel[i])
        assert b in set(run.sel[i, :n].tolist()), (slot, t, b)
        v_mean = x["v"][slot, 0, 4 * b:4 * b + 4].float().mean(0)
        assert torch.allclose(run.o[i, 0].float(), v_mean, atol=2e-2), (slot, t, b)


# --------------------------------------------------------------------------- edge cases
def test_first_tokens_attend_only_themselves_and_empty_calls_are_noops():
    wl = synth.make_workload("prefill_8k", n=8, n_seqs=1)
    x = _cuda_inputs(wl)
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, range(8))
    # token 0 attends only token 0 of its group: output = V row 0
    v0 = x["v"][0, :, 0].float()
    assert torch.allclose(run.o[0, :12].float(), v0[0].expand(12, -1), atol=1e-2)
    assert torch.allclose(run.o[0, 12:].float(), v0[1].expand(12, -1), atol=1e-2)
    # empty batch / zero-length segments
    sh = wl.shape
    cfg, cache, _ = gpu_prepare_cache(wl, x)
    segs = qsa.make_segments([(0, 0, 5, 0)])
    qsa.qsa_forward(cfg, cache, segs, 0, x["q"], x["q_idx"], x["w"], run.o, None, None, None, None)
    torch.cuda.synchronize()


def test_many_segments_span_several_launch_tables():
    """More than one launch table of segments (batched launches), out of slot order, with gaps."""
    sh = synth.Shape()
    n_seq, ctx = 150, 700
    wl = synth.Workload("many", sh, [], n_seq, 1024, [ctx] * n_seq, [0] * n_seq, [], 11)
    segs = []
    for s in reversed(range(n_seq)):
        segs.append(synth.Segment(s, ctx - 3 - (s % 3), 1 + (s % 3)))
    wl.segments = segs
    wl.cached_blocks = [0] * n_seq
    x = _cuda_inputs(wl)
    # pool each sequence's prefix blocks first (they precede the queries)
    for i, sg in enumerate(wl.segments):
        wl.cached_blocks[sg.slot] = sg.pos0 // 4
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, range(0, wl.n_tokens, 5))


def test_duplicate_blocks_tie_toward_lower_index():
    """Hundreds of blocks with identical pooled keys score identically and above every
    other candidate; the kept ones must be the lowest indices among them."""
    wl = synth.make_workload("decode_256k", ctx=8192, n_seqs=2)
    x = synth.make_inputs(wl)
    rho = wl.shape.rope_dims
    # a key aligned with sequence 0's decode query, rotary dims zeroed so that
    # the block position encoding leaves every copy identical
    u = (x["w"][0].unsqueeze(1) * x["q_idx"][0].float()).sum(0)
    u[:rho] = 0
    for b in range(100, 1900, 3):
        x["k_idx"][0, 4 * b:4 * b + 4] = u.to(x["k_idx"].dtype)
    x = {k: v.cuda() for k, v in x.items()}
    run = gpu_forward(wl, x)
    compare_forward(wl, x, run, range(wl.n_tokens), min_exact=1.0)
    kept = run.sel[0, :511].tolist()
    dup = list(range(100, 1900, 3))
    assert sum(1 for b in kept if b in set(dup)) > 400


# --------------------------------------------------------------------------- determinism
def test_forward_is_deterministic_across_calls():
    """No atomics order results on the forward path: two calls on the same inputs
    give bit-identical outputs, log-sum-exps and selections."""
    wl = synth.make_workload("mixed_1m", ctx=16384, n_decode=3, chunk=300, chunk_pos0=5001)
    x = _cuda_inputs(wl)
    a = gpu_forward(wl, x)
    b = gpu_forward(wl, x)
    assert torch.equal(a.sel, b.sel) and torch.equal(a.nsel, b.nsel)
    assert torch.equal(a.o.view(torch.int16), b.o.view(torch.int16))
    assert torch.equal(a.lse, b.lse)
