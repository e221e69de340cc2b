"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against a closed form, an invariant, a brute-force
enumeration or a library routine (numpy, torch CPU), so that a plausible slip
anywhere in the oracle (a dropped term, a wrong sign, a wrong index or pairing,
a transposed operand) fails at least one of them.

Sources of the facts: the design report summary page ("Qwen3.8-Next
architecture design report", QSA item: micro-block r=4, pooled keys get a
position encoding after pooling, 4 indexer heads, budget K=2048) and the Miles
docs page "Qwen3.8-Flash-Next", section 1 (24 heads, 2 query groups, head dim
256, rotary base 1e7 at rotary percent 0.25; attention reads only the kept
tokens).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def small_cfg(**kw):
    base = dict(r=4, budget_tokens=16, n_heads=4, n_groups=2, head_dim=16, idx_heads=4,
                idx_dim=32, rope_dims=8, rope_base=1e7, round_bf16=False)
    base.update(kw)
    return oracle.config(**base)


# --------------------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10,
                         np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, -0.0,
                                   3.3895314e38, 1e-40], np.float32)])
    want = torch.from_numpy(xs).to(torch.bfloat16).float().numpy()
    got = np.array([oracle.round_bf16(float(x)) for x in xs], np.float32)
    np.testing.assert_array_equal(got, want)


# --------------------------------------------------------------------------- rotary encoding
def test_rope_theta_formula():
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    for i in range(16):
        assert oracle.rope_theta(cfg, i) == pytest.approx(1e7 ** (-2.0 * i / 32), rel=1e-15)


@pytest.mark.parametrize("pos", [0, 1, 4, 12345, 1048572])
def test_rope_unit_vectors_closed_form(pos):
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    half = 16
    for i in [0, 3, 15]:
        th = 1e7 ** (-2.0 * i / 32)
        e = np.zeros(128, np.float32)
        e[i] = 1
        out = oracle.rope_vec(cfg, e, pos)
        want = np.zeros(128)
        want[i] = math.cos(pos * th)
        want[i + half] = math.sin(pos * th)
        np.testing.assert_allclose(out, want, atol=1e-7)
        e = np.zeros(128, np.float32)
        e[i + half] = 1
        out = oracle.rope_vec(cfg, e, pos)
        want = np.zeros(128)
        want[i] = -math.sin(pos * th)
        want[i + half] = math.cos(pos * th)
        np.testing.assert_allclose(out, want, atol=1e-7)


def test_rope_passthrough_and_norm():
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    x = np.random.default_rng(1).standard_normal(128).astype(np.float32)
    out = oracle.rope_vec(cfg, x, 777)
    np.testing.assert_array_equal(out[32:], x[32:])
    assert np.linalg.norm(out[:32]) == pytest.approx(np.linalg.norm(x[:32]), rel=2e-7)
    assert not np.allclose(out[:32], x[:32])


def test_rope_bf16_output_is_representable():
    cfg = small_cfg(idx_dim=128, rope_dims=32, round_bf16=True)
    x = torch.randn(128, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).float().numpy()
    out = oracle.rope_vec(cfg, x, 99)
    np.testing.assert_array_equal(out, torch.from_numpy(out).to(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------- pooling
def test_compress_is_mean_without_rope():
    cfg = small_cfg(rope_dims=0)
    k = np.random.default_rng(3).standard_normal((64, 32)).astype(np.float32)
    kh = oracle.compress_keys(cfg, k, 0, 16)
    want = k.astype(np.float64).reshape(16, 4, 32).mean(1)
    np.testing.assert_allclose(kh, want, rtol=1e-6, atol=1e-7)


def test_compress_constant_keys_pool_to_themselves():
    cfg = small_cfg(rope_dims=0)
    row = np.random.default_rng(4).standard_normal(32).astype(np.float32)
    k = np.tile(row, (40, 1))
    kh = oracle.compress_keys(cfg, k, 2, 10)
    np.testing.assert_allclose(kh, np.tile(row, (8, 1)), rtol=1e-7)


def test_compress_block_zero_is_unrotated_and_subrange_consistent():
    cfg = small_cfg()
    k = np.random.default_rng(5).standard_normal((64, 32)).astype(np.float32)
    kh = oracle.compress_keys(cfg, k, 0, 16)
    np.testing.assert_allclose(kh[0], k[:4].astype(np.float64).mean(0), rtol=1e-6, atol=1e-7)
    np.testing.assert_array_equal(oracle.compress_keys(cfg, k, 5, 9), kh[5:9])


def test_compress_rotates_at_block_start_position():
    """k^_b is the pooled key rotated by the angle of token position r*b."""
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    i = 5
    th = 1e7 ** (-2.0 * i / 32)
    k = np.zeros((4 * 300, 128), np.float32)
    k[:, i] = 1.0
    kh = oracle.compress_keys(cfg, k, 0, 300)
    for b in [1, 7, 299]:
        assert kh[b, i] == pytest.approx(math.cos(4 * b * th), abs=1e-7)
        assert kh[b, i + 16] == pytest.approx(math.sin(4 * b * th), abs=1e-7)


def test_compress_norm_preserved():
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    k = np.random.default_rng(6).standard_normal((400, 128)).astype(np.float32)
    kh = oracle.compress_keys(cfg, k, 0, 100)
    m = k.astype(np.float64).reshape(100, 4, 128).mean(1)
    np.testing.assert_allclose(np.linalg.norm(kh, axis=1), np.linalg.norm(m, axis=1), rtol=1e-6)


# --------------------------------------------------------------------------- scores
def _rand_index_case(seed, n=400, d=32, hi=4, rope=8):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n, d)).astype(np.float32)
    q = rng.standard_normal((hi, d)).astype(np.float32)
    w = rng.random(hi).astype(np.float32)
    return k, q, w


def test_scores_single_head_is_relu_of_dot():
    cfg = small_cfg()
    k, q, w = _rand_index_case(7)
    t = 397
    kh = oracle.compress_keys(cfg, k, 0, t // 4)
    for h in range(4):
        wh = np.zeros(4, np.float32)
        wh[h] = 1
        s = oracle.index_scores(cfg, q, wh, t, kh)
        qr = oracle.rope_vec(cfg, q[h], t)
        want = np.maximum(kh.astype(np.float64) @ qr.astype(np.float64), 0)
        np.testing.assert_allclose(s, want, rtol=1e-12, atol=1e-12)


def test_scores_weighted_sum_over_heads_and_nonnegative():
    cfg = small_cfg()
    k, q, w = _rand_index_case(8)
    t = 399
    kh = oracle.compress_keys(cfg, k, 0, t // 4)
    parts = []
    for h in range(4):
        wh = np.zeros(4, np.float32)
        wh[h] = 1
        parts.append(oracle.index_scores(cfg, q, wh, t, kh))
    s = oracle.index_scores(cfg, q, w, t, kh)
    np.testing.assert_allclose(s, sum(w[h] * parts[h] for h in range(4)), rtol=1e-12)
    assert (s >= 0).all() and (s == 0).any()


def test_scores_negated_query_complements():
    cfg = small_cfg()
    k, q, _ = _rand_index_case(9)
    t = 250
    kh = oracle.compress_keys(cfg, k, 0, t // 4)
    w1 = np.array([1, 0, 0, 0], np.float32)
    a = oracle.index_scores(cfg, q, w1, t, kh)
    b = oracle.index_scores(cfg, -q, w1, t, kh)
    qr = oracle.rope_vec(cfg, q[0], t).astype(np.float64)
    np.testing.assert_allclose(a - b, kh.astype(np.float64) @ qr, rtol=1e-12, atol=1e-12)
    assert (np.minimum(a, b) == 0).all()


def test_scores_closed_form_relative_angle():
    """Unit-vector query at t against unit-vector keys at block b: cos((t - r*b) theta)."""
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    i = 2
    th = 1e7 ** (-2.0 * i / 32)
    n = 4 * 200
    k = np.zeros((n, 128), np.float32)
    k[:, i] = 1
    q = np.zeros((4, 128), np.float32)
    q[:, i] = 1
    w = np.array([0.5, 0.25, 0.125, 1.0], np.float32)
    t = 795
    kh = oracle.compress_keys(cfg, k, 0, t // 4)
    s = oracle.index_scores(cfg, q, w, t, kh)
    b = np.arange(t // 4)
    want = w.astype(np.float64).sum() * np.maximum(np.cos((t - 4 * b) * th), 0)
    np.testing.assert_allclose(s, want, atol=1e-6)


def test_scores_depend_on_relative_position_only():
    cfg = small_cfg(idx_dim=128, rope_dims=32)
    rng = np.random.default_rng(10)
    nb = 64
    blocks = rng.standard_normal((nb * 4, 128)).astype(np.float32)
    q = rng.standard_normal((4, 128)).astype(np.float32)
    w = rng.random(4).astype(np.float32)
    t0 = nb * 4 + 2
    s0 = oracle.index_scores(cfg, q, w, t0, oracle.compress_keys(cfg, blocks, 0, nb))
    shift = 4 * 1000                      # shift everything by 1000 blocks
    k = np.zeros((shift + nb * 4, 128), np.float32)
    k[shift:] = blocks
    kh = oracle.compress_keys(cfg, k, 0, (shift + t0) // 4)
    s1 = oracle.index_scores(cfg, q, w, shift + t0, kh)[1000:]
    np.testing.assert_allclose(s1, s0, rtol=2e-5, atol=2e-5)


# --------------------------------------------------------------------------- selection
def _brute_force_select(scores, t, S, r):
    bt = t // r
    if bt + 1 <= S:
        return list(range(bt + 1))
    best_key, best = None, None
    for sub in itertools.combinations(range(bt), S - 1):
        key = (sum(scores[b] for b in sub), tuple(-b for b in sub))
        if best_key is None or key > best_key:
            best_key, best = key, sub
    return sorted(best) + [bt]


@pytest.mark.parametrize("seed", range(12))
def test_select_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    S = 4
    cfg = small_cfg(budget_tokens=4 * S)
    t = int(rng.integers(0, 40))
    scores = rng.integers(0, 4, size=max(t // 4, 1)).astype(np.float64)  # many exact ties
    sel, n = oracle.select(cfg, scores, t)
    want = _brute_force_select(scores, t, S, 4)
    assert n == len(want)
    assert list(sel[:n]) == want
    assert (sel[n:] == -1).all()


def test_select_structure_at_page_budget():
    cfg = oracle.config()
    rng = np.random.default_rng(11)
    for t in [0, 3, 2047, 2048, 2051, 9000, 65535]:
        bt = t // 4
        s = rng.standard_normal(max(bt, 1))
        sel, n = oracle.select(cfg, s, t)
        assert n == min(512, bt + 1)
        assert sel[n - 1] == bt
        assert (np.diff(sel[:n]) > 0).all()
        assert (sel[n:] == -1).all()
        if bt + 1 > 512:
            kept = set(sel[:n - 1])
            thr = min(s[b] for b in kept)
            assert all(s[b] <= thr for b in range(bt) if b not in kept)


def test_select_negative_zero_ties_with_positive_zero():
    cfg = small_cfg(budget_tokens=8)   # S = 2: own block + 1
    t = 4 * 5
    s = np.array([-1.0, -0.0, 0.0, -2.0, 0.0])
    sel, n = oracle.select(cfg, s, t)
    assert list(sel[:n]) == [1, 5]


# --------------------------------------------------------------------------- attention
def _dense_gqa_reference(q, k, v, mask, scale):
    """fp64 torch SDPA over an explicit boolean mask [nq, n]; q [nq,H,D], k/v [G,n,D]."""
    H, G = q.shape[1], k.shape[0]
    kk = torch.from_numpy(k).double().repeat_interleave(H // G, 0)      # [H, n, D]
    vv = torch.from_numpy(v).double().repeat_interleave(H // G, 0)
    qq = torch.from_numpy(q).double().permute(1, 0, 2)                  # [H, nq, D]
    m = torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=m, scale=scale)
    s = (qq @ kk.transpose(1, 2)) * scale
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return o.permute(1, 0, 2).numpy(), lse.T.numpy()


def _rand_attn_case(seed, n, H=4, G=2, D=16, dI=32):
    rng = np.random.default_rng(seed)
    return dict(q=rng.standard_normal((n, H, D)).astype(np.float32),
                q_idx=rng.standard_normal((n, 4, dI)).astype(np.float32),
                w=rng.random((n, 4)).astype(np.float32),
                k_idx=rng.standard_normal((n, dI)).astype(np.float32),
                k=rng.standard_normal((G, n, D)).astype(np.float32),
                v=rng.standard_normal((G, n, D)).astype(np.float32))


def test_forward_with_budget_covering_context_is_dense_causal_attention():
    n = 64
    cfg = small_cfg(budget_tokens=256)
    c = _rand_attn_case(12, n)
    pos = np.arange(n)
    out = oracle.forward(cfg, c["q"], c["q_idx"], c["w"], pos, c["k_idx"], c["k"], c["v"])
    mask = np.tril(np.ones((n, n), bool))
    o, lse = _dense_gqa_reference(c["q"], c["k"], c["v"], mask, cfg.softmax_scale)
    np.testing.assert_allclose(out["o"], o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-12, atol=1e-12)
    assert (out["nsel"] == pos // 4 + 1).all()


def test_forward_equals_masked_dense_attention_on_its_selection():
    n = 200
    cfg = small_cfg(budget_tokens=16)   # 4 blocks
    c = _rand_attn_case(13, n)
    pos = np.arange(n)
    out = oracle.forward(cfg, c["q"], c["q_idx"], c["w"], pos, c["k_idx"], c["k"], c["v"])
    mask = np.zeros((n, n), bool)
    for t in range(n):
        for b in out["sel"][t, :out["nsel"][t]]:
            for j in range(4 * b, 4 * b + 4):
                if j <= t:
                    mask[t, j] = True
    assert (mask.sum(1) == np.minimum(pos + 1, 12 + pos % 4 + 1)).all()
    o, lse = _dense_gqa_reference(c["q"], c["k"], c["v"], mask, cfg.softmax_scale)
    np.testing.assert_allclose(out["o"], o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-12, atol=1e-12)


def test_forward_uses_own_index_scores_for_selection():
    n = 120
    cfg = small_cfg(budget_tokens=12)   # 3 blocks: own + 2
    c = _rand_attn_case(14, n)
    pos = np.arange(n)
    out = oracle.forward(cfg, c["q"], c["q_idx"], c["w"], pos, c["k_idx"], c["k"], c["v"])
    kh = oracle.compress_keys(cfg, c["k_idx"], 0, n // 4)
    for t in [13, 57, 119]:
        s = oracle.index_scores(cfg, c["q_idx"][t], c["w"][t], t, kh)
        top = sorted(sorted(range(t // 4), key=lambda b: (-s[b], b))[:2]) + [t // 4]
        assert list(out["sel"][t, :3]) == top


def test_attention_constant_values_and_group_mapping():
    n = 96
    cfg = small_cfg(budget_tokens=16)
    c = _rand_attn_case(15, n)
    c["v"][0] = 0.25
    c["v"][1] = -3.0
    out = oracle.forward(cfg, c["q"], c["q_idx"], c["w"], np.arange(n), c["k_idx"], c["k"], c["v"])
    np.testing.assert_allclose(out["o"][:, :2], 0.25, rtol=1e-14)
    np.testing.assert_allclose(out["o"][:, 2:], -3.0, rtol=1e-14)


def test_attention_own_block_is_causally_masked():
    cfg = small_cfg(budget_tokens=16)
    n = 64
    c = _rand_attn_case(16, n)
    t = 41                                        # own block 10 holds tokens 40..43
    sel = np.array([10, -1, -1, -1], np.int32)
    o, lse = oracle.attend(cfg, c["q"][t], c["k"], c["v"], t, sel, 1)
    mask = np.zeros((1, n), bool)
    mask[0, 40:42] = True
    o2, lse2 = _dense_gqa_reference(c["q"][t:t + 1], c["k"], c["v"], mask, cfg.softmax_scale)
    np.testing.assert_allclose(o, o2[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse2[0], rtol=1e-12)


def test_needles_are_selected_and_retrieved():
    """Planted needle blocks (key = scaled copy of the query) are kept and dominate head 0."""
    from block_sparse_attention_22_b200 import synth
    wl = synth.make_workload("prefill_8k", n=4096, n_seqs=1)
    x = synth.make_inputs(wl)
    cfg = oracle.config_from_shape(wl.shape)
    tgt = [(t, b) for (s, t, b) in wl.needles][:6]
    pos = np.array([t for t, _ in tgt])
    f = lambda a: a.float().numpy()
    out = oracle.forward(cfg, f(x["q"][pos]), f(x["q_idx"][pos]), f(x["w"][pos]), pos,
                         f(x["k_idx"][0]), f(x["k"][0]), f(x["v"][0]))
    for i, (t, b) in enumerate(tgt):
        assert b in set(out["sel"][i, :out["nsel"][i]])
        needle_v = f(x["v"][0, 0, 4 * b:4 * b + 4]).astype(np.float64).mean(0)
        np.testing.assert_allclose(out["o"][i, 0], needle_v, atol=5e-3)


# --------------------------------------------------------------------------- cross-checks
def test_fp32_accumulation_build_agrees_with_fp64_build():
    from block_sparse_attention_22_b200 import synth
    wl = synth.make_workload("tiny_fp32")
    x = synth.make_inputs(wl)
    cfg = oracle.config_from_shape(wl.shape)
    pos = np.arange(256)
    f = lambda a: a.float().numpy()
    args = (f(x["q"]), f(x["q_idx"]), f(x["w"]), pos, f(x["k_idx"][0]), f(x["k"][0]), f(x["v"][0]))
    a = oracle.forward(cfg, *args, acc="f64")
    b = oracle.forward(cfg, *args, acc="f32")
    assert oracle.acc_bits("f64") == 64 and oracle.acc_bits("f32") == 32
    same = (a["sel"] == b["sel"]).all(1)
    assert same.mean() > 0.99
    np.testing.assert_allclose(b["o"][same], a["o"][same], atol=1e-5)
    np.testing.assert_allclose(b["lse"][same], a["lse"][same], atol=1e-5)


# --------------------------------------------------------------------------- attention backward
def _loss(cfg, q, k, v, t, sel, nsel, dout):
    o, _ = oracle.attend(cfg, q, k, v, t, sel, nsel)
    return float((o * dout.astype(np.float64)).sum())


def test_backward_matches_finite_differences_of_the_forward():
    """Central differences of the forward oracle's loss sum(dout * o) against the
    backward oracle, on coordinates of q, of kept keys and values, of a key outside
    the causal range (zero gradient) and of a key not kept (zero gradient)."""
    cfg = small_cfg(budget_tokens=12)
    n, t = 40, 37                                  # own block 9 holds 36..39: 36, 37 attended
    c = _rand_attn_case(21, n)
    sel = np.array([2, 5, 9], np.int32)
    rng = np.random.default_rng(5)
    dout = rng.standard_normal((cfg.n_heads, cfg.head_dim)).astype(np.float32)
    q, k, v = c["q"][t].copy(), c["k"].copy(), c["v"].copy()
    dq, dk, dv = oracle.attend_bwd(cfg, q, k, v, t, sel, 3, dout)
    eps = 2.0 ** -11

    def fd(arr, idx):
        x = arr[idx]
        arr[idx] = x + eps
        lp = _loss(cfg, q, k, v, t, sel, 3, dout)
        arr[idx] = x - eps
        lm = _loss(cfg, q, k, v, t, sel, 3, dout)
        arr[idx] = x
        return (lp - lm) / (2 * eps)

    for h, d in [(0, 0), (1, 7), (3, 15), (2, 3)]:
        np.testing.assert_allclose(fd(q, (h, d)), dq[h, d], rtol=2e-5, atol=1e-7)
    for g, j, d in [(0, 8, 1), (1, 21, 4), (0, 36, 9), (1, 37, 15), (0, 11, 0)]:
        np.testing.assert_allclose(fd(k, (g, j, d)), dk[g, j, d], rtol=2e-5, atol=1e-7)
        np.testing.assert_allclose(fd(v, (g, j, d)), dv[g, j, d], rtol=2e-5, atol=1e-7)
    # key 38 is in the own block but after t; key 12 is in a block not kept
    for g, j in [(0, 38), (1, 38), (0, 12), (1, 12)]:
        assert np.all(dk[g, j] == 0) and np.all(dv[g, j] == 0)
        assert fd(k, (g, j, 3)) == 0.0 and fd(v, (g, j, 3)) == 0.0


def test_backward_with_budget_covering_context_is_dense_attention_backward():
    """Budget >= context: the sparse backward equals torch autograd of dense causal
    GQA attention in fp64 (dq per query; dk, dv summed over the queries)."""
    n = 48
    cfg = small_cfg(budget_tokens=256)
    c = _rand_attn_case(22, n)
    rng = np.random.default_rng(6)
    dout = rng.standard_normal((n, cfg.n_heads, cfg.head_dim)).astype(np.float32)
    dk = np.zeros(c["k"].shape, np.float64)
    dv = np.zeros(c["v"].shape, np.float64)
    dqs = []
    for t in range(n):
        nb = t // 4 + 1
        sel = np.arange(nb, dtype=np.int32)
        dq, dk, dv = oracle.attend_bwd(cfg, c["q"][t], c["k"], c["v"], t, sel, nb, dout[t], dk, dv)
        dqs.append(dq)
    H, G = cfg.n_heads, cfg.n_groups
    q = torch.from_numpy(c["q"]).double().permute(1, 0, 2).requires_grad_(True)     # [H, n, D]
    k = torch.from_numpy(c["k"]).double().requires_grad_(True)                      # [G, n, D]
    v = torch.from_numpy(c["v"]).double().requires_grad_(True)
    kk = k.repeat_interleave(H // G, 0)
    vv = v.repeat_interleave(H // G, 0)
    s = (q @ kk.transpose(1, 2)) * cfg.softmax_scale
    s = s.masked_fill(~torch.tril(torch.ones(n, n, dtype=torch.bool)), float("-inf"))
    o = torch.softmax(s, -1) @ vv
    (o * torch.from_numpy(dout).double().permute(1, 0, 2)).sum().backward()
    np.testing.assert_allclose(np.stack(dqs), q.grad.permute(1, 0, 2).numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_backward_constant_values_give_zero_query_and_key_gradients():
    """Constant V makes every dp equal to its mean: ds = 0, so dq = dk = 0, while dv
    of each attended key is its probability times dout."""
    cfg = small_cfg(budget_tokens=16)
    n, t = 64, 50
    c = _rand_attn_case(23, n)
    c["v"][:] = 1.5
    sel = np.array([3, 7, 11, 12], np.int32)
    dout = np.random.default_rng(7).standard_normal((cfg.n_heads, cfg.head_dim)).astype(np.float32)
    dq, dk, dv = oracle.attend_bwd(cfg, c["q"][t], c["k"], c["v"], t, sel, 4, dout)
    np.testing.assert_allclose(dq, 0, atol=1e-12)
    np.testing.assert_allclose(dk, 0, atol=1e-12)
    # sum over attended keys of dv = (sum of probabilities) * dout per head = dout, per group
    hpg = cfg.n_heads // cfg.n_groups
    for g in range(cfg.n_groups):
        np.testing.assert_allclose(dv[g].sum(0), dout[g * hpg:(g + 1) * hpg].astype(np.float64).sum(0),
                                   rtol=1e-12, atol=1e-12)
