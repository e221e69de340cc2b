"""The GPU-vs-oracle acceptance checks themselves, on planted mistakes (CPU).

tests/qsa_testlib.py decides whether a GPU selection or output agrees with the
oracle.  Here the "GPU" side is the oracle's own result with one mistake
planted (a block swapped for a clearly worse one, a missing own block, a
wrong count, an unsorted row, an output off by more than the tolerance, a
NaN); each must be rejected, while the exact result and a swap inside the
tie band are accepted.
"""
import numpy as np
import pytest

import oracle
from qsa_testlib import check_outputs, selection_verdict

S = 16          # budget blocks of the small configuration below
R = 4


def _row(seed=0, t=400):
    cfg = oracle.config(budget_tokens=S * R, idx_dim=64)
    rng = np.random.default_rng(seed)
    bt = t // R
    s = rng.standard_normal(bt)
    sel, n = oracle.select(cfg, s, t)
    return cfg, s, np.asarray(sel), int(n), t


def test_exact_selection_is_accepted():
    _, s, sel, n, t = _row()
    assert selection_verdict(s, sel, n, sel.copy(), n, t, S) == "exact"


def test_swap_inside_the_tie_band_is_accepted():
    _, s, sel, n, t = _row()
    s = s.copy()
    order = np.lexsort((np.arange(len(s)), -s))
    last_kept, first_out = int(order[S - 2]), int(order[S - 1])
    s[first_out] = s[last_kept]                   # a tie between the last kept and the first dropped block
    cfg = oracle.config(budget_tokens=S * R, idx_dim=64)
    sel, n = oracle.select(cfg, s, t)
    sel = np.asarray(sel)
    kept = [int(b) for b in sel[:n - 1]]
    other = first_out if first_out not in kept else last_kept
    dropped = last_kept if other == first_out else first_out
    gpu = sorted([b for b in kept if b != dropped] + [other]) + [int(sel[n - 1])]
    gpu = np.array(gpu + [-1] * (S - len(gpu)), dtype=np.int32)
    assert selection_verdict(s, sel, n, gpu, n, t, S) == "band"


@pytest.mark.parametrize("mistake", ["worse_block", "own_block_missing", "short_count", "unsorted"])
def test_planted_selection_mistakes_are_rejected(mistake):
    _, s, sel, n, t = _row(seed=3)
    gpu = sel.copy()
    n_gpu = n
    kept = set(int(b) for b in sel[:n])
    if mistake == "worse_block":
        worst = int(np.argmin(s))
        assert worst not in kept
        best_kept = max(sel[:n - 1], key=lambda b: s[b])
        row = sorted([int(b) for b in sel[:n - 1] if b != best_kept] + [worst]) + [int(sel[n - 1])]
        gpu[:n] = row
    elif mistake == "own_block_missing":
        gpu[n - 1] = int(np.argmax([s[b] if b not in kept else -np.inf for b in range(len(s))]))
        gpu[:n] = np.sort(gpu[:n])
    elif mistake == "short_count":
        n_gpu = n - 1
        gpu[n - 1] = -1
    else:
        gpu[0], gpu[1] = gpu[1], gpu[0]
    with pytest.raises(AssertionError):
        selection_verdict(s, sel, n, gpu, n_gpu, t, S)


def test_padding_past_the_count_is_checked_on_a_short_row():
    _, s, sel, n, t = _row(seed=5, t=40)          # 10 complete blocks + own: n = 11 < S
    assert n < S
    gpu = sel.copy()
    gpu[n] = 3
    with pytest.raises(AssertionError):
        selection_verdict(s, sel, n, gpu, n, t, S)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_output_tolerances_reject_planted_errors(dtype):
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((8, 4, 32))
    lse = rng.standard_normal((8, 4))
    check_outputs(ref.astype(np.float32), ref, lse.astype(np.float32), lse, dtype, "exact")
    bad = ref.copy()
    bad[3, 1, 7] += 0.1                           # one element far outside both tolerances
    with pytest.raises(AssertionError):
        check_outputs(bad.astype(np.float32), ref, lse.astype(np.float32), lse, dtype, "one element")
    nan = ref.astype(np.float32)
    nan[0, 0, 0] = np.nan
    with pytest.raises(AssertionError):
        check_outputs(nan, ref, lse.astype(np.float32), lse, dtype, "nan")
    bad_lse = lse.copy()
    bad_lse[2, 2] += 0.01
    with pytest.raises(AssertionError):
        check_outputs(ref.astype(np.float32), ref, bad_lse.astype(np.float32), lse, dtype, "lse")
