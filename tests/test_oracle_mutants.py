"""Planted mistakes in the oracle must fail its pins.

Each case copies oracle/qsa_oracle.c, plants one plausible mistake (a
dropped term, a wrong sign, index, operand or bound), builds both
accumulation variants of the mutant with the oracle's own flags, and runs
tests/test_oracle_pins.py against it in a child process.  The pins are
independent of the oracle's code: closed forms, torch routines, brute force
and invariants.  At least one of them must fail, or the pins would not
catch that mistake.  Everything runs on the CPU.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qsa_oracle.c")

ATTEND_SCORE = """        if (j > t) continue;
        acc_t dot = 0;
        for (int e = 0; e < D; ++e) dot += (acc_t)qh[e] * (acc_t)kg[j * D + e];
        acc_t sj"""
ATTEND_GROUP = """    int g = h / hpg;
    const float* qh = q + (int64_t)h * D;
    const float* kg"""

MUTANTS = {
    # bf16 rounding: truncation instead of round-to-nearest-even
    "bf16_truncates": ("u += 0x7fffu + keep_lsb;", "u += 0u * keep_lsb;"),
    # rotary encoding
    "rope_sign": ("out[i] = ac - bs;", "out[i] = ac + bs;"),
    "rope_partner_sign": ("out[i + half] = bc + as;", "out[i + half] = bc - as;"),
    "rope_theta_denominator": ("-(2.0 * (double)i) / (double)c->rope_dims", "-(2.0 * (double)i) / (double)c->idx_dim"),
    # pooling
    "pool_sum_not_mean": ("mean[j] = s / (float)r;", "mean[j] = s;"),
    "pool_rope_at_block_end": ("qsa_ref_rope_vec(c, mean, b * r, khat", "qsa_ref_rope_vec(c, mean, b * r + r - 1, khat"),
    # scores
    "query_not_rotated": ("qsa_ref_rope_vec(c, q_idx + h * d, t, qr + h * d);",
                          "qsa_ref_rope_vec(c, q_idx + h * d, 0, qr + h * d);"),
    "score_without_relu": ("acc_t relu = dot > 0 ? dot : 0;", "acc_t relu = dot;"),
    "score_without_head_weight": ("total += (acc_t)w[h] * relu;", "total += relu;"),
    # selection
    "ties_toward_higher_index": ("return (a->b < b->b) ? -1 : (a->b > b->b);",
                                 "return (a->b > b->b) ? -1 : (a->b < b->b);"),
    "one_candidate_short": ("for (int i = 0; i < S - 1; ++i) sel[n++]", "for (int i = 0; i < S - 2; ++i) sel[n++]"),
    # attention
    "causal_bound_strict": (ATTEND_SCORE, ATTEND_SCORE.replace("if (j > t)", "if (j >= t)")),
    "attention_without_scale": ("acc_t sj = (acc_t)c->softmax_scale * dot;", "acc_t sj = dot;"),
    "group_by_modulo": (ATTEND_GROUP, ATTEND_GROUP.replace("h / hpg", "h % G")),
    "lse_without_max": ("if (lse) lse[h] = (double)(m + ACC_LOG(l));", "if (lse) lse[h] = (double)(ACC_LOG(l));"),
    # backward
    "dk_without_scale": ("dk[((int64_t)g * ld + j) * D + e] += (double)(sds * (acc_t)qh[e]);",
                         "dk[((int64_t)g * ld + j) * D + e] += (double)(ds * (acc_t)qh[e]);"),
    "ds_without_delta": ("const acc_t ds = p[i] * (dp[i] - delta);", "const acc_t ds = p[i] * dp[i];"),
    "dv_wrong_operand": ("dv[((int64_t)g * ld + j) * D + e] += (double)(p[i] * (acc_t)doh[e]);",
                         "dv[((int64_t)g * ld + j) * D + e] += (double)(p[i] * (acc_t)qh[e]);"),
}


def _build(src_text, out_dir):
    from oracle import build as obuild
    path = os.path.join(out_dir, "qsa_oracle.c")
    with open(path, "w") as f:
        f.write(src_text)
    for name, extra in obuild.VARIANTS.items():
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-I", os.path.join(ROOT, "oracle"), *extra, path, "-o", os.path.join(out_dir, name), "-lm"]
        subprocess.run(cmd, check=True, capture_output=True)
    return os.path.join(out_dir, "libqsa_oracle.so"), os.path.join(out_dir, "libqsa_oracle_f32.so")


def _run_pins(lib64, lib32):
    env = dict(os.environ, QSA_ORACLE_LIB=lib64, QSA_ORACLE_LIB_F32=lib32)
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                           "-x", "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=600)


def test_unmutated_copy_passes_the_pins():
    """The harness itself: a plain copy built the same way passes."""
    with tempfile.TemporaryDirectory() as d:
        r = _run_pins(*_build(open(SRC).read(), d))
        assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, ("mutation site not found once", name)
    with tempfile.TemporaryDirectory() as d:
        r = _run_pins(*_build(src.replace(old, new), d))
        assert r.returncode != 0, f"{name}: every pin passed\n{r.stdout[-1500:]}"
        assert "failed" in r.stdout or "error" in r.stdout.lower(), r.stdout[-1500:]
