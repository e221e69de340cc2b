"""Helpers for the parity tests: run the CUDA path (through the C ABI) and the
CPU oracle on the same seeded inputs, and compare.

Acceptance (stated in the tests, derived from the method's arithmetic):
  * pooled keys k^: bit-exact (both sides compute the fixed fp32 sequence and
    round to the I/O dtype the same way);
  * scores: |s_gpu - s_ref| <= 2e-5 * max_b |s_ref(t, b)| + 1e-6 per row (fp32
    accumulation of idx_dim bf16 products in a different order);
  * selection: exact, except inside the tie band of the oracle's (S-1)-th
    score s_k: band = 1e-5 * max(|s_k|, |s_k+1|) + 1e-6 * max_b |s_ref|;
    blocks above the band must be kept, blocks below must not, counts equal;
  * outputs: bf16 I/O max-abs <= 2e-2 and mean-abs <= 1e-3; fp32 I/O
    max-abs <= 1e-4; log-sum-exp within 2e-3 (bf16) / 1e-4 (fp32).  A query
    whose selection differs from the oracle's only inside the tie band is
    compared with the oracle's attention over the GPU's own selection.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

import block_sparse_attention_22_b200 as qsa
import oracle
from block_sparse_attention_22_b200 import synth

TOL = {
    "bf16": dict(max_abs=2e-2, mean_abs=1e-3, lse=2e-3),
    "f32": dict(max_abs=1e-4, mean_abs=1e-4, lse=1e-4),
}


def segments_of(wl: synth.Workload):
    return qsa.make_segments([(off, s.q_len, s.pos0, s.slot)
                              for off, s in zip(wl.token_offsets(), wl.segments)])


@dataclass
class GpuRun:
    o: torch.Tensor
    lse: torch.Tensor
    sel: torch.Tensor
    nsel: torch.Tensor
    khat: torch.Tensor


def gpu_prepare_cache(wl: synth.Workload, x: Dict[str, torch.Tensor]):
    """k^ buffer with every slot's cached prefix pooled (the state earlier steps left)."""
    sh = wl.shape
    cfg = qsa.make_config(sh)
    khat = torch.zeros((wl.n_slots, wl.n_cap // sh.r, sh.idx_dim), dtype=sh.torch_dtype, device="cuda")
    cache = qsa.make_cache(x["k_idx"], khat, x["k"], x["v"])
    slots = [s for s in range(wl.n_slots) if wl.cached_blocks[s] > 0]
    if slots:
        qsa.qsa_compress_keys(cfg, cache, slots, [0] * len(slots), [wl.cached_blocks[s] for s in slots])
    return cfg, cache, khat


def gpu_forward(wl: synth.Workload, x: Dict[str, torch.Tensor], lowmem: bool = False) -> GpuRun:
    """One forward call over the workload (qsa_forward_prefixed when it has
    shared prefixes)."""
    sh = wl.shape
    cfg, cache, khat = gpu_prepare_cache(wl, x)
    segs = segments_of(wl)
    T = wl.n_tokens
    o = torch.full((T, sh.n_heads, sh.head_dim), float("nan"), dtype=sh.torch_dtype, device="cuda")
    lse = torch.full((T, sh.n_heads), float("nan"), dtype=torch.float32, device="cuda")
    sel = torch.full((T, sh.budget_blocks), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((T,), -7, dtype=torch.int32, device="cuda")
    if wl.prefix:
        ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, qsa.QSA_OP_FORWARD_PREFIXED)), dtype=torch.uint8,
                         device="cuda")
        qsa.qsa_forward_prefixed(cfg, cache, segs, qsa.make_prefixes(wl.prefix), T, x["q"], x["q_idx"], x["w"], o,
                                 lse, sel, nsel, ws)
        torch.cuda.synchronize()
        qsa.qsa_device_status()
        return GpuRun(o, lse, sel, nsel, khat)
    op = qsa.QSA_OP_FORWARD_LOWMEM if lowmem else qsa.QSA_OP_FORWARD
    ws = torch.empty(max(1, qsa.workspace_size(cfg, segs, T, op)), dtype=torch.uint8, device="cuda")
    fwd = qsa.qsa_forward_lowmem if lowmem else qsa.qsa_forward
    fwd(cfg, cache, segs, T, x["q"], x["q_idx"], x["w"], o, lse, sel, nsel, ws)
    torch.cuda.synchronize()
    qsa.qsa_device_status()
    return GpuRun(o, lse, sel, nsel, khat)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


class OracleSeq:
    """Oracle state of one cache slot: its k^ for every complete block."""

    def __init__(self, wl: synth.Workload, x: Dict[str, torch.Tensor], slot: int):
        self.cfg = oracle.config_from_shape(wl.shape)
        self.r = wl.shape.r
        fill = wl.fill[slot]
        k_idx, k, v = synth.sequence_cache(wl, x, slot, fill)     # with a shared prefix: its rows first
        self.k_idx = to_np(k_idx)
        self.k = to_np(k)
        self.v = to_np(v)
        self.khat = oracle.compress_keys(self.cfg, self.k_idx, 0, fill // self.r)

    def attend(self, q, t, sel, nsel):
        return oracle.attend(self.cfg, q, self.k, self.v, t, np.asarray(sel, dtype=np.int32), nsel)

    def query(self, q, q_idx, w, t):
        s = oracle.index_scores(self.cfg, q_idx, w, t, self.khat)
        sel, n = oracle.select(self.cfg, s, t)
        o, lse = oracle.attend(self.cfg, q, self.k, self.v, t, sel, n)
        return dict(scores=s, sel=sel, nsel=n, o=o, lse=lse)


def selection_verdict(s_ref: np.ndarray, sel_ref, n_ref: int, sel_gpu, n_gpu: int, t: int, S: int,
                      r: int = 4) -> str:
    """'exact', 'band' (differs only inside the tie band) or raises AssertionError."""
    bt = t // r
    sel_gpu = np.asarray(sel_gpu)
    assert n_gpu == n_ref == min(S, bt + 1), (t, n_gpu, n_ref)
    assert (sel_gpu[n_gpu:] == -1).all(), (t, sel_gpu[n_gpu:])
    assert sel_gpu[n_gpu - 1] == bt, (t, sel_gpu[n_gpu - 1])
    assert (np.diff(sel_gpu[:n_gpu]) > 0).all(), t
    if list(sel_gpu[:n_gpu]) == list(sel_ref[:n_ref]):
        return "exact"
    assert bt + 1 > S, (t, "short rows keep every block")
    K = S - 1
    order = np.lexsort((np.arange(bt), -s_ref))
    s_k = s_ref[order[K - 1]]
    s_k1 = s_ref[order[K]] if bt > K else s_k
    band = 1e-5 * max(abs(s_k), abs(s_k1)) + 1e-6 * float(np.abs(s_ref).max())
    kept = set(int(b) for b in sel_gpu[:K])
    assert len(kept) == K
    above = np.nonzero(s_ref > s_k + band)[0]
    below = np.nonzero(s_ref < s_k - band)[0]
    missing = [int(b) for b in above if int(b) not in kept]
    extra = [int(b) for b in below if int(b) in kept]
    assert not missing and not extra, (t, "outside tie band", missing[:5], extra[:5], s_k, band)
    return "band"


def check_outputs(o_gpu: np.ndarray, o_ref: np.ndarray, lse_gpu: Optional[np.ndarray],
                  lse_ref: Optional[np.ndarray], dtype: str, what: str = ""):
    tol = TOL[dtype]
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    assert np.isfinite(o_gpu).all(), what
    assert err.max() <= tol["max_abs"], (what, "max-abs", float(err.max()))
    assert err.mean() <= tol["mean_abs"], (what, "mean-abs", float(err.mean()))
    if lse_gpu is not None:
        lerr = np.abs(lse_gpu.astype(np.float64) - lse_ref)
        assert lerr.max() <= tol["lse"], (what, "lse", float(lerr.max()))
    return float(err.max()), float(err.mean())


def compare_forward(wl: synth.Workload, x: Dict[str, torch.Tensor], run: GpuRun,
                    tokens: Optional[Sequence[int]] = None, min_exact: float = 0.99) -> Dict:
    """Compare sampled (or all) tokens of a forward run against the oracle."""
    sh = wl.shape
    S = sh.budget_blocks
    offs = wl.token_offsets()
    pos = wl.token_positions().numpy()
    slots = wl.token_slots().numpy()
    if tokens is None:
        tokens = range(wl.n_tokens)
    tokens = sorted(set(int(i) for i in tokens))
    seqs: Dict[int, OracleSeq] = {}
    sel_gpu = run.sel.cpu().numpy()
    nsel_gpu = run.nsel.cpu().numpy()
    q = x["q"][tokens].float().cpu().numpy()
    qi = x["q_idx"][tokens].float().cpu().numpy()
    w = x["w"][tokens].float().cpu().numpy()
    o_gpu = to_np(run.o[tokens])
    lse_gpu = to_np(run.lse[tokens])
    verdicts = {"exact": 0, "band": 0}
    o_ref = np.zeros(o_gpu.shape)
    lse_ref = np.zeros(lse_gpu.shape)
    same = np.zeros(len(tokens), bool)
    for n, i in enumerate(tokens):
        slot = int(slots[i])
        if slot not in seqs:
            seqs.clear()                      # one sequence's host copies at a time
            seqs[slot] = OracleSeq(wl, x, slot)
        ref = seqs[slot].query(q[n], qi[n], w[n], int(pos[i]))
        v = selection_verdict(ref["scores"], ref["sel"], ref["nsel"], sel_gpu[i], int(nsel_gpu[i]),
                              int(pos[i]), S, sh.r)
        verdicts[v] += 1
        same[n] = v == "exact"
        o_ref[n] = ref["o"]
        lse_ref[n] = ref["lse"]
        if v == "band":
            # the kept sets differ legitimately inside the tie band: compare with
            # the oracle's attention over the GPU's own selection instead
            o_ref[n], lse_ref[n] = seqs[slot].attend(q[n], int(pos[i]), sel_gpu[i], int(nsel_gpu[i]))
    frac = verdicts["exact"] / max(1, len(tokens))
    assert frac >= min_exact, verdicts
    mx, mean = check_outputs(o_gpu, o_ref, lse_gpu, lse_ref, sh.dtype, wl.name)
    return dict(verdicts=verdicts, max_abs=mx, mean_abs=mean, n=len(tokens))


def sample_tokens(wl: synth.Workload, every: int, extra: Sequence[int] = ()) -> List[int]:
    """Every `every`-th token, the first and last 8 of each segment, and needle targets."""
    out = set(extra)
    for off, s in zip(wl.token_offsets(), wl.segments):
        out.update(range(off, off + s.q_len, every))
        out.update(range(off, off + min(8, s.q_len)))
        out.update(range(off + max(0, s.q_len - 8), off + s.q_len))
    for (slot, t, b) in wl.needles:
        for off, s in zip(wl.token_offsets(), wl.segments):
            if s.slot == slot and s.pos0 <= t < s.pos0 + s.q_len:
                out.add(off + t - s.pos0)
    return sorted(out)
