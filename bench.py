#!/usr/bin/env python
"""Benchmark of the QSA forward pass on B200 (one JSON line on rank 0).

A step is one qsa_forward over the workload's batch: pooling of the blocks
the batch completes, indexer scores, top-k selection and sparse attention.
Default workload: 128K-token prefill (1 sequence x 131072 tokens, bf16, 24
heads / 2 KV groups, head dim 256, 4-head indexer of dim 128, r = 4, budget
2048 tokens, needles every 8192 positions).  Two 1M-context steps are
measured in the same run and reported beside the main line: "decode_1m"
(8 decode queries, each against its own 1048576-token cache) and "mixed_1m"
(the same decode queries plus a 4096-query chunk of a 90%-cached sequence).

Inputs are synthetic (seeded, N(0,1) with planted needles) and resident in
HBM before the timed region; L2 is flushed (a 256 MiB write, then a 256 MiB
read so that no dirty line is left for the step to write back; outside the
timed events) before every timed step.  Times are CUDA events on the
launching stream, max over ranks.  With torchrun and N > 1 every rank runs
an independent replica of the workload on its own GPU (the method has no
cross-GPU exchange): scaling is weak.

Besides the main line's device-timed step the JSON line carries: "stages"
(each public entry point timed alone) and the attention "roofline" (gathered
bytes over the attention stage, DRAM traffic from the committed ncu record);
"e2e" (the step through qsa_forward with every input copied from pinned host
memory and the output copied back inside the timed region, as 8 chunked-
prefill calls whose copies overlap the neighbouring chunks' compute; output
checked equal to one call); "lowmem_forward" (the same step through
qsa_forward_lowmem, with both workspace sizes); "decode_1m" / "mixed_1m";
"attn_backward" (qsa_sparse_attn_bwd on a 2 x 8192-token prefill);
"attn_union" (the attention of prefill_128k_local, whose indexer queries drift
along the sequence, on union tiles of neighbouring queries beside the
per-query path);
"cpu_baseline" (the oracle on a bounded sample); "gpu_launches"; "clocks";
"tensor_roofline" (the step's flops over its time against the bf16 peak, the
index stage alone, and the attainable step time).  Side lines "decode_256k"
and "prefill_8k" (the 256K-context decode batch and the 2 x 8K prefill) carry
their own CPU oracle timing.  Each side line's "hbm_roofline" counts the
algorithmic bytes only (no score round trip), with the bytes the
score-matrix path actually moves beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qsa|reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import block_sparse_attention_22_b200 as qsa  # noqa: E402
from block_sparse_attention_22_b200 import synth  # noqa: E402

METRIC = "QSA fwd tokens/s (prefill 128K, decode 1M ctx); % of HBM/tensor roofline"
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock/throttle samples of this process's GPU during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.target = None

    def start(self):
        if self.target is None:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ workload set-up
class Prepared:
    """Device-resident inputs, caches, outputs and workspace of one workload."""

    def __init__(self, wl: synth.Workload):
        self.wl = wl
        sh = wl.shape
        self.sh = sh
        self.x = synth.make_inputs(wl, device="cuda")
        self.cfg = qsa.make_config(sh)
        self.khat = torch.zeros((wl.n_slots, wl.n_cap // sh.r, sh.idx_dim), dtype=sh.torch_dtype, device="cuda")
        self.cache = qsa.make_cache(self.x["k_idx"], self.khat, self.x["k"], self.x["v"])
        slots = [s for s in range(wl.n_slots) if wl.cached_blocks[s] > 0]
        if slots:   # the cached prefix: pooled by earlier steps, not part of this step
            qsa.qsa_compress_keys(self.cfg, self.cache, slots, [0] * len(slots),
                                  [wl.cached_blocks[s] for s in slots])
        self.segl = [(off, s.q_len, s.pos0, s.slot) for off, s in zip(wl.token_offsets(), wl.segments)]
        self.segs = qsa.make_segments(self.segl)
        T = self.T = wl.n_tokens
        self.o = torch.empty((T, sh.n_heads, sh.head_dim), dtype=sh.torch_dtype, device="cuda")
        self.lse = torch.empty((T, sh.n_heads), dtype=torch.float32, device="cuda")
        self.sel = torch.empty((T, sh.budget_blocks), dtype=torch.int32, device="cuda")
        self.nsel = torch.empty((T,), dtype=torch.int32, device="cuda")
        self.ld = max(4, math.ceil(max((p + n - 1) // sh.r for _, n, p, _ in self.segl) / 4) * 4)
        self.ranges = step_ranges(wl)
        self._bufs = {}
        self.prefixes = qsa.make_prefixes(wl.prefix) if wl.prefix else None

    # workspaces and the score matrix, allocated on first use (a profiling run of
    # one stage holds only what that stage needs)
    def _ws(self, op):
        if op not in self._bufs:
            self._bufs[op] = torch.empty(max(1, qsa.workspace_size(self.cfg, self.segs, self.T, op)),
                                         dtype=torch.uint8, device="cuda")
        return self._bufs[op]

    @property
    def ws(self):
        return self._ws(qsa.QSA_OP_FORWARD)

    @property
    def ws_low(self):
        return self._ws(qsa.QSA_OP_FORWARD_LOWMEM)

    @property
    def ws_sel(self):
        return self._ws(qsa.QSA_OP_SELECT)

    @property
    def ws_attn(self):
        return self._ws(qsa.QSA_OP_ATTN)

    @property
    def scores(self):
        if "scores" not in self._bufs:
            self._bufs["scores"] = torch.empty((self.T, self.ld), dtype=torch.float32, device="cuda")
        return self._bufs["scores"]

    def workspace_bytes(self, lowmem: bool) -> int:
        op = qsa.QSA_OP_FORWARD_LOWMEM if lowmem else qsa.QSA_OP_FORWARD
        return qsa.workspace_size(self.cfg, self.segs, self.T, op)

    def forward(self, lowmem: bool = False):
        x = self.x
        if self.wl.prefix:
            qsa.qsa_forward_prefixed(self.cfg, self.cache, self.segs, self.prefixes, self.T, x["q"], x["q_idx"],
                                     x["w"], self.o, self.lse, self.sel, self.nsel,
                                     self._ws(qsa.QSA_OP_FORWARD_PREFIXED))
        elif lowmem:
            qsa.qsa_forward_lowmem(self.cfg, self.cache, self.segs, self.T, x["q"], x["q_idx"], x["w"], self.o,
                                   self.lse, self.sel, self.nsel, self.ws_low)
        else:
            qsa.qsa_forward(self.cfg, self.cache, self.segs, self.T, x["q"], x["q_idx"], x["w"], self.o, self.lse,
                            self.sel, self.nsel, self.ws)

    # the same four calls qsa_forward makes, one public entry point each
    def stage(self, i):
        x = self.x
        if i == 0:
            qsa.qsa_compress_keys(self.cfg, self.cache, [r[0] for r in self.ranges], [r[1] for r in self.ranges],
                                  [r[2] for r in self.ranges])
        elif i == 1:
            qsa.qsa_index_scores(self.cfg, self.cache, self.segs, self.T, x["q_idx"], x["w"], self.scores, self.ld)
        elif i == 2:
            qsa.qsa_select_topk(self.cfg, self.segs, self.T, self.scores, self.ld, self.sel, self.nsel, self.ws_sel)
        else:
            qsa.qsa_sparse_attn_fwd(self.cfg, self.cache, self.segs, self.T, x["q"], self.sel, self.nsel, self.o,
                                    self.lse, self.ws_attn)

    def work(self):
        return algorithmic_work(self.wl)


def step_ranges(wl: synth.Workload):
    """(slot, first block, end block) of the blocks each segment completes."""
    r = wl.shape.r
    return [(s.slot, s.pos0 // r, (s.pos0 + s.q_len) // r) for s in wl.segments]


def algorithmic_work(wl: synth.Workload):
    """Algorithmic bytes / flops of each stage for this batch (what QSA must touch)."""
    sh = wl.shape
    T = wl.n_tokens
    pos = wl.token_positions().double()
    bt = torch.floor(pos / sh.r)
    nsel = torch.clamp(bt + 1, max=sh.budget_blocks)
    el = 2 if sh.dtype == "bf16" else 4
    D, H, G, DI, HI = sh.head_dim, sh.n_heads, sh.n_groups, sh.idx_dim, sh.idx_heads
    n_new_blocks = sum(b1 - b0 for _, b0, b1 in step_ranges(wl))
    comp_bytes = n_new_blocks * (sh.r + 1) * DI * el
    cand = bt.sum().item()
    idx_flops = 2.0 * HI * DI * cand
    # scores: score writes + query rows; k^ of prefill-like segments (64-query tiles) is
    # L2-resident, while decode-like segments (< 16 queries, 4-query tiles) stream their
    # sequence's k^ from HBM once per tile of 4 consecutive queries
    idx_q = T * HI * (DI * el + 4)
    idx_khat = 0.0
    shared = {}
    for i, s in enumerate(wl.segments):
        pb = wl.prefix[i][1] if wl.prefix else 0
        if pb > 0:                      # its own blocks here; the prefix's once per 16 sharing queries, below
            shared[wl.prefix[i]] = shared.get(wl.prefix[i], 0) + s.q_len
        if s.q_len < 16:
            for q0 in range(0, s.q_len, 4):
                t_last = s.pos0 + min(q0 + 4, s.q_len) - 1
                idx_khat += (t_last // sh.r - pb) * DI * el
    for (_, pb), m in shared.items():
        idx_khat += math.ceil(m / 16) * pb * DI * el
    score_bytes = cand * 4                     # the fp32 score matrix, written once and read once
    idx_bytes = score_bytes + idx_q + idx_khat
    sel_out = T * (sh.budget_blocks + 1) * 4
    sel_bytes = score_bytes + sel_out
    gathered = float((nsel * sh.r).sum().item()) * G * D * el * 2
    attn_bytes = gathered + T * H * D * el * 2 + T * H * 4 + T * (sh.budget_blocks + 1) * 4
    attn_flops = 4.0 * H * D * float((nsel * sh.r).sum().item())
    # what the method must touch (no score round trip; the selection's algorithmic
    # bytes are 0 when it is fused with the scoring): pooling, the k^ stream of
    # decode-like queries, query rows, kept K/V rows, q/o/lse and sel
    alg = comp_bytes + idx_q + idx_khat + sel_out + attn_bytes
    return dict(compress=dict(bytes=comp_bytes),
                index=dict(bytes=idx_bytes, flops=idx_flops, khat_bytes=idx_khat, query_bytes=idx_q,
                           score_bytes=score_bytes),
                select=dict(bytes=sel_bytes), attn=dict(bytes=attn_bytes, flops=attn_flops, gathered_bytes=gathered),
                algorithmic_bytes=alg, actual_bytes=comp_bytes + idx_bytes + sel_bytes + attn_bytes,
                flops=idx_flops + attn_flops)


class L2Flush:
    """Empties L2 between timed steps: a write of a buffer larger than L2, then
    a read of another one, so the step starts with no useful line in L2 and
    without a cache full of dirty lines whose write-back it would pay for."""

    def __init__(self, nbytes: int = L2_FLUSH_BYTES):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device="cuda")
        self.sink = torch.empty((), dtype=torch.float32, device="cuda")

    def zero_(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def timed(prep: Prepared, steps: int, warmup: int, flush: L2Flush, staged: bool, lowmem: bool = False):
    """Device time of `steps` steps (ms each), L2 flushed before every step."""
    st = torch.cuda.current_stream()
    n_ev = 5 if staged else 2
    for _ in range(warmup):
        flush.zero_()
        if staged:
            for i in range(4):
                prep.stage(i)
        else:
            prep.forward(lowmem)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    launches0 = qsa.launch_count()
    for s in range(steps):
        flush.zero_()
        evs[s][0].record(st)
        if staged:
            for i in range(4):
                prep.stage(i)
                evs[s][i + 1].record(st)
        else:
            prep.forward(lowmem)
            evs[s][1].record(st)
    torch.cuda.synchronize()
    launches = qsa.launch_count() - launches0
    per = [[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(n_ev - 1)] for s in range(steps)]
    return per, launches


def e2e_prefill(prep: Prepared, steps: int, warmup: int, n_chunks: int = 8):
    """The prefill step end to end through the public API: every step's inputs
    are copied from pinned host memory and its output read back, all inside the
    timed region.  A step runs as n_chunks chunked-prefill calls of qsa_forward
    (query rows [r0, r1) at positions [r0, r1), each call pooling its own blocks
    over the prefix the earlier calls pooled: the same results as one call), so
    the upload of chunk j+1 and the download of chunk j-1 overlap chunk j's
    compute.  Three streams (copy-in, compute, copy-out) and two device buffer
    sets let consecutive steps overlap the same way."""
    x, wl = prep.x, prep.wl
    assert len(wl.segments) == 1 and wl.segments[0].pos0 == 0, "a prefill from position 0"
    o_single = prep.o.cpu()                           # the single-call output of the device-timed steps
    slot = wl.segments[0].slot
    T = prep.T
    G = prep.sh.n_groups
    host = {"q": x["q"].cpu().pin_memory(), "q_idx": x["q_idx"].cpu().pin_memory(), "w": x["w"].cpu().pin_memory(),
            "k_idx": x["k_idx"][slot, :T].cpu().pin_memory(), "k": x["k"][slot, :, :T].cpu().pin_memory(),
            "v": x["v"][slot, :, :T].cpu().pin_memory()}
    o_host = torch.empty(prep.o.shape, dtype=prep.o.dtype).pin_memory()
    lse_host = torch.empty(prep.lse.shape, dtype=prep.lse.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * lse_host.element_size()
    C = -(-T // n_chunks)
    C = -(-C // 64) * 64
    chunks = [(r0, min(T, r0 + C)) for r0 in range(0, T, C)]
    chunk_segs = [qsa.make_segments([(r0, r1 - r0, r0, slot)]) for r0, r1 in chunks]

    def pieces(d, r0, r1):
        out = [(d["q"][r0:r1], host["q"][r0:r1]), (d["q_idx"][r0:r1], host["q_idx"][r0:r1]),
               (d["w"][r0:r1], host["w"][r0:r1]), (d["k_idx"][slot, r0:r1], host["k_idx"][r0:r1])]
        for g in range(G):
            out += [(d["k"][slot, g, r0:r1], host["k"][g, r0:r1]), (d["v"][slot, g, r0:r1], host["v"][g, r0:r1])]
        return out

    # two device buffer sets (inputs, caches, outputs); the score workspace is shared
    sets = []
    for b in range(2):
        d = x if b == 0 else {k: torch.empty_like(v) for k, v in x.items()}
        khat = prep.khat if b == 0 else torch.empty_like(prep.khat)
        o = prep.o if b == 0 else torch.empty_like(prep.o)
        lse = prep.lse if b == 0 else torch.empty_like(prep.lse)
        sets.append(dict(d=d, khat=khat, o=o, lse=lse, cache=qsa.make_cache(d["k_idx"], khat, d["k"], d["v"])))
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    nc = len(chunks)
    in_done = [[torch.cuda.Event() for _ in range(nc)] for _ in range(2)]
    cmp_done = [[torch.cuda.Event() for _ in range(nc)] for _ in range(2)]
    out_done = [[torch.cuda.Event() for _ in range(nc)] for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i & 1
        st_ = sets[b]
        d = st_["d"]
        for j, (r0, r1) in enumerate(chunks):
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(cmp_done[b][j])      # compute of step i-2 is done with these rows
                for dst, src in pieces(d, r0, r1):
                    dst.copy_(src, non_blocking=True)
                in_done[b][j].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_done[b][j])
                if used[b]:
                    s_cmp.wait_event(out_done[b][j])     # download of step i-2 has read these output rows
                qsa.qsa_forward(prep.cfg, st_["cache"], chunk_segs[j], T, d["q"], d["q_idx"], d["w"], st_["o"],
                                st_["lse"], prep.sel, prep.nsel, prep.ws, stream=s_cmp)
                cmp_done[b][j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b][j])
                o_host[r0:r1].copy_(st_["o"][r0:r1], non_blocking=True)
                lse_host[r0:r1].copy_(st_["lse"][r0:r1], non_blocking=True)
                out_done[b][j].record(s_out)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    s_cmp.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(warmup, warmup + steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    ok = bool(torch.equal(o_host, o_single))
    del sets
    return e0.elapsed_time(e1) / steps, h2d, d2h, nc, ok


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(wl: synth.Workload, x, target_s: float = 10.0, max_slots: int = 0, phase: float = 0.0):
    """Time the CPU oracle on a stratified sample of the workload's queries and
    extrapolate to the whole batch (per-query work grows linearly with the
    position, so evenly spaced positions give an unbiased mean; `phase` in
    [0, 1) shifts the evenly spaced picks).  With max_slots > 0 only that many
    cache slots are timed (evenly spaced) and the estimate is scaled by the
    query count of all slots (for batches of like sequences whose caches
    would not all fit in host memory).  Returns (tokens/s, threads,
    description)."""
    import oracle
    sh = wl.shape
    cfg = oracle.config_from_shape(sh)
    threads = len(os.sched_getaffinity(0))
    pos_all = wl.token_positions().numpy()
    f = lambda t: t.float().cpu().numpy()
    # per slot: pooled-key cost once (all blocks the queries need), then queries
    total_s, n_done, desc = 0.0, 0, []
    seg_rows = {}
    for off, s in zip(wl.token_offsets(), wl.segments):
        seg_rows.setdefault(s.slot, []).extend(range(off, off + s.q_len))
    all_rows = sum(len(r) for r in seg_rows.values())
    if max_slots and len(seg_rows) > max_slots:
        keys = sorted(seg_rows)
        keep = [keys[i] for i in np.linspace(0, len(keys) - 1, max_slots).astype(int)]
        seg_rows = {k: seg_rows[k] for k in keep}
    timed_rows = sum(len(r) for r in seg_rows.values())

    def picks(rows, n):
        if n >= len(rows):
            return rows
        return rows[np.minimum(len(rows) - 1, ((np.arange(n) + phase) * len(rows) / n).astype(int))]

    budget_per_slot = target_s / max(1, len(seg_rows))
    est_total = 0.0
    for slot, rows in seg_rows.items():
        fill = wl.fill[slot]
        k_idx = f(x["k_idx"][slot, :fill])
        k = f(x["k"][slot, :, :fill])
        v = f(x["v"][slot, :, :fill])
        rows = np.array(rows)
        nb_new = sum((s.pos0 + s.q_len) // sh.r - s.pos0 // sh.r for s in wl.segments if s.slot == slot)
        t0 = time.perf_counter()
        oracle.compress_keys(cfg, k_idx, 0, max(1, nb_new))     # the blocks this step pools
        t_comp = time.perf_counter() - t0
        # calibrate with a few queries, then size the sample to the budget
        n_cal = min(len(rows), max(2, threads))
        pick = rows[np.linspace(0, len(rows) - 1, n_cal).astype(int)]
        t0 = time.perf_counter()
        oracle.forward(cfg, f(x["q"][pick]), f(x["q_idx"][pick]), f(x["w"][pick]), pos_all[pick], k_idx, k, v)
        t_cal = time.perf_counter() - t0
        n_s = int(min(len(rows), max(n_cal, n_cal * budget_per_slot / max(t_cal, 1e-3))))
        pick = picks(rows, n_s)
        t0 = time.perf_counter()
        oracle.forward(cfg, f(x["q"][pick]), f(x["q_idx"][pick]), f(x["w"][pick]), pos_all[pick], k_idx, k, v)
        t_s = time.perf_counter() - t0
        # oracle.forward also pools every block up to max(pick); remove that part once
        t0 = time.perf_counter()
        oracle.compress_keys(cfg, k_idx, 0, int(pos_all[pick].max()) // sh.r)
        t_pool_all = time.perf_counter() - t0
        per_query = max(t_s - t_pool_all, 1e-9) / n_s
        est_total += t_comp + per_query * len(rows)
        total_s += t_s + t_comp
        n_done += n_s
        desc.append(f"slot {slot}: {n_s} of {len(rows)} queries" +
                    (" (all)" if n_s == len(rows) else " at evenly spaced positions"))
    est_total *= all_rows / timed_rows
    tokens = wl.n_tokens
    slots_note = (f"{len(seg_rows)} of {len(set(s.slot for s in wl.segments))} sequences timed; "
                  if timed_rows < all_rows else "")
    return tokens / est_total, threads, slots_note + "; ".join(desc) + \
        f"; {total_s:.1f} s of oracle wall time, extrapolated by query count (pooling of the step's new " \
        f"blocks timed in full)"


# ------------------------------------------------------------------ main
def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank


def max_over_ranks(v: float, ws: int, device: str = "cuda") -> float:
    """Max of a per-rank value over all ranks (device timing: the slowest replica)."""
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, slowest_ms: float, ws: int) -> float:
    """Whole-job tokens/s: every rank runs its own replica, timed by the slowest."""
    return ws * tokens_per_rank / (slowest_ms * 1e-3)


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def measure(prep: Prepared, steps, warmup, ws, flush, peaks, clocks=None):
    barrier(ws)
    if clocks:
        clocks.start()
    per, launches = timed(prep, steps, warmup, flush, staged=False)
    if clocks:
        clk = clocks.stop()
    else:
        clk = None
    barrier(ws)
    fused_ms = sum(p[0] for p in per) / steps
    fused_ms = max_over_ranks(fused_ms, ws)
    work = prep.work()
    names = ["compress", "index", "select", "attn"]
    stages = {}
    if prep.wl.prefix:          # the per-stage entry points take no shared prefixes: the fused step only
        return dict(fused_ms=fused_ms, stage_ms=None, stages=None, work=work, launches=launches, clocks=clk)
    per_s, launches_s = timed(prep, steps, max(1, warmup // 2), flush, staged=True)
    barrier(ws)
    stage_ms = [sum(p[i] for p in per_s) / steps for i in range(4)]
    for n, ms in zip(names, stage_ms):
        d = {"ms": ms}
        if "bytes" in work[n]:
            d["gbs"] = work[n]["bytes"] / (ms * 1e-3) / 1e9
            d["hbm_frac"] = d["gbs"] / peaks["hbm_gbs"]
        if "flops" in work[n]:
            d["tflops"] = work[n]["flops"] / (ms * 1e-3) / 1e12
            d["tensor_frac"] = d["tflops"] / peaks["bf16_tflops"]
        stages[n] = d
    return dict(fused_ms=fused_ms, stage_ms=stage_ms, stages=stages, work=work, launches=launches,
                clocks=clk)


def measure_backward(name, steps, warmup, ws, flush, peaks):
    """qsa_sparse_attn_bwd on one workload: the forward runs once for o, lse and
    the selection; each timed step zeroes dk/dv (outside the events) and runs the
    backward.  Algorithmic work per (query, group, kept key): five dot products
    of head_dim per head (scores, dp, and the dq, dk, dv contributions), the K
    and V rows read (2 x 256 x 2 B) and the dK and dV rows accumulated (read and
    written: 2 x 2 x 256 x 4 B).  bf16 runs on tensor cores and streams that
    traffic: roofline against the HBM copy peak (tensor fraction alongside);
    fp32 runs on CUDA cores: roofline against the fp32 FMA peak from the unit
    count and clock (148 SMs x 128 lanes x 2 flop x 1.965 GHz)."""
    wl = synth.make_workload(name)
    prep = Prepared(wl)
    prep.forward()
    sh, x = prep.sh, prep.x
    T = prep.T
    g = torch.Generator(device="cuda").manual_seed(31)
    dout = torch.randn((T, sh.n_heads, sh.head_dim), generator=g, device="cuda").to(sh.torch_dtype)
    dq = torch.empty((T, sh.n_heads, sh.head_dim), dtype=torch.float32, device="cuda")
    dk = torch.zeros(x["k"].shape, dtype=torch.float32, device="cuda")
    dv = torch.zeros(x["v"].shape, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()

    def step():
        qsa.qsa_sparse_attn_bwd(prep.cfg, prep.cache, prep.segs, T, x["q"], prep.o, prep.lse, dout, prep.sel,
                                prep.nsel, dq, dk, dv)

    for _ in range(warmup):
        dk.zero_()
        dv.zero_()
        flush.zero_()
        step()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        dk.zero_()
        dv.zero_()
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        step()
        e1.record(st)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = max_over_ranks(sum(times) / steps, ws)
    pos = wl.token_positions().double()
    keys = float((torch.clamp(torch.floor(pos / sh.r) + 1, max=sh.budget_blocks) * sh.r).sum().item())
    flops = 10.0 * sh.head_dim * sh.n_heads * keys
    tflops = flops / (ms * 1e-3) / 1e12
    D, H, G = sh.head_dim, sh.n_heads, sh.n_groups
    del prep
    torch.cuda.empty_cache()
    out = {"workload": name, "ms_per_step": ms, "tokens_per_s": job_throughput(T, ms, ws)}
    if sh.dtype == "bf16":
        nbytes = keys * G * (2 * D * 2 + 2 * 2 * D * 4) + T * H * (3 * D * 2 + D * 4 + 4)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out["roofline"] = {"bound": "gather (L2/HBM)", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": nbytes,
                           "peak_source": peaks["source"], "tflops": tflops,
                           "tensor_frac": tflops / peaks["bf16_tflops"],
                           "basis": "kept K/V rows read and dK/dV rows read and written, as logical bytes over "
                                    "the HBM copy peak; the two sequences' K/V and dK/dV (about 100 MB) stay "
                                    "in L2, so DRAM moves a small part of it"}
    else:
        peak = 148 * 128 * 2 * 1.965e9 / 1e12
        out["roofline"] = {"bound": "alu", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                           "peak_source": "fp32 FMA lanes x clock (148 x 128 x 2 x 1.965 GHz)"}
    return out


def union_lengths(sel: torch.Tensor, nsel: torch.Tensor, segl, mq: int) -> torch.Tensor:
    """Distinct kept blocks of every tile of mq consecutive queries of a segment
    (computed here with a sort, independently of the library's union lists)."""
    out = []
    S = sel.shape[1]
    cols = torch.arange(S, device=sel.device)
    for off, q_len, _, _ in segl:
        s = sel[off:off + q_len].clone()
        s[cols[None, :] >= nsel[off:off + q_len, None]] = -1
        pad = (-q_len) % mq
        if pad:
            s = torch.cat([s, torch.full((pad, S), -1, dtype=s.dtype, device=s.device)])
        s = torch.sort(s.view(-1, mq * S), dim=1).values
        new = torch.ones_like(s, dtype=torch.bool)
        new[:, 1:] = s[:, 1:] != s[:, :-1]
        out.append((new & (s >= 0)).sum(1))
    return torch.cat(out)


def measure_union(name, steps, warmup, ws, flush, peaks, n=None):
    """The attention stage of one workload on union tiles
    (qsa_sparse_attn_fwd_union) beside the per-query path (qsa_sparse_attn_fwd),
    both over the selection the forward made, L2 flushed before every step.
    Algorithmic bytes of the union path: per tile and KV group the union's K and
    V rows (2 x r x head_dim x 2 B per block), plus Q read and O written
    (H x head_dim x 2 B each per query), lse, the sel rows read and the union
    lists written and read (8 B per entry, twice).  `n`: a shorter prefill of the
    same recipe (profiles)."""
    wl = synth.make_workload(name, **({"n": n} if n else {}))
    prep = Prepared(wl)
    prep.forward()
    torch.cuda.synchronize()
    sh, x, T = prep.sh, prep.x, prep.T
    mq = min(32, 128 // (sh.n_heads // sh.n_groups))
    o_ref = prep.o.clone()
    o_u = torch.empty_like(prep.o)
    lse_u = torch.empty_like(prep.lse)
    ws_u = torch.empty(max(1, qsa.workspace_size(prep.cfg, prep.segs, T, qsa.QSA_OP_ATTN_UNION)),
                       dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream()

    def per_query():
        prep.stage(3)

    def union():
        qsa.qsa_sparse_attn_fwd_union(prep.cfg, prep.cache, prep.segs, T, x["q"], prep.sel, prep.nsel, o_u, lse_u,
                                      ws_u)

    def time_of(fn):
        for _ in range(warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(st)
            fn()
            e1.record(st)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        return max_over_ranks(tot / steps, ws)

    n0 = qsa.launch_count()
    ms_u = time_of(union)
    launches = (qsa.launch_count() - n0) // (steps + warmup)
    ms_q = time_of(per_query)
    diff = float((o_u.float() - o_ref.float()).abs().max().item())
    lens = union_lengths(prep.sel, prep.nsel, prep.segl, mq).double()
    el = 2
    D, H, G = sh.head_dim, sh.n_heads, sh.n_groups
    blocks_u = float(lens.sum().item())
    blocks_q = float(prep.nsel.double().sum().item())
    gathered_u = blocks_u * G * sh.r * D * el * 2
    gathered_q = blocks_q * G * sh.r * D * el * 2
    nbytes = gathered_u + T * H * D * el * 2 + T * H * 4 + T * sh.budget_blocks * 4 + blocks_u * 16
    gbs = nbytes / (ms_u * 1e-3) / 1e9
    out = {"workload": name, "drift": wl.drift, "tile_queries": mq, "ms_union": ms_u, "ms_per_query": ms_q,
           "speedup": ms_q / ms_u, "tokens_per_s_union": job_throughput(T, ms_u, ws),
           "union_blocks_per_tile": blocks_u / len(lens), "kept_blocks_per_query": blocks_q / T,
           "gathered_bytes_union": gathered_u, "gathered_bytes_per_query": gathered_q,
           "max_abs_diff_vs_per_query": diff, "gpu_launches_per_call": launches,
           "roofline": {"bound": "gather (L2/HBM)", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": gbs / peaks["hbm_gbs"], "bytes_per_launch": nbytes, "peak_source": peaks["source"],
                        "basis": "union K/V rows gathered once per tile and group, as logical bytes over the "
                                 "HBM copy peak; neighbouring tiles share blocks, so most gathers hit L2"}}
    del prep
    torch.cuda.empty_cache()
    return out


KERNEL_SOURCES = {
    "attn": ["attn_tc.cuh", "sm100.cuh", "qsa_internal.cuh"],
    "index": ["index_tc.cuh", "sm100.cuh", "qsa_internal.cuh"],
    "select": ["topk.cuh", "sm100.cuh", "qsa_internal.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha1()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "block_sparse_attention_22_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, alg_bytes: float):
    """DRAM bytes per launch from the committed ncu record of this kernel build
    (profiles/traffic.txt: kernel, source hash, captured workload, dram bytes
    read+write per launch, algorithmic bytes of that launch), scaled to this
    launch by its algorithmic bytes.  None if no record matches the current
    kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = kernel_source_hash(kernel)
    for line in open(p):
        f = line.split()
        if len(f) == 5 and not line.startswith("#") and f[0] == kernel and f[1] == want:
            return float(f[3]) * alg_bytes / float(f[4])
    return None


def attention_roofline(work, attn_ms: float, peaks) -> dict:
    """Roofline of the dominant kernel, the sparse attention.  Its algorithmic
    bytes are the kept K/V rows gathered at zero reuse (2 x r x head_dim x 2 B
    per kept block and KV group) plus q, o, lse and sel.  Part of that gather is
    served from L2 (a group's K/V is about the size of L2), so the fraction of
    the HBM copy peak can pass 1; the DRAM bytes of the committed ncu record
    (scaled to this launch) give the fraction DRAM actually moved."""
    nbytes = work["attn"]["bytes"]
    achieved = nbytes / (attn_ms * 1e-3) / 1e9
    traffic = traffic_record("attn", nbytes)
    r = {"kernel": "sparse attention (attn stage)", "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peaks["source"],
         "bytes_per_launch": nbytes,
         "basis": "gathered K/V bytes at zero reuse, partly served from L2 (not all HBM traffic)",
         "tensor_frac": work["attn"]["flops"] / (attn_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}
    if traffic is not None:
        r["dram_gbs"] = traffic / (attn_ms * 1e-3) / 1e9
        r["dram_frac"] = r["dram_gbs"] / peaks["hbm_gbs"]
    return r


def step_tensor_roofline(work, step_ms: float, stage_ms, peaks) -> dict:
    """The whole step's algorithmic flops (indexer and attention contractions)
    over its device time, against the bf16 tensor peak: the literal figure for
    the prefill target.  Beside it: the index stage alone (the one dense
    contraction, k^ L2-resident) and the attainable step time, the sum over the
    stages of max(flops / tensor peak, algorithmic bytes / HBM peak), where the
    attention's bytes are its zero-reuse gather and the selection's are 0 (it
    can be fused with the scoring)."""
    tp, bw = peaks["bf16_tflops"] * 1e12, peaks["hbm_gbs"] * 1e9
    flops = work["flops"]
    achieved = flops / (step_ms * 1e-3) / 1e12
    idx_ms = stage_ms[1]
    att = [work["compress"]["bytes"] / bw,
           max(work["index"]["flops"] / tp, (work["index"]["khat_bytes"] + work["index"]["query_bytes"]) / bw),
           0.0,
           max(work["attn"]["flops"] / tp, work["attn"]["bytes"] / bw)]
    attainable_ms = sum(att) * 1e3
    return {"flops_per_step": flops, "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_tflops"], "peak_source": peaks["source"],
            "index_stage": {"ms": idx_ms, "flops": work["index"]["flops"],
                            "achieved": work["index"]["flops"] / (idx_ms * 1e-3) / 1e12,
                            "frac": work["index"]["flops"] / (idx_ms * 1e-3) / tp},
            "attainable": {"ms_per_step": attainable_ms, "stage_ms": [a * 1e3 for a in att],
                           "frac": attainable_ms / step_ms,
                           "basis": "per stage max(flops / bf16 peak, algorithmic bytes / HBM peak); "
                                    "attention bytes = zero-reuse gather; selection fused (0)"}}


def side_line(name: str, args, ws: int, rank: int, flush, peaks) -> dict:
    """One more workload's step beside the main line: device time, per-stage
    times, the step's roofline on its algorithmic bytes (no score round trip)
    and flops, the actual bytes the score-matrix path moves, and (rank 0, one
    GPU) the CPU oracle on a bounded sample."""
    wl2 = synth.make_workload(name)
    prep2 = Prepared(wl2)
    m2 = measure(prep2, args.steps, args.warmup, ws, flush, peaks)
    w2 = m2["work"]
    ms = m2["fused_ms"]
    d = {"workload": name, "ms_per_step": ms, "tokens_per_step": wl2.n_tokens,
         "tokens_per_s": job_throughput(wl2.n_tokens, ms, ws), "stages": m2["stages"], "gpu_launches": m2["launches"]}
    alg, act = w2["algorithmic_bytes"], w2["actual_bytes"]
    d["hbm_roofline"] = {"bytes_per_step": alg, "achieved_gbs": alg / (ms * 1e-3) / 1e9,
                         "frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
                         "peak_source": peaks["source"],
                         "basis": "algorithmic bytes: pooling, k^ stream, query rows, kept K/V (zero reuse), "
                                  "q/o/lse, sel; no score round trip",
                         "actual_bytes_per_step": act,
                         "actual_frac": act / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    if wl2.n_tokens <= 64:
        # the same step captured once in a CUDA graph and replayed (a decode loop's usual form)
        gr = graph_replay(prep2, args.steps, args.warmup, flush, ws)
        gr["hbm_frac"] = alg / (gr["ms_per_step"] * 1e-3) / 1e9 / peaks["hbm_gbs"]
        d["graph_replay"] = gr
    if wl2.prefix:
        import dataclasses
        alone = algorithmic_work(dataclasses.replace(wl2, prefix=[]))["index"]["khat_bytes"]
        d["shared_prefix"] = {"khat_bytes_per_step": w2["index"]["khat_bytes"],
                              "khat_bytes_if_unshared": alone,
                              "khat_cut": alone / max(1.0, w2["index"]["khat_bytes"]),
                              "prefix_blocks": wl2.prefix[0][1], "sequences": len(wl2.segments)}
    d["tensor_roofline"] = {"flops_per_step": w2["flops"], "achieved": w2["flops"] / (ms * 1e-3) / 1e12,
                            "frac": w2["flops"] / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                            "peak": peaks["bf16_tflops"]}
    if rank == 0 and ws == 1 and not args.no_cpu and args.side_cpu_seconds > 0 and name in ORACLE_SIDE:
        slots, budget = ORACLE_SIDE[name]
        v, threads, desc = oracle_sample(wl2, prep2.x, args.side_cpu_seconds * budget, max_slots=slots)
        d["cpu_oracle"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc}
    del prep2
    torch.cuda.empty_cache()
    return d


def graph_replay(prep: Prepared, steps: int, warmup: int, flush, ws: int) -> dict:
    """Device time of the workload's forward captured in a CUDA graph and
    replayed (L2 flushed before each replay), and whether a replay's output
    equals a direct call's."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        prep.forward()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        prep.forward()
    for _ in range(warmup):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    o = prep.o.clone()
    prep.forward()
    torch.cuda.synchronize()
    same = bool(torch.equal(o, prep.o))
    del graph
    ms = max_over_ranks(tot / steps, ws)
    return {"ms_per_step": ms, "tokens_per_s": job_throughput(prep.T, ms, ws), "output_matches_direct_call": same}


# side lines with an oracle timing: (sequences it times, 0 = all; time budget in
# units of --side-cpu-seconds).  Each 256K-context sequence's K/V is 1 GiB in the
# oracle's fp32; the 8K prefill's budget covers all of its queries on 16 cores.
ORACLE_SIDE = {"tiny_fp32": (0, 1.0), "prefill_8k": (0, 6.0), "decode_256k": (8, 1.0)}


def parse_overrides(text: str) -> dict:
    """'n_seqs=2,ctx=262144' -> {'n_seqs': 2, 'ctx': 262144} (integer or float values)."""
    out = {}
    for kv in [t for t in text.split(",") if t]:
        k, v = kv.split("=")
        out[k.strip()] = float(v) if "." in v else int(v)
    return out


def profile_stage(prep: Prepared, args, flush, peaks) -> int:
    """One stage's public entry point alone, --warmup + --steps times, L2 flushed
    before each; the stages before it run once, untimed, for its inputs."""
    i = ["compress", "index", "select", "attn"].index(args.profile_stage)
    for j in range(i):
        prep.stage(j)
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        prep.stage(i)
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(st)
        prep.stage(i)
        e1.record(st)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / args.steps
    w = prep.work()[args.profile_stage]
    out = {"profile_stage": args.profile_stage, "workload": args.workload, "overrides": args.wl, "ms": ms}
    if "bytes" in w:
        out["algorithmic_bytes"] = w["bytes"]
        out["gbs"] = w["bytes"] / (ms * 1e-3) / 1e9
        out["hbm_frac"] = out["gbs"] / peaks["hbm_gbs"]
    if "flops" in w:
        out["tflops"] = w["flops"] / (ms * 1e-3) / 1e12
        out["tensor_frac"] = out["tflops"] / peaks["bf16_tflops"]
    print(json.dumps(out), flush=True)
    return 0


def bench_config(name: str, wl: synth.Workload, ws: int) -> dict:
    """The workload description both arms print."""
    return {"workload": name, "batch": len(wl.segments), "seq_len": wl.segments[0].q_len,
            "budget_tokens": wl.shape.budget_tokens, "heads": wl.shape.n_heads, "kv_groups": wl.shape.n_groups,
            "head_dim": wl.shape.head_dim, "idx_heads": wl.shape.idx_heads, "idx_dim": wl.shape.idx_dim,
            "parallelism": f"replicas x{ws}",
            "l2": "flushed before every timed step (256 MiB write, then 256 MiB read)"}


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.make_workload(args.workload)
    x = synth.make_inputs(wl, device="cuda" if torch.cuda.is_available() else "cpu")
    # warm-up steps: a short sample each; timed steps: the time budget split over
    # the steps, each on evenly spaced queries at its own phase, so that together
    # they cover more distinct queries than the cpu_baseline leg's sample
    for i in range(args.warmup):
        oracle_sample(wl, x, target_s=0.5, phase=0.5)
    est = []
    desc = ""
    threads = 0
    per_step = max(1.0, args.ref_seconds / max(1, args.steps))
    for i in range(args.steps):
        v, threads, d = oracle_sample(wl, x, target_s=per_step, phase=(i + 0.5) / args.steps)
        est.append(wl.n_tokens / v)
        desc = d
    val = wl.n_tokens / statistics.mean(est)
    desc = f"{args.steps} timed steps of about {per_step:.1f} s each, each a different evenly spaced query " \
           f"sample; the last: {desc}"
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wl.n_tokens / val * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": bench_config(args.workload, wl, ws),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["qsa", "reference"], default="qsa")
    ap.add_argument("--workload", default="prefill_128k")
    ap.add_argument("--decode-workload", default="decode_1m,mixed_1m,decode_256k,prefill_8k,tiny_fp32,shared_prefix_1m",
                    help="comma-separated extra workloads reported beside the main line; 'none' to skip")
    ap.add_argument("--side-cpu-seconds", type=float, default=8.0,
                    help="oracle time budget of each side line's CPU timing (0: none)")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="oracle time budget of the reference arm's timed steps, all together")
    ap.add_argument("--bwd-workload", default="prefill_8k",
                    help="workload of the attention-backward measurement; 'none' to skip")
    ap.add_argument("--union-workload", default="prefill_128k_local",
                    help="attention on union tiles beside the per-query path ('none' to skip)")
    ap.add_argument("--union-n", type=int, default=0, help="query tokens of the union workload (0: its own)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-lowmem", action="store_true", help="skip the low-memory forward line")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--wl", default="",
                    help="size overrides of --workload's recipe, e.g. n_seqs=2,ctx=262144 (profiling cases)")
    ap.add_argument("--profile-stage", choices=["compress", "index", "select", "attn"], default=None,
                    help="run one stage's entry point --warmup + --steps times on --workload and print its "
                         "mean device time (the earlier stages run once, untimed); for ncu captures")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)

    ws, rank = dist_setup()
    peaks = load_peaks()
    flush = L2Flush()
    wl = synth.make_workload(args.workload, **parse_overrides(args.wl))
    prep = Prepared(wl)
    if args.profile_stage:
        return profile_stage(prep, args, flush, peaks)
    clocks = ClockSampler(torch.cuda.current_device())
    m = measure(prep, args.steps, args.warmup, ws, flush, peaks, clocks)
    tokens = wl.n_tokens
    value = job_throughput(tokens, m["fused_ms"], ws)

    work = m["work"]
    roofline = tensor_roofline = None
    if m["stage_ms"] is not None:    # (a shared-prefix workload has no per-stage times)
        roofline = attention_roofline(work, m["stage_ms"][3], peaks)
        tensor_roofline = step_tensor_roofline(work, m["fused_ms"], m["stage_ms"], peaks)

    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h, n_calls, same = e2e_prefill(prep, args.steps, args.warmup)
        e2e_ms = max_over_ranks(e2e_ms, ws)
        e2e = {"value": job_throughput(tokens, e2e_ms, ws), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "api": f"qsa_forward, {n_calls} chunked-prefill calls per step",
               "output_matches_single_call": same}

    lowmem = None
    if not args.no_lowmem:
        # the same step through qsa_forward_lowmem (no score matrix)
        qsa.select_fallbacks()
        barrier(ws)
        per_l, launches_l = timed(prep, args.steps, args.warmup, flush, staged=False, lowmem=True)
        barrier(ws)
        ms_l = max_over_ranks(sum(p[0] for p in per_l) / args.steps, ws)
        lowmem = {"ms_per_step": ms_l, "tokens_per_s": job_throughput(tokens, ms_l, ws),
                  "workspace_bytes": prep.workspace_bytes(True), "workspace_bytes_default": prep.workspace_bytes(False),
                  "fallback_rows": qsa.select_fallbacks(), "gpu_launches": launches_l}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        v, threads, desc = oracle_sample(wl, prep.x, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc}
    del prep
    torch.cuda.empty_cache()

    extra = {}
    for name in [n for n in args.decode_workload.split(",") if n and n != "none"]:
        extra[name] = side_line(name, args, ws, rank, flush, peaks)

    if args.union_workload != "none":
        extra["attn_union"] = measure_union(args.union_workload, args.steps, args.warmup, ws, flush, peaks,
                                            args.union_n or None)

    if args.bwd_workload != "none":
        extra["attn_backward"] = measure_backward(args.bwd_workload, args.steps, args.warmup, ws, flush, peaks)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": m["fused_ms"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": wl.shape.dtype, "data": "synthetic",
                "config": bench_config(args.workload, wl, ws),
                "roofline": roofline, "tensor_roofline": tensor_roofline, "stages": m["stages"],
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": m["launches"], "clocks": m["clocks"], "lowmem_forward": lowmem}
        line.update(extra)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
