"""Seeded synthetic inputs for the QSA forward pass.

This module only draws random tensors and plants needles.  It holds none of
the method's arithmetic (no pooling, rotary encoding, scoring, selection or
attention), so the oracle side and the CUDA side can both consume what it
produces without sharing any of the method's code.

Workloads mirror the shapes the pages describe for Qwen3.8-Flash-Next's QSA
layers (Miles docs "Qwen3.8-Flash-Next", section 1: 24 heads, 2 query groups,
kv-channels 256, rotary 0.25 at base 1e7; design report, QSA item: r=4, a
4-head indexer, budget 2048 tokens):

  tiny_fp32     1 sequence, 256 tokens, indexer dim 64, budget 64 tokens, fp32
  prefill_8k    2 sequences x 8192 tokens, bf16, 4 needles per 1024 queries
  prefill_128k  1 sequence x 131072 tokens, bf16, a needle every 8192 positions
  decode_256k   32 sequences x 1 decode query against a 262144-token cache
  mixed_1m      8 decode queries at 1048576-token context plus one 4096-query
                prefill chunk at [942080, 946176) of a 90%-cached sequence
  decode_1m     the decode part of mixed_1m alone: 8 sequences x 1 decode
                query against a 1048576-token cache
  mixed_1m_tail mixed_1m with the prefill chunk at the end of its sequence,
                [1044480, 1048576)
  spec_decode_1m  8 sequences x 4 consecutive query tokens (a speculative
                decode step) at the end of a 1048576-token cache; the 4
                queries of a sequence share one stream of its k^
  chunk_128k    one 4096-query prefill chunk at [126976, 131072) of a
                131072-token sequence whose prefix is cached (a ~1 GB case
                whose K/V still exceeds L2; used for kernel profiles)
  shared_prefix_1m  8 sequences x 1 decode query at 1048576-token context
                that share a cached prefix of 943716 tokens (90 %): the
                prefix lives once in its own cache slot, each sequence's
                suffix in its slot; 4 needles per sequence in the prefix and
                4 in its suffix
  prefill_128k_local  prefill_128k with indexer queries that drift slowly
                along the sequence (below), so neighbouring tokens keep
                mostly the same blocks

Distributions: q, k, v, indexer q and indexer k ~ N(0, 1) drawn in fp32 and
rounded once to the I/O dtype; head weights w ~ U(0, 1) in fp32.

Locality (`drift` rho > 0, an input made to have it, not a property the pages
state): along each segment's tokens the indexer queries follow a stationary
AR(1) process, q_idx[t] = rho q_idx[t-1] + sqrt(1 - rho^2) e[t] with e ~ N(0,1)
(so every q_idx[t] is still N(0,1)), and the head weights a convex one,
w[t] = rho w[t-1] + (1 - rho) u[t] with u ~ U(0,1).  prefill_128k_local uses
rho = 0.99.

Needles ("key = scaled copy of query"): for a target query t* of cache slot s
and a block b* < floor(t*/r), the r indexer-key rows of b* are set to
alpha * u, u = sum_h w[t*,h] * q_idx[t*,h] with the rotary dims zeroed (so the
block's position encoding leaves it unchanged), and the main K rows of b* in
every group are set to beta * q[t*, head 0].  alpha = beta = 1.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import torch


@dataclass(frozen=True)
class Shape:
    n_heads: int = 24
    n_groups: int = 2
    head_dim: int = 256
    idx_heads: int = 4
    idx_dim: int = 128
    r: int = 4
    budget_tokens: int = 2048
    rope_fraction: float = 0.25
    rope_base: float = 1e7
    dtype: str = "bf16"           # "bf16" or "f32": I/O dtype of q, k, v, indexer q/k, k^, o

    @property
    def rope_dims(self) -> int:
        d = int(self.idx_dim * self.rope_fraction)
        return d - (d % 2)

    @property
    def budget_blocks(self) -> int:
        return self.budget_tokens // self.r

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


@dataclass(frozen=True)
class Segment:
    """A run of consecutive query tokens of one cached sequence."""
    slot: int        # cache slot of the sequence
    pos0: int        # absolute position of the first query token
    q_len: int       # number of query tokens (positions pos0 .. pos0+q_len-1)


@dataclass
class Workload:
    name: str
    shape: Shape
    segments: List[Segment]
    n_slots: int
    n_cap: int                         # cache capacity per slot (tokens)
    fill: List[int]                    # tokens present in each slot's cache
    cached_blocks: List[int]           # k^ blocks already pooled before the step
    needles: List[Tuple[int, int, int]] = field(default_factory=list)  # (slot, t*, b*)
    seed: int = 0
    drift: float = 0.0                 # AR(1) coefficient of the indexer queries along a segment
    # per segment (prefix slot, prefix blocks), or empty: blocks below the
    # prefix's end live in the prefix slot; the segment's slot holds the rest
    prefix: List[Tuple[int, int]] = field(default_factory=list)
    start: List[int] = field(default_factory=list)   # first present row of each slot (default 0)

    @property
    def n_tokens(self) -> int:
        return sum(s.q_len for s in self.segments)

    def token_offsets(self) -> List[int]:
        out, acc = [], 0
        for s in self.segments:
            out.append(acc)
            acc += s.q_len
        return out

    def token_positions(self) -> torch.Tensor:
        return torch.cat([torch.arange(s.pos0, s.pos0 + s.q_len, dtype=torch.int64)
                          for s in self.segments])

    def token_slots(self) -> torch.Tensor:
        return torch.cat([torch.full((s.q_len,), s.slot, dtype=torch.int64) for s in self.segments])


def _needles_per_window(rng: torch.Generator, slot: int, lo: int, hi: int, per_1k: int,
                        r: int) -> List[Tuple[int, int, int]]:
    out = []
    for w0 in range(lo, hi, 1024):
        w1 = min(hi, w0 + 1024)
        for _ in range(per_1k):
            t = int(torch.randint(max(w0, r), w1, (1,), generator=rng)) if w1 > max(w0, r) else None
            if t is None:
                continue
            b = int(torch.randint(0, t // r, (1,), generator=rng))
            out.append((slot, t, b))
    return out


def _distinct_blocks(rng: torch.Generator, nblk: int, k: int) -> List[int]:
    picks: List[int] = []
    while len(picks) < k:
        b = int(torch.randint(0, nblk, (1,), generator=rng))
        if b not in picks:
            picks.append(b)
    return picks


def make_workload(name: str, seed: Optional[int] = None, **over) -> Workload:
    """Return one of the named workloads (see module docstring).

    Keyword overrides allow reduced sizes of the same recipe for parity tests:
    n (prefill length), n_seqs, ctx (decode context), chunk (prefill chunk
    length), chunk_pos0, n_decode; `shape` (Shape fields) for prefill_8k and
    the decode workloads.
    """
    rng = torch.Generator().manual_seed(1000 + (seed if seed is not None else 0))
    if name == "tiny_fp32":
        sh = Shape(idx_dim=64, budget_tokens=64, dtype="f32")
        n = over.get("n", 256)
        wl = Workload(name, sh, [Segment(0, 0, n)], 1, _round_cap(n, sh.r), [n], [0], [], seed or 0)
        return wl
    if name == "prefill_8k":
        sh = Shape(**over.get("shape", {}))
        n = over.get("n", 8192)
        n_seqs = over.get("n_seqs", 2)
        segs = [Segment(s, 0, n) for s in range(n_seqs)]
        needles = []
        for s in range(n_seqs):
            needles += _needles_per_window(rng, s, 0, n, 4, sh.r)
        return Workload(name, sh, segs, n_seqs, _round_cap(n, sh.r), [n] * n_seqs, [0] * n_seqs, needles,
                        seed if seed is not None else 1, over.get("drift", 0.0))
    if name in ("prefill_128k", "prefill_128k_local"):
        sh = Shape()
        n = over.get("n", 131072)
        every = over.get("every", 8192)
        needles = []
        for i in range(n // every):
            t = every * i + every - 1
            b = int(torch.randint(0, t // sh.r, (1,), generator=rng))
            needles.append((0, t, b))
        drift = over.get("drift", 0.99 if name == "prefill_128k_local" else 0.0)
        return Workload(name, sh, [Segment(0, 0, n)], 1, _round_cap(n, sh.r), [n], [0], needles,
                        seed if seed is not None else 2, drift)
    if name in ("decode_256k", "decode_1m"):
        sh = Shape(**over.get("shape", {}))
        big = name == "decode_1m"
        ctx = over.get("ctx", (1 << 20) if big else 262144)
        n_seqs = over.get("n_seqs", 8 if big else 32)
        segs = [Segment(s, ctx - 1, 1) for s in range(n_seqs)]
        needles = []
        for s in range(n_seqs):
            t = ctx - 1
            for b in _distinct_blocks(rng, t // sh.r, 8):
                needles.append((s, t, b))
        # the decode token completes block (ctx-1)//r; earlier blocks are cached
        cached = [(ctx - 1) // sh.r] * n_seqs
        return Workload(name, sh, segs, n_seqs, _round_cap(ctx, sh.r), [ctx] * n_seqs, cached, needles,
                        seed if seed is not None else (6 if big else 3))
    if name == "shared_prefix_1m":
        sh = Shape(**over.get("shape", {}))
        ctx = over.get("ctx", 1 << 20)
        n_seqs = over.get("n_seqs", 8)
        q_len = over.get("q_len", 1)
        p_tok = over.get("prefix", int(0.9 * ctx) // sh.r * sh.r)
        P = p_tok // sh.r
        pslot = n_seqs
        segs = [Segment(s, ctx - q_len, q_len) for s in range(n_seqs)]
        needles = []
        for s in range(n_seqs):
            t = ctx - 1
            needles += [(s, t, b) for b in _distinct_blocks(rng, P, 4)]
            needles += [(s, t, P + b) for b in _distinct_blocks(rng, (ctx - 1) // sh.r - P - (q_len - 1), 4)]
        cached = [(ctx - q_len) // sh.r] * n_seqs + [P]
        return Workload(name, sh, segs, n_seqs + 1, _round_cap(ctx, sh.r), [ctx] * n_seqs + [p_tok], cached,
                        needles, seed if seed is not None else 9, prefix=[(pslot, P)] * n_seqs,
                        start=[p_tok] * n_seqs + [0])
    if name == "spec_decode_1m":
        sh = Shape(**over.get("shape", {}))
        ctx = over.get("ctx", 1 << 20)
        n_seqs = over.get("n_seqs", 8)
        q_len = over.get("q_len", 4)
        segs = [Segment(s, ctx - q_len, q_len) for s in range(n_seqs)]
        needles = []
        for s in range(n_seqs):
            for b in _distinct_blocks(rng, (ctx - 1) // sh.r, 8):
                needles.append((s, ctx - 1, b))
        cached = [(ctx - q_len) // sh.r] * n_seqs
        return Workload(name, sh, segs, n_seqs, _round_cap(ctx, sh.r), [ctx] * n_seqs, cached, needles,
                        seed if seed is not None else 7)
    if name in ("mixed_1m", "mixed_1m_tail"):
        sh = Shape()
        ctx = over.get("ctx", 1 << 20)
        n_dec = over.get("n_decode", 8)
        chunk = over.get("chunk", 4096)
        pos0 = over.get("chunk_pos0", ctx - chunk if name == "mixed_1m_tail" else 942080)
        segs = [Segment(s, ctx - 1, 1) for s in range(n_dec)]
        segs.append(Segment(n_dec, pos0, chunk))
        needles = []
        for s in range(n_dec):
            for b in _distinct_blocks(rng, (ctx - 1) // sh.r, 8):
                needles.append((s, ctx - 1, b))
        needles += _needles_per_window(rng, n_dec, pos0, pos0 + chunk, 4, sh.r)
        fill = [ctx] * n_dec + [pos0 + chunk]
        cached = [(ctx - 1) // sh.r] * n_dec + [pos0 // sh.r]
        return Workload(name, sh, segs, n_dec + 1, _round_cap(max(ctx, pos0 + chunk), sh.r), fill, cached, needles,
                        seed if seed is not None else 4)
    if name == "chunk_128k":
        sh = Shape()
        n = over.get("n", 131072)
        chunk = over.get("chunk", 4096)
        pos0 = n - chunk
        needles = _needles_per_window(rng, 0, pos0, n, 4, sh.r)
        return Workload(name, sh, [Segment(0, pos0, chunk)], 1, _round_cap(n, sh.r), [n], [pos0 // sh.r],
                        needles, seed if seed is not None else 5)
    raise KeyError(name)


def _round_cap(n: int, r: int) -> int:
    return (n + r - 1) // r * r


def _randn(shape, gen, device, dtype, chunk_elems=1 << 28):
    """N(0,1) drawn in fp32 and rounded once to dtype, generated in pieces."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    for i in range(0, flat.numel(), chunk_elems):
        n = min(chunk_elems, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def _ar1_(x: torch.Tensor, rho: float, innov: float, block: int = 256) -> None:
    """In place along dim 0: y[0] = x[0], y[t] = rho y[t-1] + innov x[t]
    (fp32 carry, one rounding to x's dtype), evaluated block by block as
    y[s:s+L] = A (innov x[s:s+L]) + rho^(1..L) y[s-1] with A[i,j] = rho^(i-j)."""
    n = x.shape[0]
    if n < 2 or rho == 0.0:
        return
    flat = x.view(n, -1)
    i = torch.arange(block, dtype=torch.float64, device=x.device)
    d = i[:, None] - i[None, :]
    A = torch.where(d >= 0, rho ** d.clamp(min=0), torch.zeros_like(d)).float()
    pw = (rho ** (i + 1)).float()
    prev = None
    for s in range(0, n, block):
        e = flat[s:s + block].float()
        L = e.shape[0]
        inn = innov * e
        if prev is None:
            inn[0] = e[0]
            y = A[:L, :L] @ inn
        else:
            y = A[:L, :L] @ inn + pw[:L, None] * prev
        flat[s:s + L] = y.to(x.dtype)
        prev = y[-1]


def make_inputs(wl: Workload, device="cpu") -> Dict[str, torch.Tensor]:
    """Draw every input tensor of the workload on `device` (seeded).

    Returns token-major query tensors (q [T,H,D], q_idx [T,Hi,dI], w [T,Hi])
    and slot-major caches (k_idx [S,N,dI], k and v [S,G,N,D]).  Cache rows
    beyond a slot's fill are zero.
    """
    sh = wl.shape
    dt = sh.torch_dtype
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(wl.seed)
    T = wl.n_tokens
    q = _randn((T, sh.n_heads, sh.head_dim), gen, dev, dt)
    q_idx = _randn((T, sh.idx_heads, sh.idx_dim), gen, dev, dt)
    w = torch.rand((T, sh.idx_heads), generator=gen, device=dev, dtype=torch.float32)
    k_idx = torch.zeros((wl.n_slots, wl.n_cap, sh.idx_dim), dtype=dt, device=dev)
    k = torch.zeros((wl.n_slots, sh.n_groups, wl.n_cap, sh.head_dim), dtype=dt, device=dev)
    v = torch.zeros_like(k)
    for s in range(wl.n_slots):
        f = wl.fill[s]
        f0 = wl.start[s] if wl.start else 0
        k_idx[s, f0:f] = _randn((f - f0, sh.idx_dim), gen, dev, dt)
        for g in range(sh.n_groups):
            k[s, g, f0:f] = _randn((f - f0, sh.head_dim), gen, dev, dt)
            v[s, g, f0:f] = _randn((f - f0, sh.head_dim), gen, dev, dt)
    offs = wl.token_offsets()
    if wl.drift > 0:
        rho = wl.drift
        for o0, seg in zip(offs, wl.segments):
            _ar1_(q_idx[o0:o0 + seg.q_len], rho, (1.0 - rho * rho) ** 0.5)
            _ar1_(w[o0:o0 + seg.q_len], rho, 1.0 - rho)
    # needles
    n_rot = sh.rope_dims
    for (slot, t, b) in wl.needles:
        tok = None
        for si, seg in enumerate(wl.segments):
            if seg.slot == slot and seg.pos0 <= t < seg.pos0 + seg.q_len:
                tok = offs[si] + (t - seg.pos0)
        if tok is None:
            continue
        u = (w[tok].unsqueeze(1) * q_idx[tok].float()).sum(0)
        u[:n_rot] = 0
        dst = slot
        if wl.prefix:                          # a needle in a shared prefix lives in the prefix's slot
            ps, pb = wl.prefix[[sg.slot for sg in wl.segments].index(slot)]
            if b < pb:
                dst = ps
        k_idx[dst, b * sh.r:(b + 1) * sh.r] = u.to(dt)
        for g in range(sh.n_groups):
            k[dst, g, b * sh.r:(b + 1) * sh.r] = q[tok, 0]
    return {"q": q, "q_idx": q_idx, "w": w, "k_idx": k_idx, "k": k, "v": v}


def describe(wl: Workload) -> dict:
    d = dataclasses.asdict(wl)
    d["n_tokens"] = wl.n_tokens
    d.pop("needles")
    d["n_needles"] = len(wl.needles)
    return d


def sequence_cache(wl: Workload, x: Dict[str, torch.Tensor], slot: int, fill: int):
    """A sequence's whole cache rows [0, fill) (k_idx [fill, dI], k and v
    [G, fill, D]): with a shared prefix, its first rows come from the prefix's
    slot and the rest from the sequence's slot."""
    k_idx, k, v = x["k_idx"][slot, :fill], x["k"][slot, :, :fill], x["v"][slot, :, :fill]
    if wl.prefix:
        ps, pb = wl.prefix[[sg.slot for sg in wl.segments].index(slot)]
        n = min(fill, pb * wl.shape.r)
        if n > 0:
            k_idx = torch.cat([x["k_idx"][ps, :n], k_idx[n:]])
            k = torch.cat([x["k"][ps, :, :n], k[:, n:]], dim=1)
            v = torch.cat([x["v"][ps, :, :n], v[:, n:]], dim=1)
    return k_idx, k, v
