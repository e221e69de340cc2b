"""The C ABI library: loads without a GPU, exports every entry point that
include/qsa.h declares, and rejects bad arguments on the host before any
CUDA call (CPU only; no compute is launched)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_22_b200 as qsa
from block_sparse_attention_22_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(qsa_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert {"qsa_compress_keys", "qsa_index_scores", "qsa_select_topk", "qsa_sparse_attn_fwd",
            "qsa_forward", "qsa_workspace_size"} <= set(names)
    lib = ctypes.CDLL(qsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {qsa.LIB_PATH}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {n for n in exported if n.startswith("qsa_")}
    assert ours == set(declared_functions())


def _setup(shape=None):
    sh = shape or synth.Shape()
    cfg = qsa.make_config(sh)
    segs = qsa.make_segments([(0, 16, 100, 0)])
    cache = qsa.qsa_cache_t(16, 16, 16, 16, 1, 1024)    # fake aligned addresses: never dereferenced
    return sh, cfg, segs, cache


def _call_forward(cfg, cache, segs, T=16, ws_bytes=1 << 40, **kw):
    L = qsa.get_lib()
    args = dict(q=16, q_idx=16, w=16, o=16, lse=None, sel=None, nsel=None, ws=16)
    args.update(kw)
    return L.qsa_forward(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], T, args["q"], args["q_idx"],
                         args["w"], args["o"], args["lse"], args["sel"], args["nsel"], args["ws"], ws_bytes, None)


@pytest.mark.parametrize("field,value,status", [
    ("r", 8, qsa.QSA_ERR_UNSUPPORTED),
    ("r", 0, qsa.QSA_ERR_INVALID_ARG),
    ("budget_tokens", 2047, qsa.QSA_ERR_INVALID_ARG),
    ("budget_tokens", 8192, qsa.QSA_ERR_UNSUPPORTED),
    ("head_dim", 128, qsa.QSA_ERR_UNSUPPORTED),
    ("n_kv_groups", 5, qsa.QSA_ERR_INVALID_ARG),
    ("n_kv_groups", 1, qsa.QSA_ERR_UNSUPPORTED),
    ("idx_heads", 8, qsa.QSA_ERR_UNSUPPORTED),
    ("idx_dim", 96, qsa.QSA_ERR_UNSUPPORTED),
    ("rope_fraction", 1.5, qsa.QSA_ERR_INVALID_ARG),
    ("rope_base", -1.0, qsa.QSA_ERR_INVALID_ARG),
    ("dtype", 7, qsa.QSA_ERR_INVALID_ARG),
])
def test_bad_config_is_rejected_on_host(field, value, status):
    sh, cfg, segs, cache = _setup()
    setattr(cfg, field, value)
    assert _call_forward(cfg, cache, segs) == status


def test_bad_segments_pointers_and_workspace_are_rejected_on_host():
    sh, cfg, segs, cache = _setup()
    for bad in [(0, 16, 1020, 0), (8, 16, 0, 0), (0, -1, 0, 0), (0, 4, 0, 3), (-1, 4, 0, 0)]:
        assert _call_forward(cfg, cache, qsa.make_segments([bad])) == qsa.QSA_ERR_INVALID_ARG, bad
    assert _call_forward(cfg, cache, segs, q=None) == qsa.QSA_ERR_INVALID_ARG
    assert _call_forward(cfg, cache, segs, q=18) == qsa.QSA_ERR_INVALID_ARG      # misaligned
    assert _call_forward(cfg, cache, segs, sel=16) == qsa.QSA_ERR_INVALID_ARG   # sel without nsel
    assert _call_forward(cfg, cache, segs, ws_bytes=10) == qsa.QSA_ERR_WORKSPACE
    assert _call_forward(cfg, cache, segs, ws=None) == qsa.QSA_ERR_WORKSPACE
    bad_cache = qsa.qsa_cache_t(16, 16, 16, 16, 1, 1023)
    assert _call_forward(cfg, bad_cache, segs) == qsa.QSA_ERR_INVALID_ARG


def _call_prefixed(cfg, cache, segs, prefixes, T, ws_bytes=1 << 40, **kw):
    L = qsa.get_lib()
    args = dict(q=16, q_idx=16, w=16, o=16, ws=16)
    args.update(kw)
    return L.qsa_forward_prefixed(ctypes.byref(cfg), ctypes.byref(cache), segs[0], prefixes, segs[1], T, args["q"],
                                  args["q_idx"], args["w"], args["o"], None, None, None, args["ws"], ws_bytes, None)


def test_prefix_arguments_are_checked_on_host():
    """qsa_forward_prefixed: a prefix's slot, length (at most the query's
    position, in blocks) and the decode-only rule are checked before any
    CUDA call; a valid table passes every check and stops at the workspace."""
    sh = synth.Shape()
    cfg = qsa.make_config(sh)
    cache = qsa.qsa_cache_t(16, 16, 16, 16, 3, 4096)       # 3 slots of 4096 tokens (fake addresses)
    segs = qsa.make_segments([(0, 1, 2000, 0), (1, 1, 3000, 1)])
    ok = qsa.make_prefixes([(2, 400), (2, 400)])
    assert _call_prefixed(cfg, cache, segs, ok, 2, ws_bytes=10) == qsa.QSA_ERR_WORKSPACE
    for bad in ([(3, 400), (2, 400)],      # slot past the cache
                [(-1, 400), (2, 400)],     # negative slot
                [(2, -1), (2, 400)],       # negative length
                [(2, 501), (2, 400)]):     # 501 blocks = 2004 tokens > position 2000
        assert _call_prefixed(cfg, cache, segs, qsa.make_prefixes(bad), 2) == qsa.QSA_ERR_INVALID_ARG, bad
    assert _call_prefixed(cfg, cache, segs, None, 2) == qsa.QSA_ERR_INVALID_ARG       # no prefix table
    no_share = qsa.make_prefixes([(0, 0), (0, 0)])                                  # nothing shared: plain forward
    assert _call_prefixed(cfg, cache, segs, no_share, 2, ws_bytes=10) == qsa.QSA_ERR_WORKSPACE
    long_seg = qsa.make_segments([(0, 16, 2000, 0), (16, 1, 3000, 1)])
    assert _call_prefixed(cfg, cache, long_seg, ok, 17) == qsa.QSA_ERR_UNSUPPORTED     # 16 queries on a prefix
    f32 = qsa.make_config(synth.Shape(dtype="f32"))
    assert _call_prefixed(f32, cache, segs, ok, 2) == qsa.QSA_ERR_UNSUPPORTED


def test_noalloc_selection_checks_run_before_the_scratch_lookup():
    """qsa_select_topk_noalloc rejects bad arguments and a batch whose
    selection needs more than its fixed scratch before it looks the scratch
    up or launches anything (fake pointers, never dereferenced)."""
    cfg = qsa.make_config(synth.Shape())
    L = qsa.get_lib()

    def call(segs, T, scores=16, ld=524288, sel=16, nsel=16):
        return L.qsa_select_topk_noalloc(ctypes.byref(cfg), segs[0], segs[1], T, scores, ld, sel, nsel, None)

    big = qsa.make_segments([(i, 1, (1 << 21) - 1, 0) for i in range(500)])   # 48 KiB of scratch per row
    assert qsa.workspace_size(cfg, big, 500, qsa.QSA_OP_SELECT) > (16 << 20)
    assert call(big, 500) == qsa.QSA_ERR_WORKSPACE
    small = qsa.make_segments([(0, 1, 40003, 0)])                              # 10000 candidate blocks
    assert call(small, 1, ld=9999) == qsa.QSA_ERR_INVALID_ARG                 # row pitch below the row
    assert call(small, 1, sel=18) == qsa.QSA_ERR_INVALID_ARG                  # misaligned sel
    assert call(small, 1, scores=None) == qsa.QSA_ERR_INVALID_ARG
    assert call(qsa.make_segments([]), 0) == qsa.QSA_OK                        # empty batch: nothing to do


def test_backward_arguments_are_checked_on_host():
    """qsa_sparse_attn_bwd rejects missing or misaligned buffers and bad
    segments before any CUDA call; an empty batch is a no-op."""
    sh, cfg, segs, cache = _setup()
    L = qsa.get_lib()

    def call(segs, T=16, **kw):
        a = dict(q=16, o=16, lse=16, dout=16, sel=16, nsel=16, dq=16, dk=16, dv=16)
        a.update(kw)
        return L.qsa_sparse_attn_bwd(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], T, a["q"], a["o"],
                                     a["lse"], a["dout"], a["sel"], a["nsel"], a["dq"], a["dk"], a["dv"], None)

    for name in ("q", "o", "lse", "dout", "sel", "nsel", "dq", "dk", "dv"):
        assert call(segs, **{name: None}) == qsa.QSA_ERR_INVALID_ARG, name
    for name in ("q", "o", "dout", "dq", "dk", "dv"):
        assert call(segs, **{name: 24}) == qsa.QSA_ERR_INVALID_ARG, name          # not 16-byte aligned
    assert call(qsa.make_segments([(0, 16, 1020, 0)])) == qsa.QSA_ERR_INVALID_ARG   # past the cache
    assert call(qsa.make_segments([]), T=0) == qsa.QSA_OK


def test_stage_entry_points_check_arguments_on_host():
    """The four stage entry points and the low-memory forward reject bad
    ranges, missing or misaligned buffers and short score rows before any
    CUDA call (fake pointers, never dereferenced)."""
    sh, cfg, segs, cache = _setup()           # 16 queries at positions 100..115: up to 28 candidate blocks
    L = qsa.get_lib()

    def compress(slots, b0, b1, n=None):
        n = len(slots) if n is None else n
        return L.qsa_compress_keys(ctypes.byref(cfg), ctypes.byref(cache), (ctypes.c_int32 * 2)(*slots),
                                   (ctypes.c_int64 * 2)(*b0), (ctypes.c_int64 * 2)(*b1), n, None)

    assert compress([0], [0], [0], n=-1) == qsa.QSA_ERR_INVALID_ARG
    assert compress([1], [0], [4]) == qsa.QSA_ERR_INVALID_ARG        # slot past the cache
    assert compress([0], [5], [4]) == qsa.QSA_ERR_INVALID_ARG        # end before begin
    assert compress([0], [0], [257]) == qsa.QSA_ERR_INVALID_ARG      # past 1024 / r blocks
    assert compress([], [], []) == qsa.QSA_OK
    assert L.qsa_compress_keys(ctypes.byref(cfg), ctypes.byref(cache), None, None, None, 1, None) == \
        qsa.QSA_ERR_INVALID_ARG

    def index(q_idx=16, w=16, scores=16, ld=28):
        return L.qsa_index_scores(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], 16, q_idx, w, scores,
                                  ld, None)

    assert index(q_idx=None) == qsa.QSA_ERR_INVALID_ARG
    assert index(scores=20) == qsa.QSA_ERR_INVALID_ARG               # not 16-byte aligned
    assert index(ld=27) == qsa.QSA_ERR_INVALID_ARG                   # row pitch below 28 blocks

    def select(scores=16, ld=28, sel=16, nsel=16):
        return L.qsa_select_topk(ctypes.byref(cfg), segs[0], segs[1], 16, scores, ld, sel, nsel, 16, 1 << 40, None)

    assert select(scores=None) == qsa.QSA_ERR_INVALID_ARG
    assert select(sel=20) == qsa.QSA_ERR_INVALID_ARG
    assert select(nsel=None) == qsa.QSA_ERR_INVALID_ARG
    assert select(ld=27) == qsa.QSA_ERR_INVALID_ARG

    def attend(q=16, sel=16, nsel=16, o=16):
        return L.qsa_sparse_attn_fwd(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], 16, q, sel, nsel, o,
                                     None, 16, 1 << 40, None)

    assert attend(q=24) == qsa.QSA_ERR_INVALID_ARG
    assert attend(sel=None) == qsa.QSA_ERR_INVALID_ARG
    assert attend(o=None) == qsa.QSA_ERR_INVALID_ARG

    def lowmem(**kw):
        a = dict(q=16, q_idx=16, w=16, o=16)
        a.update(kw)
        return L.qsa_forward_lowmem(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], 16, a["q"], a["q_idx"],
                                    a["w"], a["o"], None, None, None, 16, 10, None)

    assert lowmem(q_idx=None) == qsa.QSA_ERR_INVALID_ARG
    assert lowmem(w=20) == qsa.QSA_ERR_INVALID_ARG
    assert lowmem() == qsa.QSA_ERR_WORKSPACE                          # valid arguments, 10-byte workspace


def test_empty_batches_are_noops_without_touching_the_device():
    sh, cfg, segs, cache = _setup()
    empty = qsa.make_segments([(0, 0, 100, 0)])
    assert _call_forward(cfg, cache, empty, T=0, ws=None, ws_bytes=0) == qsa.QSA_OK
    none = qsa.make_segments([])
    assert _call_forward(cfg, cache, none, T=0, ws=None, ws_bytes=0) == qsa.QSA_OK


def test_workspace_sizes_are_host_only_and_grow_with_the_batch():
    sh = synth.Shape()
    cfg = qsa.make_config(sh)
    small = qsa.make_segments([(0, 1024, 0, 0)])
    big = qsa.make_segments([(0, 131072, 0, 0)])
    a = qsa.workspace_size(cfg, small, 1024, qsa.QSA_OP_FORWARD)
    b = qsa.workspace_size(cfg, big, 131072, qsa.QSA_OP_FORWARD)
    assert 0 < a < b
    assert b >= 131072 * 32767 * 4           # the score rows
    # the low-memory forward keeps sample scores (every 16th of 32767 blocks)
    # and 4096-entry candidate lists per query instead of the score rows
    lo = qsa.workspace_size(cfg, big, 131072, qsa.QSA_OP_FORWARD_LOWMEM)
    assert 131072 * (2048 * 4 + 4096 * 8) <= lo < 131072 * 32767 * 4 // 3
    # fp32 and decode-like segments keep the score rows in both
    sh32 = synth.Shape(dtype="f32")
    b32 = qsa.workspace_size(qsa.make_config(sh32), big, 131072, qsa.QSA_OP_FORWARD_LOWMEM)
    assert b32 >= 131072 * 32767 * 4
    # decode-like rows keep their score rows in both forwards
    dec_fwd = qsa.make_segments([(i, 1, (1 << 20) - 1, i) for i in range(8)])
    for op in (qsa.QSA_OP_FORWARD, qsa.QSA_OP_FORWARD_LOWMEM):
        assert qsa.workspace_size(cfg, dec_fwd, 8, op) >= 8 * 262143 * 4
    assert qsa.workspace_size(cfg, small, 1024, qsa.QSA_OP_COMPRESS) == 0
    dec = qsa.make_segments([(i, 1, (1 << 20) - 1, i) for i in range(8)])
    assert qsa.workspace_size(cfg, dec, 8, qsa.QSA_OP_SELECT) > 0     # few long rows: row histograms
    assert qsa.workspace_size(cfg, dec, 8, qsa.QSA_OP_ATTN) > 0       # few units: split-K
    dec2 = qsa.make_segments([(i, 1, (1 << 21) - 1, i) for i in range(8)])
    short = qsa.make_segments([(i, 1, 100000, i) for i in range(8)])
    assert qsa.workspace_size(cfg, short, 8, qsa.QSA_OP_SELECT) == 0  # few short rows: one wide CTA each
    bad = qsa.make_segments([(0, 10, 0, 0)])
    assert qsa.workspace_size(cfg, bad, 5, qsa.QSA_OP_FORWARD) == 2 ** 64 - 1


def test_status_strings_and_version():
    assert qsa.status_string(qsa.QSA_OK) == "ok"
    assert "workspace" in qsa.status_string(qsa.QSA_ERR_WORKSPACE)
    assert qsa.version() >= 100


def _call_union(cfg, cache, segs, T=16, ws_bytes=1 << 40, **kw):
    L = qsa.get_lib()
    args = dict(q=16, o=16, lse=None, sel=16, nsel=16, ws=16)
    args.update(kw)
    return L.qsa_sparse_attn_fwd_union(ctypes.byref(cfg), ctypes.byref(cache), segs[0], segs[1], T, args["q"],
                                       args["sel"], args["nsel"], args["o"], args["lse"], args["ws"], ws_bytes,
                                       None)


def test_union_attention_host_checks_and_workspace():
    """The union-tile attention: tiles of min(32, 128 / heads per group) query
    tokens per segment, one length word plus a block and a mask word per
    union entry (tile size x budget blocks) per tile; bf16 only."""
    sh, cfg, segs, cache = _setup()
    big = qsa.make_segments([(0, 131072, 0, 0)])
    tiles = -(-131072 // 10)                     # 12 heads per group -> 10 queries per tile
    ws = qsa.workspace_size(cfg, big, 131072, qsa.QSA_OP_ATTN_UNION)
    assert tiles * (4 + 2 * 10 * 512 * 4) <= ws < tiles * (4 + 2 * 10 * 512 * 4) + 1024
    mha = qsa.make_config(synth.Shape(n_heads=16, n_groups=16))
    assert qsa.workspace_size(mha, big, 131072, qsa.QSA_OP_ATTN_UNION) >= (131072 // 32) * 2 * 32 * 512 * 4
    ragged = qsa.make_segments([(0, 11, 0, 0), (11, 1, 50, 1)])
    assert qsa.workspace_size(cfg, ragged, 12, qsa.QSA_OP_ATTN_UNION) >= 3 * (4 + 2 * 10 * 512 * 4)
    assert _call_union(cfg, cache, segs, ws_bytes=10) == qsa.QSA_ERR_WORKSPACE
    assert _call_union(cfg, cache, segs, q=18) == qsa.QSA_ERR_INVALID_ARG
    assert _call_union(cfg, cache, segs, sel=None) == qsa.QSA_ERR_INVALID_ARG
    assert _call_union(cfg, cache, qsa.make_segments([(0, 0, 100, 0)]), T=0, ws=None, ws_bytes=0) == qsa.QSA_OK
    f32 = qsa.make_config(synth.Shape(dtype="f32"))
    assert _call_union(f32, cache, segs) == qsa.QSA_ERR_UNSUPPORTED


def test_missing_library_fails_loudly():
    """No fallback: without the built library every entry point raises."""
    import subprocess
    import sys
    code = ("import block_sparse_attention_22_b200 as q\n"
            "q.LIB_PATH = q.LIB_PATH + '.absent'\n"
            "q.qsa_device_status()\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "not built" in r.stderr


def test_product_never_reaches_the_oracle():
    """The library and its binding neither import, load nor link the oracle."""
    import ast
    pkg = os.path.join(ROOT, "block_sparse_attention_22_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            tree = ast.parse(open(os.path.join(pkg, fn)).read())
            for node in ast.walk(tree):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    names = [a.name for a in node.names] + [getattr(node, "module", None) or ""]
                    assert not any("oracle" in n for n in names), (fn, names)
    csrc = os.path.join(pkg, "csrc")
    for fn in os.listdir(csrc):
        src = open(os.path.join(csrc, fn)).read()
        assert "qsa_oracle" not in src and "qsa_ref_" not in src, fn
    deps = os.popen(f"ldd {qsa.LIB_PATH}").read()
    assert "oracle" not in deps
    syms = os.popen(f"nm -D {qsa.LIB_PATH}").read()
    assert "qsa_ref_" not in syms
