// qsa_api.cu -- the C ABI of libqsa.so (declared in include/qsa.h).
//
// Host side only: validates arguments (before anything is enqueued), splits
// the segment list into launch-sized tables, picks kernels by I/O dtype and
// enqueues them on the caller's stream.  It never allocates, never
// synchronises (except qsa_device_status, a diagnostic) and keeps no state
// beyond per-function attribute set-up.
//
// One translation unit: every kernel file is included here.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <functional>
#include <vector>

#include "qsa_internal.cuh"
#include "compress.cuh"
#include "index_simt.cuh"
#include "topk.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "attn_union_tc.cuh"
#include "index_tc.cuh"
#include "prefix.cuh"

#include <cudaTypedefs.h>

#define QSA_API extern "C" __attribute__((visibility("default")))

namespace qsa {
namespace {

constexpr int kNumSms = 148;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int rope_dims_of(const qsa_config_t* c) {
  int d = (int)floor((double)c->idx_dim * (double)c->rope_fraction);
  return d - (d & 1);
}

qsa_status_t check_cfg(const qsa_config_t* c) {
  if (!c) return QSA_ERR_INVALID_ARG;
  if (c->r <= 0 || c->budget_tokens <= 0 || c->n_q_heads <= 0 || c->n_kv_groups <= 0 ||
      c->head_dim <= 0 || c->idx_heads <= 0 || c->idx_dim <= 0)
    return QSA_ERR_INVALID_ARG;
  if (c->budget_tokens % c->r != 0 || c->n_q_heads % c->n_kv_groups != 0) return QSA_ERR_INVALID_ARG;
  if (!(c->rope_fraction >= 0.f && c->rope_fraction <= 1.f) || !(c->rope_base > 0.0))
    return QSA_ERR_INVALID_ARG;
  if (c->dtype != QSA_DTYPE_F32 && c->dtype != QSA_DTYPE_BF16) return QSA_ERR_INVALID_ARG;
  if (c->r != 4 || c->head_dim != kHeadDim || c->idx_heads != 4 ||
      (c->idx_dim != 64 && c->idx_dim != 128))
    return QSA_ERR_UNSUPPORTED;
  if (c->n_q_heads / c->n_kv_groups > kMaxHpg) return QSA_ERR_UNSUPPORTED;
  if (c->budget_tokens / c->r > kMaxBudgetBlocks) return QSA_ERR_UNSUPPORTED;
  if (rope_dims_of(c) / 2 > kMaxRopeHalf) return QSA_ERR_UNSUPPORTED;
  if (c->dtype == QSA_DTYPE_BF16 && rope_dims_of(c) / 2 > tc_index::kMaxRopeHalf) return QSA_ERR_UNSUPPORTED;
  return QSA_OK;
}

qsa_status_t check_cache(const qsa_config_t* c, const qsa_cache_t* k) {
  if (!k || k->n_slots <= 0 || k->n_cap <= 0 || k->n_cap % c->r != 0) return QSA_ERR_INVALID_ARG;
  if (k->n_cap > ((int64_t)1 << 31) - 1) return QSA_ERR_UNSUPPORTED;
  return QSA_OK;
}

qsa_status_t check_segments(const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                            const qsa_cache_t* cache, int64_t n_cap_if_no_cache) {
  if (n_segs < 0 || n_tokens < 0 || (n_segs > 0 && !segs)) return QSA_ERR_INVALID_ARG;
  const int64_t n_cap = cache ? cache->n_cap : n_cap_if_no_cache;
  for (int i = 0; i < n_segs; ++i) {
    const qsa_segment_t& s = segs[i];
    if (s.q_len < 0 || s.q_offset < 0 || s.pos0 < 0) return QSA_ERR_INVALID_ARG;
    if ((int64_t)s.q_offset + s.q_len > n_tokens) return QSA_ERR_INVALID_ARG;
    if (n_cap > 0 && (int64_t)s.pos0 + s.q_len > n_cap) return QSA_ERR_INVALID_ARG;
    if (cache && (s.slot < 0 || s.slot >= cache->n_slots)) return QSA_ERR_INVALID_ARG;
  }
  return QSA_OK;
}

Geo make_geo(const qsa_config_t* c, const qsa_cache_t* k) {
  Geo g;
  memset(&g, 0, sizeof g);
  g.r = c->r;
  g.S = c->budget_tokens / c->r;
  g.H = c->n_q_heads;
  g.G = c->n_kv_groups;
  g.hpg = c->n_q_heads / c->n_kv_groups;
  g.HI = c->idx_heads;
  g.DI = c->idx_dim;
  const int rd = rope_dims_of(c);
  g.rope_half = rd / 2;
  g.scale = c->softmax_scale > 0.f ? c->softmax_scale : (float)(1.0 / sqrt((double)c->head_dim));
  g.n_slots = k ? k->n_slots : 0;
  g.n_cap = k ? k->n_cap : 0;
  for (int i = 0; i < g.rope_half; ++i) g.theta[i] = pow(c->rope_base, -(2.0 * (double)i) / (double)rd);
  return g;
}

int64_t seg_max_blocks(const qsa_segment_t* segs, int n, int r) {
  int64_t m = 0;
  for (int i = 0; i < n; ++i)
    if (segs[i].q_len > 0) m = std::max<int64_t>(m, ((int64_t)segs[i].pos0 + segs[i].q_len - 1) / r);
  return m;
}

int64_t seg_rows(const qsa_segment_t* segs, int n) {
  int64_t t = 0;
  for (int i = 0; i < n; ++i) t += std::max(0, segs[i].q_len);
  return t;
}

// Calls launch(table) for batches of at most kMaxSegs non-empty segments;
// items(seg) gives each segment's work-item count; extra (or null) the
// segments' SegExtra fields.
template <typename Items, typename Launch>
qsa_status_t for_each_table(const qsa_segment_t* segs, int n_segs, Items items, Launch launch,
                            const SegExtra* extra = nullptr) {
  SegTable st;
  memset(&st, 0, sizeof st);
  auto flush = [&]() -> qsa_status_t {
    if (st.n == 0 || st.item0[st.n] == 0) {
      st.n = 0;
      return QSA_OK;
    }
    cudaError_t e = launch(st);
    st.n = 0;
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
  };
  for (int i = 0; i < n_segs; ++i) {
    const qsa_segment_t& s = segs[i];
    if (s.q_len <= 0) continue;
    const int64_t it = items(s);
    if (st.n > 0 && ((int64_t)st.item0[st.n] + it > INT32_MAX / 2)) {
      qsa_status_t r = flush();
      if (r != QSA_OK) return r;
    }
    st.q_offset[st.n] = s.q_offset;
    st.q_len[st.n] = s.q_len;
    st.pos0[st.n] = s.pos0;
    st.slot[st.n] = s.slot;
    const SegExtra e = extra ? extra[i] : SegExtra{0, 0, 0, 0};
    st.blk_lo[st.n] = e.blk_lo;
    st.blk_cap[st.n] = e.blk_cap;
    st.pslot[st.n] = e.pslot;
    st.pblk[st.n] = e.pblk;
    if (st.n == 0) st.item0[0] = 0;
    st.item0[st.n + 1] = st.item0[st.n] + (int32_t)it;
    st.n++;
    if (st.n == kMaxSegs) {
      qsa_status_t r = flush();
      if (r != QSA_OK) return r;
    }
  }
  return flush();
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int sm_count();

// ------------------------------------------------------------------ selection plan
struct TopkPlan {
  bool wide;       // few rows: one wide CTA per row
  bool hist;       // few long rows: 4096-score chunks sharing a row histogram
  size_t ws;
  size_t zero;     // leading workspace bytes to clear before the launches
};

// Workspace of the few-long-rows selection, per token row: a record of
// counters and the histogram (cleared first), a list of S-1 indices and a
// list of CAP key/index pairs.
struct TopkHistLayout {
  size_t rec, hist, sure, key, idx, zero, total;
};

TopkHistLayout topk_hist_layout(int64_t T) {
  TopkHistLayout L;
  L.rec = 0;
  L.hist = (size_t)T * topk::kRecWords * 4;
  L.zero = align_up(L.hist + (size_t)T * (topk::kHistBins + topk::kCoarseBins) * 4, 256);
  L.sure = L.zero;
  L.key = L.sure + align_up((size_t)T * topk::KMAX * 4, 256);
  L.idx = L.key + align_up((size_t)T * topk::CAP * 4, 256);
  L.total = L.idx + align_up((size_t)T * topk::CAP * 4, 256);
  return L;
}

// Many rows: one 4-warp CTA per row.  Few rows (too few to fill the GPU with
// 4-warp CTAs): one 32-warp CTA per row while rows are short, else 4096-score
// chunks sharing a histogram of the row's top key bits, in three launches:
// histograms, filter, final selection (one CTA per row).
TopkPlan topk_plan(const Geo& g, const qsa_segment_t* segs, int n) {
  TopkPlan p{false, false, 0, 0};
  const int64_t nblk = seg_max_blocks(segs, n, g.r);
  const int64_t rows = seg_rows(segs, n);
  if (nblk + 1 <= g.S || rows >= 4 * kNumSms) return p;
  if (nblk <= topk::kWideMaxBlocks) {
    p.wide = true;
    return p;
  }
  p.hist = true;
  int64_t T = 0;
  for (int i = 0; i < n; ++i) T = std::max<int64_t>(T, (int64_t)segs[i].q_offset + segs[i].q_len);
  const TopkHistLayout L = topk_hist_layout(T);
  p.zero = L.zero;
  p.ws = L.total;
  return p;
}

// ------------------------------------------------------------------ attention plan
struct AttnPlan {
  int n_split;
  int blocks_per_split;
  size_t ws;
};

// bf16 runs on the tensor-core kernel (splits in whole 32-block chunks,
// one CTA per SM: as many splits as keep every (query, group) split in one
// round of CTAs), fp32 on the CUDA-core kernel (8-block chunks, several
// CTAs per SM).
AttnPlan attn_plan(const Geo& g, const qsa_segment_t* segs, int n, bool tc) {
  int64_t T = 0;
  for (int i = 0; i < n; ++i) T = std::max<int64_t>(T, (int64_t)segs[i].q_offset + segs[i].q_len);
  const int64_t units = seg_rows(segs, n) * g.G;
  AttnPlan p{1, g.S, 0};
  const int gran = tc ? tc_attn::kBlk : simt_attn::KC / 4;
  const int64_t slots = tc ? kNumSms : 2 * kNumSms;      // fixed: workspace sizes make no CUDA call
  if (units > 0 && units * 2 <= slots) {
    int ns = (int)std::min<int64_t>(tc ? slots / units : cdiv(slots, units), cdiv(g.S, gran));
    p.blocks_per_split = (int)(cdiv(cdiv(g.S, ns), gran) * gran);
    p.n_split = (int)cdiv(g.S, p.blocks_per_split);
  }
  if (p.n_split > 1)
    p.ws = align_up((size_t)T * g.G * p.n_split * g.hpg * kHeadDim * 4, 256) +
           align_up((size_t)T * g.G * p.n_split * g.hpg * 2 * 4, 256);
  return p;
}

// ------------------------------------------------------------------ stage launchers
qsa_status_t run_compress(const Geo& g, const qsa_config_t* c, const qsa_cache_t* cache,
                          const int32_t* slots, const int64_t* b0, const int64_t* b1, int n,
                          cudaStream_t st, bool late_wait = false) {
  RangeTable rt;
  memset(&rt, 0, sizeof rt);
  auto flush = [&]() -> qsa_status_t {
    if (rt.n == 0) return QSA_OK;
    cudaError_t e = c->dtype == QSA_DTYPE_BF16
                        ? launch_compress<__nv_bfloat16>(g, rt, cache->k_idx, cache->khat, st, late_wait)
                        : launch_compress<float>(g, rt, cache->k_idx, cache->khat, st, late_wait);
    rt.n = 0;
    return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
  };
  for (int i = 0; i < n; ++i) {
    if (b1[i] <= b0[i]) continue;
    rt.slot[rt.n] = slots[i];
    rt.b0[rt.n] = b0[i];
    if (rt.n == 0) rt.item0[0] = 0;
    rt.item0[rt.n + 1] = rt.item0[rt.n] + (b1[i] - b0[i]);
    if (++rt.n == kMaxSegs) {
      qsa_status_t r = flush();
      if (r != QSA_OK) return r;
    }
  }
  return flush();
}

// Tensor map of the k^ cache (every stride-th pooled block of each slot).
bool make_khat_map(CUtensorMap* m, const qsa_config_t* c, const qsa_cache_t* cache, int stride);
int sm_count();

template <int NQ>
cudaError_t launch_index_tc(const Geo& g, const SegTable& t, const CUtensorMap& tm, const IndexTcArgs& a,
                            cudaStream_t st) {
  const int units = t.item0[t.n];
  if (units == 0) return cudaSuccess;
  const int smem = IndexTcCfg<NQ>::kSmemBytes;
  cudaFuncSetAttribute(index_tc_kernel<NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  count_launch();
  // persistent: one CTA per SM, each an equal slice of the work units
  const int grid = std::min(units, sm_count());
  return launch_chained(index_tc_kernel<NQ>, dim3(grid), dim3(IndexTcCfg<NQ>::kThreads), smem, st, tm, g, t, a);
}

qsa_status_t run_index(const Geo& g, const qsa_config_t* c, const qsa_cache_t* cache,
                       const qsa_segment_t* segs, int n, const void* q_idx, const float* w,
                       float* scores, int64_t ld, cudaStream_t st, const SegExtra* extra = nullptr) {
  if (c->dtype == QSA_DTYPE_BF16) {
    CUtensorMap tm;
    if (!make_khat_map(&tm, c, cache, 1)) return QSA_ERR_CUDA;
    IndexTcArgs a{};
    a.q_idx = (const __nv_bfloat16*)q_idx;
    a.w = w;
    a.scores = scores;
    a.ld = ld;
    a.stride = 1;
    // prefill-like segments on 64-query tiles, decode-like ones on 4-query tiles
    std::vector<qsa_segment_t> wide, narrow;
    std::vector<SegExtra> xw, xn;
    for (int i = 0; i < n; ++i) {
      const bool wd = segs[i].q_len >= 16;
      (wd ? wide : narrow).push_back(segs[i]);
      (wd ? xw : xn).push_back(extra ? extra[i] : SegExtra{0, 0, 0, 0});
    }
    qsa_status_t r = for_each_table(
        wide.data(), (int)wide.size(),
        [&](const qsa_segment_t& s) {
          const SegExtra& e = xw[&s - wide.data()];
          return index_tc_units<64>(s.q_len, s.pos0, g.r, 1, e.blk_lo, e.blk_cap);
        },
        [&](const SegTable& t) { return launch_index_tc<64>(g, t, tm, a, st); }, xw.data());
    if (r != QSA_OK) return r;
    return for_each_table(
        narrow.data(), (int)narrow.size(),
        [&](const qsa_segment_t& s) {
          const SegExtra& e = xn[&s - narrow.data()];
          return index_tc_units<4>(s.q_len, s.pos0, g.r, 1, e.blk_lo, e.blk_cap);
        },
        [&](const SegTable& t) { return launch_index_tc<4>(g, t, tm, a, st); }, xn.data());
  }
  size_t smem = sizeof(float) * (simt_index::QT * g.HI * g.DI + simt_index::QT * g.HI);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(index_scores_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return for_each_table(
      segs, n, [&](const qsa_segment_t& s) { return (int64_t)simt_index_items(s.q_len, s.pos0, g.r); },
      [&](const SegTable& t) { return launch_index_simt<float>(g, t, q_idx, w, cache->khat, scores, ld, st); });
}

// Fused selection of prefill-like bf16 segments (no score matrix): sample
// scores, row thresholds, filtered scoring into candidate lists, selection.
struct FusedBufs {
  float* samples;
  int64_t ld_s;
  float* tau;
  float* cand_score;
  int32_t* cand_idx;
  int32_t* cand_cnt;
};

qsa_status_t run_fused_select(const Geo& g, const qsa_config_t* c, const qsa_cache_t* cache,
                              const qsa_segment_t* segs, int n, const void* q_idx, const float* w,
                              const FusedBufs& f, int32_t* sel, int32_t* nsel, cudaStream_t st,
                              const std::function<qsa_status_t()>& after_filter = nullptr) {
  constexpr int kStride = topk::kFusedStride;
  CUtensorMap tm_s, tm;
  if (!make_khat_map(&tm_s, c, cache, kStride) || !make_khat_map(&tm, c, cache, 1)) return QSA_ERR_CUDA;
  // prefill-like segments on 64-query index tiles, decode-like ones on 4-query tiles
  std::vector<qsa_segment_t> wide, narrow;
  for (int i = 0; i < n; ++i) (segs[i].q_len >= 16 ? wide : narrow).push_back(segs[i]);
  auto index_pass = [&](const IndexTcArgs& a, const CUtensorMap& m) -> qsa_status_t {
    qsa_status_t r = for_each_table(
        wide.data(), (int)wide.size(),
        [&](const qsa_segment_t& s) { return index_tc_units<64>(s.q_len, s.pos0, g.r, a.stride); },
        [&](const SegTable& t) { return launch_index_tc<64>(g, t, m, a, st); });
    if (r != QSA_OK) return r;
    return for_each_table(
        narrow.data(), (int)narrow.size(),
        [&](const qsa_segment_t& s) { return index_tc_units<4>(s.q_len, s.pos0, g.r, a.stride); },
        [&](const SegTable& t) { return launch_index_tc<4>(g, t, m, a, st); });
  };
  IndexTcArgs a{};
  a.q_idx = (const __nv_bfloat16*)q_idx;
  a.w = w;
  a.scores = f.samples;
  a.ld = f.ld_s;
  a.stride = kStride;
  qsa_status_t r = index_pass(a, tm_s);
  if (r != QSA_OK) return r;
  FusedSelArgs fa;
  memset(&fa, 0, sizeof fa);
  fa.samples = f.samples;
  fa.ld_s = f.ld_s;
  fa.stride = kStride;
  fa.tau = f.tau;
  fa.cand_score = f.cand_score;
  fa.cand_idx = f.cand_idx;
  fa.cand_cnt = f.cand_cnt;
  fa.sel = sel;
  fa.nsel = nsel;
  fa.q_idx = (const __nv_bfloat16*)q_idx;
  fa.w = w;
  fa.khat = (const __nv_bfloat16*)cache->khat;
  // many rows: a 4-warp CTA per row, six per SM; few rows: 32 warps per row
  const bool many = seg_rows(segs, n) >= 4 * kNumSms;
  const int ctas = 6 * sm_count();
  auto rows = [](const qsa_segment_t& s) { return (int64_t)s.q_len; };
  auto per_row = [&](auto kernel_many, auto kernel_few) {
    return for_each_table(segs, n, rows, [&](const SegTable& t) {
      count_launch();
      const int items = t.item0[t.n];
      return many ? launch_chained(kernel_many, dim3(std::min(items, ctas)), dim3(topk::THREADS), 0, st, g, t, fa)
                  : launch_chained(kernel_few, dim3(items), dim3(topk::kWideThreads), 0, st, g, t, fa);
    });
  };
  r = per_row(topk_tau_kernel<topk::THREADS>, topk_tau_kernel<topk::kWideThreads>);
  if (r != QSA_OK) return r;
  a.scores = nullptr;
  a.ld = 0;
  a.stride = 1;
  a.tau = f.tau;
  a.cand_score = f.cand_score;
  a.cand_idx = f.cand_idx;
  a.cand_cnt = f.cand_cnt;
  a.cand_cap = topk::CAP;
  if ((r = index_pass(a, tm)) != QSA_OK) return r;
  if (after_filter && (r = after_filter()) != QSA_OK) return r;
  return per_row(topk_cand_kernel<topk::THREADS>, topk_cand_kernel<topk::kWideThreads>);
}

qsa_status_t run_select(const Geo& g, const qsa_segment_t* segs, int n, const float* scores,
                        int64_t ld, int32_t* sel, int32_t* nsel, void* ws, size_t ws_bytes,
                        cudaStream_t st) {
  const TopkPlan p = topk_plan(g, segs, n);
  if (p.ws > 0 && (!ws || ws_bytes < p.ws)) return QSA_ERR_WORKSPACE;
  TopkArgs a;
  memset(&a, 0, sizeof a);
  a.scores = scores;
  a.ld = ld;
  a.sel = sel;
  a.nsel = nsel;
  a.chunk = topk::kHistChunk;
  if (p.hist) {
    int64_t T = 0;
    for (int i = 0; i < n; ++i) T = std::max<int64_t>(T, (int64_t)segs[i].q_offset + segs[i].q_len);
    const TopkHistLayout L = topk_hist_layout(T);
    char* base = (char*)ws;
    a.hrec = (int32_t*)(base + L.rec);
    a.hhist = (uint32_t*)(base + L.hist);
    a.hsure = (int32_t*)(base + L.sure);
    a.hkey = (uint32_t*)(base + L.key);
    a.hidx = (int32_t*)(base + L.idx);
    if (cudaMemsetAsync(ws, 0, L.zero, st) != cudaSuccess) return QSA_ERR_CUDA;
  }
  const size_t smem_c = 0;
  if (p.wide) {
    return for_each_table(
        segs, n, [&](const qsa_segment_t& s) { return (int64_t)s.q_len; },
        [&](const SegTable& t) {
          cudaFuncSetAttribute(topk_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, topk::kWideRingBytes);
          count_launch();
          return launch_chained(topk_wide_kernel, dim3(t.item0[t.n]), dim3(topk::kWideThreads), topk::kWideRingBytes, st, g, t, a);
        });
  }
  if (p.hist) {
    return for_each_table(
        segs, n,
        [&](const qsa_segment_t& s) {
          const int64_t nb = ((int64_t)s.pos0 + s.q_len - 1) / g.r;
          return (int64_t)s.q_len * std::max<int64_t>(1, cdiv(nb, topk::kHistChunk));
        },
        [&](const SegTable& t) {
          count_launch();
          cudaError_t e = launch_chained(topk_hist_kernel, dim3(t.item0[t.n]), dim3(topk::kHistThreads), 0, st, g,
                                         t, a);
          if (e != cudaSuccess) return e;
          count_launch();
          e = launch_chained(topk_hfilter_kernel, dim3(t.item0[t.n]), dim3(topk::kHistThreads), 0, st, g, t, a);
          if (e != cudaSuccess) return e;
          SegTable rt = t;                                   // one item per row
          rt.item0[0] = 0;
          for (int i = 0; i < t.n; ++i) rt.item0[i + 1] = rt.item0[i] + t.q_len[i];
          count_launch();
          return launch_chained(topk_hfinal_kernel, dim3(rt.item0[rt.n]), dim3(topk::kWideThreads), 0, st, g, rt,
                                a);
        });
  }
  (void)smem_c;
  // many rows: one warp per row (topk_w::CTAS 4-warp CTAs per SM), then a CTA-level
  // selection of the rows it left (long rows, sampled thresholds that
  // missed).  Plain launches: chained, the pair ran 1.7x slower (the
  // dependent's CTAs, resident early, held the SMs the other grid needed).
  return for_each_table(
      segs, n, [&](const qsa_segment_t& s) { return (int64_t)s.q_len; },
      [&](const SegTable& t) {
        const int rows = t.item0[t.n];
        const int grid = std::min((int)cdiv(rows, topk_w::WARPS), topk_w::CTAS * sm_count());
        constexpr int smem_rows = (int)(topk_w::WARPS * sizeof(WarpRowShared));
        cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_rows);
        count_launch();
        topk_rows_kernel<<<dim3(grid), dim3(topk_w::THREADS), smem_rows, st>>>(g, t, a);
        count_launch();
        topk_rows_fallback_kernel<<<dim3(std::min(rows, 6 * sm_count())), dim3(topk::THREADS), 0, st>>>(g, t, a);
        return cudaGetLastError();
      });
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][inner] (row stride inner*2 bytes), box box_inner x
// box_rows, 128-byte swizzle, out-of-range rows read as zero.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                   uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of the k^ cache as [n_slots][rows][idx_dim] bf16 with row j of
// a slot = pooled block j*stride (stride 1: every block), boxes of 64 dims x
// 128 rows x 1 slot, 128-byte swizzle; rows past a slot's end read as zero.
bool make_khat_map(CUtensorMap* m, const qsa_config_t* c, const qsa_cache_t* cache, int stride) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const uint64_t blocks = (uint64_t)(cache->n_cap / c->r), di = (uint64_t)c->idx_dim;
  cuuint64_t dims[3] = {di, (blocks + stride - 1) / stride, (uint64_t)cache->n_slots};
  cuuint64_t strides[2] = {di * 2 * stride, di * 2 * blocks};
  cuuint32_t box[3] = {64, (cuuint32_t)tc_index::kTileRows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, cache->khat, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return kNumSms;
  return n > 0 ? n : kNumSms;
}

qsa_status_t run_attn(const Geo& g, const qsa_config_t* c, const qsa_cache_t* cache,
                      const qsa_segment_t* segs, int n, int32_t n_tokens, const void* q, const int32_t* sel,
                      const int32_t* nsel, void* o, float* lse, void* ws, size_t ws_bytes,
                      cudaStream_t st, const SegExtra* extra = nullptr) {
  const bool bf = c->dtype == QSA_DTYPE_BF16;
  const AttnPlan p = attn_plan(g, segs, n, bf);
  if (p.ws > 0 && (!ws || ws_bytes < p.ws)) return QSA_ERR_WORKSPACE;
  AttnArgs a;
  memset(&a, 0, sizeof a);
  a.q = q;
  a.k = cache->k;
  a.v = cache->v;
  a.sel = sel;
  a.nsel = nsel;
  a.o = o;
  a.lse = lse;
  a.n_split = p.n_split;
  a.blocks_per_split = p.blocks_per_split;
  if (p.n_split > 1) {
    int64_t T = 0;
    for (int i = 0; i < n; ++i) T = std::max<int64_t>(T, (int64_t)segs[i].q_offset + segs[i].q_len);
    a.part_o = (float*)ws;
    a.part_ml = (float*)((char*)ws + align_up((size_t)T * g.G * p.n_split * g.hpg * kHeadDim * 4, 256));
  }
  qsa_status_t r;
  if (bf) {
    CUtensorMap tq;
    if (!make_map_bf16(&tq, q, kHeadDim, (uint64_t)n_tokens * g.H, 64, (uint32_t)g.hpg)) return QSA_ERR_CUDA;
    AttnTcArgs ta;
    memset(&ta, 0, sizeof ta);
    ta.k = cache->k;
    ta.v = cache->v;
    ta.sel = sel;
    ta.nsel = nsel;
    ta.o = o;
    ta.lse = lse;
    ta.part_o = a.part_o;
    ta.part_ml = a.part_ml;
    ta.n_split = p.n_split;
    ta.blocks_per_split = p.blocks_per_split;
    const int smem = tc_attn::kSmemBytes;
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    const int sms = sm_count();
    r = for_each_table(
        segs, n, [&](const qsa_segment_t& s) { return (int64_t)s.q_len * p.n_split; },
        [&](const SegTable& t) {
          ta.units_per_group = t.item0[t.n];
          const int64_t units = ta.units_per_group * g.G;
          const int grid = (int)std::min<int64_t>(units, sms);
          count_launch();
          return launch_chained(attn_tc_kernel, dim3(grid), dim3(tc_attn::kThreads), smem, st, tq, g, t, ta);
        },
        extra);
  } else {
    const size_t smem = attn_simt_smem();
    cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    r = for_each_table(
        segs, n, [&](const qsa_segment_t& s) { return (int64_t)s.q_len * g.G * p.n_split; },
        [&](const SegTable& t) {
          count_launch();
          const cudaError_t e = launch_chained(attn_simt_kernel<float>, dim3(t.item0[t.n]), dim3(simt_attn::THREADS), smem, st, g, t, a);
          if (e != cudaSuccess) return e;
          return cudaGetLastError();
        });
  }
  if (r != QSA_OK || p.n_split == 1) return r;
  return for_each_table(
      segs, n, [&](const qsa_segment_t& s) { return (int64_t)s.q_len; },
      [&](const SegTable& t) {
        const int64_t total = (int64_t)t.item0[t.n] * g.H * (kHeadDim / 4);
        const unsigned blocks = (unsigned)std::min<int64_t>(cdiv(total, 256), kNumSms * 32);
        count_launch();
        return bf ? launch_chained(attn_combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st, g, t, a)
                  : launch_chained(attn_combine_kernel<float>, dim3(blocks), dim3(256), 0, st, g, t, a);
      });
}

// ------------------------------------------------------------------ union-tile attention
// Query tokens per union tile: as many as fill the 128 query rows of an MMA
// tile with one group's heads, at most the 32 bits of a member mask.
int union_mq(const Geo& g) { return std::min(tc_union::kMaxMembers, 128 / g.hpg); }

struct UnionPlan {
  int mq;
  int64_t tiles;
  int64_t cap;               // union entries per tile
  size_t off_blk, off_mask, ws;
};

UnionPlan union_plan(const Geo& g, const qsa_segment_t* segs, int n) {
  UnionPlan p;
  p.mq = union_mq(g);
  p.cap = (int64_t)p.mq * g.S;
  p.tiles = 0;
  for (int i = 0; i < n; ++i)
    if (segs[i].q_len > 0) p.tiles += union_tiles(segs[i].q_len, p.mq);
  p.off_blk = align_up((size_t)p.tiles * 4, 256);
  p.off_mask = p.off_blk + align_up((size_t)p.tiles * p.cap * 4, 256);
  p.ws = p.tiles > 0 ? p.off_mask + align_up((size_t)p.tiles * p.cap * 4, 256) : 0;
  return p;
}

qsa_status_t run_attn_union(const Geo& g, const qsa_segment_t* segs, int n, const qsa_cache_t* cache,
                            const void* q, const int32_t* sel, const int32_t* nsel, void* o, float* lse,
                            void* ws, size_t ws_bytes, cudaStream_t st) {
  const UnionPlan p = union_plan(g, segs, n);
  if (p.ws > 0 && (!ws || ws_bytes < p.ws)) return QSA_ERR_WORKSPACE;
  // the union build holds a bitmap of the context's blocks and its prefix in shared memory
  const int64_t max_words = cdiv(seg_max_blocks(segs, n, g.r) + 1, 32);
  if (((size_t)2 * max_words + (size_t)p.cap) * 4 > (size_t)227 * 1024) return QSA_ERR_UNSUPPORTED;
  UnionBuildArgs ba;
  memset(&ba, 0, sizeof ba);
  ba.sel = sel;
  ba.nsel = nsel;
  ba.ulen = (int32_t*)ws;
  ba.ublk = (int32_t*)((char*)ws + p.off_blk);
  ba.umask = (uint32_t*)((char*)ws + p.off_mask);
  ba.cap = p.cap;
  ba.mq = p.mq;
  AttnUnionArgs ta;
  memset(&ta, 0, sizeof ta);
  ta.q = q;
  ta.k = cache->k;
  ta.v = cache->v;
  ta.ulen = ba.ulen;
  ta.ublk = ba.ublk;
  ta.umask = ba.umask;
  ta.cap = p.cap;
  ta.mq = p.mq;
  ta.o = o;
  ta.lse = lse;
  cudaFuncSetAttribute(attn_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc_union::kSmemBytes);
  const int sms = sm_count();
  int64_t tile_base = 0;
  return for_each_table(
      segs, n, [&](const qsa_segment_t& s) { return union_tiles(s.q_len, p.mq); },
      [&](const SegTable& t) -> cudaError_t {
        const int64_t tiles = t.item0[t.n];
        int64_t nb = 1;
        for (int i = 0; i < t.n; ++i) nb = std::max<int64_t>(nb, ((int64_t)t.pos0[i] + t.q_len[i] - 1) / g.r + 1);
        ba.words = (int)cdiv(nb, 32);
        ba.tile_base = tile_base;
        const size_t smem = ((size_t)2 * ba.words + (size_t)p.cap) * 4;
        if (cudaFuncSetAttribute(union_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
          return cudaErrorInvalidValue;
        count_launch();
        union_build_kernel<<<dim3((unsigned)tiles), dim3(tc_union::kBuildThreads), smem, st>>>(g, t, ba);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ta.tiles = tiles;
        ta.tile_base = tile_base;
        const int grid = (int)std::min<int64_t>(tiles * g.G, sms);
        count_launch();
        attn_union_kernel<<<dim3(grid), dim3(tc_attn::kThreads), tc_union::kSmemBytes, st>>>(g, t, ta);
        tile_base += tiles;
        return cudaGetLastError();
      });
}

// ------------------------------------------------------------------ forward workspace
// Segments that select through the fused path (no score rows): in the
// low-memory forward, the bf16 prefill-like segments (64-query index tiles).
// Decode-like segments keep their score rows in both forwards: their rows are
// few, and for them the sample pass, the thresholds and the candidate
// selection took longer than the split selection they replace (1M-context
// decode step 0.164 ms against 0.144 ms).
bool fused_segment(const qsa_segment_t& s, bool tc, bool lowmem, int r) {
  (void)r;
  return lowmem && tc && s.q_len >= 16;
}

void split_fused(const qsa_segment_t* segs, int n, bool tc, bool lowmem, int r, std::vector<qsa_segment_t>& fused,
                 std::vector<qsa_segment_t>& plain) {
  for (int i = 0; i < n; ++i) (fused_segment(segs[i], tc, lowmem, r) ? fused : plain).push_back(segs[i]);
}

struct FwdLayout {
  int64_t ld;      // score rows of the plain segments
  int64_t ld_s;    // sample rows of the fused segments
  size_t scores, sel, nsel, topk, attn, samples, tau, cnt, ckey, cidx, qrot, wrot, rmap, total;
};

FwdLayout fwd_layout(const Geo& g, const qsa_segment_t* segs, int n, int32_t n_tokens, bool tc, bool lowmem,
                     bool prefixed = false) {
  std::vector<qsa_segment_t> fused, plain;
  split_fused(segs, n, tc, lowmem, g.r, fused, plain);
  FwdLayout L;
  L.ld = std::max<int64_t>(4, cdiv(seg_max_blocks(plain.data(), (int)plain.size(), g.r), 4) * 4);
  const int64_t nb_f = seg_max_blocks(fused.data(), (int)fused.size(), g.r);
  L.ld_s = std::max<int64_t>(4, cdiv(cdiv(nb_f, topk::kFusedStride), 4) * 4);
  const size_t T = (size_t)n_tokens;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align_up(bytes, 256);
    return at;
  };
  L.scores = take(plain.empty() ? 0 : T * L.ld * 4);
  L.sel = take(T * g.S * 4);
  L.nsel = take(T * 4);
  L.topk = take(topk_plan(g, plain.data(), (int)plain.size()).ws);
  L.attn = take(attn_plan(g, segs, n, tc).ws);
  const bool f = !fused.empty();
  L.samples = take(f ? T * L.ld_s * 4 : 0);
  L.tau = take(f ? T * 4 : 0);
  L.cnt = take(f ? T * 4 : 0);
  L.ckey = take(f ? T * topk::CAP * 4 : 0);
  L.cidx = take(f ? T * topk::CAP * 4 : 0);
  // shared prefixes: the sharing queries' rotated rows, head weights and score rows
  L.qrot = take(prefixed ? T * 4 * g.DI * 2 : 0);
  L.wrot = take(prefixed ? T * 16 : 0);
  L.rmap = take(prefixed ? T * 4 : 0);
  L.total = off;
  return L;
}

// Scores of the queries that share a cached prefix, over the prefix's blocks:
// the sequences with the same (prefix slot, length) form one capped segment
// of the indexer over that slot (up to 16 queries per k^ stream), whose
// queries were rotated at their own positions into workspace rows.
qsa_status_t run_index_shared(const Geo& g, const qsa_config_t* c, const qsa_cache_t* cache,
                              const qsa_segment_t* segs, const qsa_prefix_t* prefix, int n, const void* q_idx,
                              const float* w, float* scores, int64_t ld, __nv_bfloat16* q_rot, float* w_rot,
                              int32_t* row_map, cudaStream_t st) {
  // members of each (slot, blocks) group, in segment order
  std::vector<std::pair<std::pair<int, int>, std::vector<int>>> groups;
  for (int i = 0; i < n; ++i) {
    if (segs[i].q_len <= 0 || prefix[i].blocks <= 0) continue;
    const std::pair<int, int> key{prefix[i].slot, prefix[i].blocks};
    auto it = std::find_if(groups.begin(), groups.end(), [&](const auto& gr) { return gr.first == key; });
    if (it == groups.end()) {
      groups.push_back({key, {}});
      it = groups.end() - 1;
    }
    it->second.push_back(i);
  }
  if (groups.empty()) return QSA_OK;
  // 1. rotated rows: virtual row v = the v-th member query, group by group
  std::vector<qsa_segment_t> members, shared;
  std::vector<SegExtra> xs;
  int32_t v0 = 0;
  for (const auto& gr : groups) {
    int32_t m = 0;
    for (int i : gr.second) {
      members.push_back(segs[i]);
      m += segs[i].q_len;
    }
    // one capped segment per group: rows [v0, v0 + m) of the rotated buffers
    shared.push_back(qsa_segment_t{v0, m, gr.first.second * g.r, gr.first.first});
    xs.push_back(SegExtra{0, gr.first.second, 0, 0});
    v0 += m;
  }
  PrefixRotArgs ra{(const __nv_bfloat16*)q_idx, w, q_rot, w_rot, row_map};
  int32_t vbase = 0;
  qsa_status_t r = for_each_table(
      members.data(), (int)members.size(), [&](const qsa_segment_t& s) { return (int64_t)s.q_len; },
      [&](const SegTable& t) {
        PrefixRotArgs at = ra;                          // rows of this table start at vbase
        at.q_rot = q_rot + (int64_t)vbase * 4 * g.DI;
        at.w_rot = w_rot + (int64_t)vbase * 4;
        at.row_map = row_map + vbase;
        vbase += t.item0[t.n];
        count_launch();
        return launch_chained(prefix_rotate_kernel, dim3((unsigned)t.item0[t.n] * 4), dim3(128), 0, st, g, t, at);
      });
  if (r != QSA_OK) return r;
  // 2. the capped segments over the prefix slots
  CUtensorMap tm;
  if (!make_khat_map(&tm, c, cache, 1)) return QSA_ERR_CUDA;
  IndexTcArgs a{};
  a.q_idx = q_rot;
  a.w = w_rot;
  a.scores = scores;
  a.ld = ld;
  a.stride = 1;
  a.prerotated = 1;
  a.row_map = row_map;
  return for_each_table(
      shared.data(), (int)shared.size(),
      [&](const qsa_segment_t& s) {
        const SegExtra& e = xs[&s - shared.data()];
        return index_tc_units<16>(s.q_len, s.pos0, g.r, 1, e.blk_lo, e.blk_cap);
      },
      [&](const SegTable& t) { return launch_index_tc<16>(g, t, tm, a, st); }, xs.data());
}

}  // namespace
}  // namespace qsa

using namespace qsa;

QSA_API qsa_status_t qsa_compress_keys(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                       const int32_t* slots, const int64_t* blk_begin,
                                       const int64_t* blk_end, int32_t n_ranges, void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if (n_ranges < 0 || (n_ranges > 0 && (!slots || !blk_begin || !blk_end))) return QSA_ERR_INVALID_ARG;
  if (n_ranges == 0) return QSA_OK;
  if (!cache->k_idx || !cache->khat || !aligned16(cache->k_idx) || !aligned16(cache->khat))
    return QSA_ERR_INVALID_ARG;
  for (int i = 0; i < n_ranges; ++i) {
    if (slots[i] < 0 || slots[i] >= cache->n_slots) return QSA_ERR_INVALID_ARG;
    if (blk_begin[i] < 0 || blk_end[i] < blk_begin[i] || blk_end[i] > cache->n_cap / cfg->r)
      return QSA_ERR_INVALID_ARG;
  }
  const Geo g = make_geo(cfg, cache);
  return run_compress(g, cfg, cache, slots, blk_begin, blk_end, n_ranges, (cudaStream_t)stream);
}

QSA_API qsa_status_t qsa_index_scores(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                      const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                      const void* q_idx, const float* w, float* scores,
                                      int64_t ld_scores, void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, cache, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!q_idx || !w || !scores || !cache->khat || !aligned16(q_idx) || !aligned16(cache->khat) ||
      !aligned16(w) || !aligned16(scores))
    return QSA_ERR_INVALID_ARG;
  if (ld_scores < std::max<int64_t>(1, seg_max_blocks(segs, n_segs, cfg->r))) return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, cache);
  return run_index(g, cfg, cache, segs, n_segs, q_idx, w, scores, ld_scores, (cudaStream_t)stream);
}

QSA_API qsa_status_t qsa_select_topk(const qsa_config_t* cfg, const qsa_segment_t* segs,
                                     int32_t n_segs, int32_t n_tokens, const float* scores,
                                     int64_t ld_scores, int32_t* sel, int32_t* nsel, void* workspace,
                                     size_t ws_bytes, void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, nullptr, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!scores || !sel || !nsel || !aligned16(sel)) return QSA_ERR_INVALID_ARG;
  const int64_t nblk = seg_max_blocks(segs, n_segs, cfg->r);
  if (ld_scores < std::max<int64_t>(1, nblk)) return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, nullptr);
  return run_select(g, segs, n_segs, scores, ld_scores, sel, nsel, workspace, ws_bytes,
                    (cudaStream_t)stream);
}

QSA_API qsa_status_t qsa_sparse_attn_fwd(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                         const qsa_segment_t* segs, int32_t n_segs,
                                         int32_t n_tokens, const void* q, const int32_t* sel,
                                         const int32_t* nsel, void* o, float* lse, void* workspace,
                                         size_t ws_bytes, void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, cache, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!q || !sel || !nsel || !o || !cache->k || !cache->v || !aligned16(q) || !aligned16(o) ||
      !aligned16(cache->k) || !aligned16(cache->v) || !aligned16(sel))
    return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, cache);
  return run_attn(g, cfg, cache, segs, n_segs, n_tokens, q, sel, nsel, o, lse, workspace, ws_bytes,
                  (cudaStream_t)stream);
}

QSA_API qsa_status_t qsa_sparse_attn_fwd_union(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                               const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                               const void* q, const int32_t* sel, const int32_t* nsel,
                                               void* o, float* lse, void* workspace, size_t ws_bytes,
                                               void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, cache, 0)) != QSA_OK) return s;
  if (cfg->dtype != QSA_DTYPE_BF16) return QSA_ERR_UNSUPPORTED;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!q || !sel || !nsel || !o || !cache->k || !cache->v || !aligned16(q) || !aligned16(o) ||
      !aligned16(cache->k) || !aligned16(cache->v) || !aligned16(sel))
    return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, cache);
  return run_attn_union(g, segs, n_segs, cache, q, sel, nsel, o, lse, workspace, ws_bytes,
                        (cudaStream_t)stream);
}

QSA_API qsa_status_t qsa_sparse_attn_bwd(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                         const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                         const void* q, const void* o, const float* lse, const void* dout,
                                         const int32_t* sel, const int32_t* nsel, float* dq, float* dk,
                                         float* dv, void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, cache, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!q || !o || !lse || !dout || !sel || !nsel || !dq || !dk || !dv || !cache->k || !cache->v)
    return QSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(cache->k) || !aligned16(cache->v))
    return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, cache);
  const bool bf = cfg->dtype == QSA_DTYPE_BF16;
  cudaStream_t st = (cudaStream_t)stream;
  if (bf) {
    // tensor cores: one CTA per SM, persistent over (query, group) units
    CUtensorMap tq, tdo;
    if (!make_map_bf16(&tq, q, kHeadDim, (uint64_t)n_tokens * g.H, 64, (uint32_t)g.hpg) ||
        !make_map_bf16(&tdo, dout, kHeadDim, (uint64_t)n_tokens * g.H, 64, (uint32_t)g.hpg))
      return QSA_ERR_CUDA;
    AttnBwdTcArgs ta{o, lse, dout, cache->k, cache->v, sel, nsel, dq, dk, dv, 0};
    const int smem_tc = tc_bwd::kSmemBytes;
    cudaFuncSetAttribute(attn_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_tc);
    const int sms = sm_count();
    return for_each_table(
        segs, n_segs, [&](const qsa_segment_t& sg) { return (int64_t)sg.q_len; },
        [&](const SegTable& t) {
          ta.units_per_group = t.item0[t.n];
          const int64_t units = ta.units_per_group * g.G;
          count_launch();
          return launch_chained(attn_bwd_tc_kernel, dim3((unsigned)std::min<int64_t>(units, sms)),
                                dim3(tc_bwd::kThreads), smem_tc, st, tq, tdo, g, t, ta);
        });
  }
  AttnBwdArgs a{q, o, lse, dout, cache->k, cache->v, sel, nsel, dq, dk, dv};
  const size_t smem = attn_bwd_smem();
  if (bf)
    cudaFuncSetAttribute(attn_bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  else
    cudaFuncSetAttribute(attn_bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return for_each_table(
      segs, n_segs, [&](const qsa_segment_t& sg) { return (int64_t)sg.q_len * g.G; },
      [&](const SegTable& t) {
        count_launch();
        return bf ? launch_chained(attn_bwd_kernel<__nv_bfloat16>, dim3(t.item0[t.n]), dim3(bwd_attn::THREADS),
                                   smem, st, g, t, a)
                  : launch_chained(attn_bwd_kernel<float>, dim3(t.item0[t.n]), dim3(bwd_attn::THREADS), smem,
                                   st, g, t, a);
      });
}

QSA_API size_t qsa_workspace_size(const qsa_config_t* cfg, const qsa_segment_t* segs,
                                  int32_t n_segs, int32_t n_tokens, qsa_op_t op) {
  if (check_cfg(cfg) != QSA_OK || check_segments(segs, n_segs, n_tokens, nullptr, 0) != QSA_OK)
    return SIZE_MAX;
  const Geo g = make_geo(cfg, nullptr);
  switch (op) {
    case QSA_OP_COMPRESS:
    case QSA_OP_INDEX: return 0;
    case QSA_OP_SELECT: return topk_plan(g, segs, n_segs).ws;
    case QSA_OP_ATTN: return attn_plan(g, segs, n_segs, cfg->dtype == QSA_DTYPE_BF16).ws;
    case QSA_OP_FORWARD: return fwd_layout(g, segs, n_segs, n_tokens, cfg->dtype == QSA_DTYPE_BF16, false).total;
    case QSA_OP_FORWARD_LOWMEM:
      return fwd_layout(g, segs, n_segs, n_tokens, cfg->dtype == QSA_DTYPE_BF16, true).total;
    case QSA_OP_ATTN_UNION: return union_plan(g, segs, n_segs).ws;
    case QSA_OP_FORWARD_PREFIXED:
      return fwd_layout(g, segs, n_segs, n_tokens, cfg->dtype == QSA_DTYPE_BF16, false, true).total;
  }
  return SIZE_MAX;
}

namespace qsa {
namespace {
// Checks of the shared-prefix table: every segment that shares a prefix
// lies wholly past it, in a cache that holds it.
qsa_status_t check_prefix(const qsa_config_t* cfg, const qsa_cache_t* cache, const qsa_segment_t* segs,
                          const qsa_prefix_t* prefix, int32_t n_segs) {
  if (n_segs > 0 && !prefix) return QSA_ERR_INVALID_ARG;
  for (int i = 0; i < n_segs; ++i) {
    const qsa_prefix_t& p = prefix[i];
    if (p.blocks < 0) return QSA_ERR_INVALID_ARG;
    if (p.blocks == 0 || segs[i].q_len <= 0) continue;
    if (p.slot < 0 || p.slot >= cache->n_slots) return QSA_ERR_INVALID_ARG;
    if ((int64_t)p.blocks * cfg->r > segs[i].pos0 || (int64_t)p.blocks * cfg->r > cache->n_cap)
      return QSA_ERR_INVALID_ARG;
  }
  return QSA_OK;
}

qsa_status_t forward_impl(const qsa_config_t* cfg, const qsa_cache_t* cache, const qsa_segment_t* segs,
                          int32_t n_segs, int32_t n_tokens, const void* q, const void* q_idx, const float* w,
                          void* o, float* lse, int32_t* sel, int32_t* nsel, void* workspace, size_t ws_bytes,
                          void* stream, bool lowmem, const qsa_prefix_t* prefix = nullptr) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_cache(cfg, cache)) != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, cache, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!q || !q_idx || !w || !o || !cache->k || !cache->v || !cache->k_idx || !cache->khat)
    return QSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(q_idx) || !aligned16(w) || !aligned16(o) || !aligned16(cache->k) ||
      !aligned16(cache->v) || !aligned16(cache->k_idx) || !aligned16(cache->khat))
    return QSA_ERR_INVALID_ARG;
  if ((sel == nullptr) != (nsel == nullptr) || (sel && !aligned16(sel))) return QSA_ERR_INVALID_ARG;
  std::vector<SegExtra> extra;
  if (prefix) {
    if ((s = check_prefix(cfg, cache, segs, prefix, n_segs)) != QSA_OK) return s;
    if (cfg->dtype != QSA_DTYPE_BF16 || lowmem) return QSA_ERR_UNSUPPORTED;
    for (int i = 0; i < n_segs; ++i)                       // decode-like segments only (< 16 queries)
      if (prefix[i].blocks > 0 && segs[i].q_len >= 16) return QSA_ERR_UNSUPPORTED;
    for (int i = 0; i < n_segs; ++i) {
      const int32_t P = segs[i].q_len > 0 ? prefix[i].blocks : 0;
      extra.push_back(SegExtra{P, 0, P > 0 ? prefix[i].slot : 0, P});
    }
  }
  const Geo g = make_geo(cfg, cache);
  const FwdLayout L = fwd_layout(g, segs, n_segs, n_tokens, cfg->dtype == QSA_DTYPE_BF16, lowmem, prefix != nullptr);
  if (!workspace || ws_bytes < L.total || !aligned16(workspace)) return QSA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  float* scores = (float*)(ws + L.scores);
  if (!sel) {
    sel = (int32_t*)(ws + L.sel);
    nsel = (int32_t*)(ws + L.nsel);
  }
  std::vector<qsa_segment_t> fused, plain;
  split_fused(segs, n_segs, cfg->dtype == QSA_DTYPE_BF16, lowmem, g.r, fused, plain);
  // 1. pool the blocks each segment completes
  std::vector<int32_t> slots;
  std::vector<int64_t> b0, b1;
  bool own_blocks_only = true;      // no query scores a block this step completes
  for (int i = 0; i < n_segs; ++i) {
    if (segs[i].q_len <= 0) continue;
    slots.push_back(segs[i].slot);
    b0.push_back(segs[i].pos0 / cfg->r);
    b1.push_back(((int64_t)segs[i].pos0 + segs[i].q_len) / cfg->r);
    own_blocks_only &= ((int64_t)segs[i].pos0 + segs[i].q_len - 1) / cfg->r <= segs[i].pos0 / cfg->r;
  }
  const int n_plain = (int)plain.size();
  auto compress = [&](bool late) {
    return run_compress(g, cfg, cache, slots.data(), b0.data(), b1.data(), (int)slots.size(), st, late);
  };
  // 2. indexer scores of the plain segments (with shared prefixes: each
  // sequence's own blocks, then the prefixes' blocks shared by their queries)
  const SegExtra* xp = prefix ? extra.data() : nullptr;   // plain == segs when prefixes are given
  auto index = [&]() -> qsa_status_t {
    qsa_status_t r = run_index(g, cfg, cache, plain.data(), n_plain, q_idx, w, scores, L.ld, st, xp);
    if (r != QSA_OK || !prefix) return r;
    return run_index_shared(g, cfg, cache, segs, prefix, n_segs, q_idx, w, scores, L.ld,
                            (__nv_bfloat16*)(ws + L.qrot), (float*)(ws + L.wrot), (int32_t*)(ws + L.rmap), st);
  };
  bool pooled = false;
  if (own_blocks_only) {
    // decode-like batch: no query scores a block pooled now, so the pooling
    // runs alongside the indexer (its exit still waits for the indexer)
    if (n_plain > 0) {
      if ((s = index()) != QSA_OK) return s;
      if ((s = compress(true)) != QSA_OK) return s;
      pooled = true;
    }
  } else {
    if ((s = compress(false)) != QSA_OK) return s;
    pooled = true;
    if ((s = index()) != QSA_OK) return s;
  }
  // 2-3. fused scoring and selection (alongside the filtered scoring pass, the
  // pooling of a decode-like batch that has not run yet)
  if (!fused.empty()) {
    const FusedBufs f{(float*)(ws + L.samples), L.ld_s, (float*)(ws + L.tau), (float*)(ws + L.ckey),
                      (int32_t*)(ws + L.cidx), (int32_t*)(ws + L.cnt)};
    std::function<qsa_status_t()> hook;
    if (!pooled) hook = [&]() { return compress(true); };
    s = run_fused_select(g, cfg, cache, fused.data(), (int)fused.size(), q_idx, w, f, sel, nsel, st, hook);
    if (s != QSA_OK) return s;
    pooled = true;
  }
  if (!pooled && (s = compress(true)) != QSA_OK) return s;
  // 3. selection of the plain segments, 4. attention
  if (n_plain > 0 &&
      (s = run_select(g, plain.data(), n_plain, scores, L.ld, sel, nsel, ws + L.topk, L.attn - L.topk, st)) != QSA_OK)
    return s;
  return run_attn(g, cfg, cache, segs, n_segs, n_tokens, q, sel, nsel, o, lse, ws + L.attn, L.samples - L.attn, st,
                  xp);
}
}  // namespace
}  // namespace qsa

QSA_API qsa_status_t qsa_forward(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                 const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                 const void* q, const void* q_idx, const float* w, void* o,
                                 float* lse, int32_t* sel, int32_t* nsel, void* workspace,
                                 size_t ws_bytes, void* stream) {
  return forward_impl(cfg, cache, segs, n_segs, n_tokens, q, q_idx, w, o, lse, sel, nsel, workspace, ws_bytes,
                      stream, false);
}

QSA_API qsa_status_t qsa_forward_prefixed(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                          const qsa_segment_t* segs, const qsa_prefix_t* prefix, int32_t n_segs,
                                          int32_t n_tokens, const void* q, const void* q_idx, const float* w,
                                          void* o, float* lse, int32_t* sel, int32_t* nsel, void* workspace,
                                          size_t ws_bytes, void* stream) {
  if (n_segs > 0 && !prefix) return QSA_ERR_INVALID_ARG;
  return forward_impl(cfg, cache, segs, n_segs, n_tokens, q, q_idx, w, o, lse, sel, nsel, workspace, ws_bytes,
                      stream, false, prefix);
}

QSA_API qsa_status_t qsa_forward_lowmem(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                        const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                        const void* q, const void* q_idx, const float* w, void* o,
                                        float* lse, int32_t* sel, int32_t* nsel, void* workspace,
                                        size_t ws_bytes, void* stream) {
  return forward_impl(cfg, cache, segs, n_segs, n_tokens, q, q_idx, w, o, lse, sel, nsel, workspace, ws_bytes,
                      stream, true);
}

QSA_API qsa_status_t qsa_select_fallbacks(void* stream, int64_t* count) {
  if (!count) return QSA_ERR_INVALID_ARG;
  unsigned long long h = 0, zero = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyFromSymbolAsync(&h, g_qsa_select_fallbacks, sizeof h, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_qsa_select_fallbacks, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return QSA_ERR_CUDA;
  *count = (int64_t)h;
  return QSA_OK;
}

QSA_API qsa_status_t qsa_device_status(void* stream) {
  unsigned int h = 0, zero = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyFromSymbolAsync(&h, g_qsa_device_error, sizeof h, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_qsa_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return QSA_ERR_CUDA;
  if (h == kErrWaitTimeout) return QSA_ERR_TIMEOUT;
  if (h == kErrBadIndex) return QSA_ERR_BAD_INDEX;
  if (h != kErrNone) return QSA_ERR_CUDA;
  return QSA_OK;
}

// One thread waits, with the library's bounded wait and a short limit, for an
// mbarrier phase that nothing completes: the wait gives up, records the
// timeout in the error word and returns.
__global__ void selftest_wait_kernel(long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, limit_cycles);
}

QSA_API qsa_status_t qsa_selftest_wait_timeout(void* stream) {
  count_launch();
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(200000000LL);   // ~0.1 s
  return cudaGetLastError() == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}

QSA_API const char* qsa_status_string(qsa_status_t status) {
  switch (status) {
    case QSA_OK: return "ok";
    case QSA_ERR_INVALID_ARG: return "invalid argument";
    case QSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case QSA_ERR_WORKSPACE: return "workspace missing or too small";
    case QSA_ERR_CUDA: return "CUDA error";
    case QSA_ERR_TIMEOUT: return "device-side wait timed out";
    case QSA_ERR_BAD_INDEX: return "selection entry out of range (skipped)";
  }
  return "unknown status";
}

QSA_API int32_t qsa_version(void) { return 100; }

QSA_API int64_t qsa_launch_count(void) { return (int64_t)launch_counter().load(); }

// ------------------------------------------------------------------ allocation-free selection
// Top-k selection for callers that cannot allocate device memory: the
// few-long-rows buffers (per token row a record of counters, the row
// histogram and two candidate lists) live in this file-scope device array
// instead of a caller workspace.  Every device that loads the library holds
// the array until the process exits.  All calls on a device share it, so
// calls whose work overlaps on the GPU (different streams, no ordering) race
// on it; calls on one stream are ordered and safe.  What must start at zero
// (the counters and histograms) is cleared by each call, on its stream,
// before its kernels run.
static __device__ __align__(256) unsigned char g_select_scratch[QSA_NOALLOC_SCRATCH_BYTES];

namespace qsa {
namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];

// Process-unique id of the current context (cuCtxGetId, through the
// runtime's driver entry points), or 0 if the driver cannot tell.  A device
// reset replaces the context, and with it the id.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_select_scratch on the current device.  In host code
// the array's name only stands for a host-side shadow, so the address is
// looked up once per device and context, with that device current, and
// cached; a new context on the device (after a device reset) looks it up
// again.
qsa_status_t select_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QSA_ERR_CUDA;
  // 0 until the runtime has made the device's context current on this thread:
  // then the address is looked up again, which also binds the context
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev] || ctx == 0 || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) return QSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return QSA_OK;
}
}  // namespace
}  // namespace qsa

QSA_API qsa_status_t qsa_select_topk_noalloc(const qsa_config_t* cfg, const qsa_segment_t* segs,
                                             int32_t n_segs, int32_t n_tokens, const float* scores,
                                             int64_t ld_scores, int32_t* sel, int32_t* nsel,
                                             void* stream) {
  qsa_status_t s = check_cfg(cfg);
  if (s != QSA_OK) return s;
  if ((s = check_segments(segs, n_segs, n_tokens, nullptr, 0)) != QSA_OK) return s;
  if (seg_rows(segs, n_segs) == 0) return QSA_OK;
  if (!scores || !sel || !nsel || !aligned16(sel)) return QSA_ERR_INVALID_ARG;
  const int64_t nblk = seg_max_blocks(segs, n_segs, cfg->r);
  if (ld_scores < std::max<int64_t>(1, nblk)) return QSA_ERR_INVALID_ARG;
  const Geo g = make_geo(cfg, nullptr);
  if (topk_plan(g, segs, n_segs).ws > (size_t)QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((s = select_scratch(&scratch)) != QSA_OK) return s;
  return run_select(g, segs, n_segs, scores, ld_scores, sel, nsel, scratch,
                    (size_t)QSA_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream);
}
