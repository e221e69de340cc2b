// topk.cuh -- per-query top-k block selection.
//
// Pages: each query keeps a budget of 2048 tokens (design report QSA item,
// K=2048; ms-swift best-practice page, model structure: budget 2048 tokens),
// i.e. S = 512 micro-blocks of r = 4.  Readings: the query's own block is
// always kept; the other S-1 are the best candidates b < floor(t/r) under
// the total order (score descending, block index ascending), -0 == +0.
//
// Algorithm: scores are mapped to order-preserving uint32 keys and held in
// shared memory; a 3-pass MSB radix select (11/11/10-bit digits, warp-
// aggregated shared-memory histograms) finds the threshold key and how many
// keys equal to it are taken; an index-ordered ballot compaction then emits
// the kept blocks already sorted ascending, taking tied keys lowest index
// first.  Rows longer than one chunk are split: every chunk keeps its own
// top S-1 (exact under the same total order, so the union contains the
// answer), and a merge pass selects from the union.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {
namespace topk {
constexpr int THREADS = 512;
constexpr int WARPS = THREADS / 32;
constexpr int NBINS = 2048;
constexpr int kChunkLarge = 32768;
constexpr int kChunkSmall = 8192;
}

struct RadixState {
  uint32_t prefix;
  uint32_t mask;
  int k_rem;
};

struct TopkShared {
  uint32_t hist[topk::NBINS];
  int warp_a[topk::WARPS];
  int warp_b[topk::WARPS];
  uint32_t sel_digit;
  int sel_above;
  int sel_count;
};

// Finds the K-th largest key among keys[0..n) (K <= n): on return, a key x
// is kept iff (x & mask) > prefix, or (x & mask) == prefix and it is among
// the first k_rem such keys in index order.
__device__ RadixState radix_select(const uint32_t* keys, int n, int K, TopkShared& sh) {
  using namespace topk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  RadixState rs{0u, 0u, K};
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p];
    const uint32_t dmask = (1u << widths[p]) - 1u;
    for (int i = tid; i < NBINS; i += THREADS) sh.hist[i] = 0;
    __syncthreads();
    for (int base = warp * 32; base < n; base += THREADS) {
      const int i = base + lane;
      uint32_t key = i < n ? keys[i] : 0u;
      const bool valid = i < n && (key & rs.mask) == rs.prefix;
      const uint32_t digit = (key >> shift) & dmask;
      const uint32_t tag = valid ? digit : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, tag);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[digit], (uint32_t)__popc(peers));
    }
    __syncthreads();
    // locate the digit where the count of larger-or-equal keys reaches k_rem
    constexpr int PER = NBINS / THREADS;
    int local = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) local += sh.hist[tid * PER + j];
    int suf = local;   // inclusive suffix sum within the warp (lanes >= this lane)
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int v = __shfl_down_sync(0xffffffffu, suf, off);
      if (lane + off < 32) suf += v;
    }
    if (lane == 0) sh.warp_a[warp] = suf;
    __syncthreads();
    int above_warps = 0;
    for (int w = warp + 1; w < WARPS; ++w) above_warps += sh.warp_a[w];
    const int incl = suf + above_warps;          // keys with digit >= tid*PER
    const int excl = incl - local;               // keys with digit >= (tid+1)*PER
    if (excl < rs.k_rem && rs.k_rem <= incl) {
      int above = excl;
      for (int j = PER - 1; j >= 0; --j) {
        const int b = tid * PER + j;
        const int c = (int)sh.hist[b];
        if (above + c >= rs.k_rem) {
          sh.sel_digit = (uint32_t)b;
          sh.sel_above = above;
          sh.sel_count = c;
          break;
        }
        above += c;
      }
    }
    __syncthreads();
    rs.k_rem -= sh.sel_above;
    rs.prefix |= sh.sel_digit << shift;
    rs.mask |= dmask << shift;
    const int cnt = sh.sel_count;
    __syncthreads();
    if (cnt == rs.k_rem) break;                  // the whole bucket is kept
  }
  return rs;
}

// Emits the kept elements of keys[0..n) in index order.  emit(pos, i) is
// called once per kept element with its output position.  keep_all keeps
// every element.
template <typename Emit>
__device__ void compact_in_order(const uint32_t* keys, int n, const RadixState& rs, bool keep_all,
                                 TopkShared& sh, Emit emit) {
  using namespace topk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (int)cdiv(cdiv(n, WARPS), 32) * 32;
  const int beg = warp * per, end = min(n, beg + per);
  int n_gt = 0, n_tie = 0;
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < end ? keys[i] : 0u;
    const uint32_t mk = key & rs.mask;
    const bool gt = i < end && (keep_all || mk > rs.prefix);
    const bool tie = i < end && !keep_all && mk == rs.prefix;
    n_gt += __popc(__ballot_sync(0xffffffffu, gt));
    n_tie += __popc(__ballot_sync(0xffffffffu, tie));
  }
  if (lane == 0) {
    sh.warp_a[warp] = n_gt;
    sh.warp_b[warp] = n_tie;
  }
  __syncthreads();
  int gt_run = 0, tie_run = 0;
  for (int w = 0; w < warp; ++w) {
    gt_run += sh.warp_a[w];
    tie_run += sh.warp_b[w];
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < end ? keys[i] : 0u;
    const uint32_t mk = key & rs.mask;
    const bool gt = i < end && (keep_all || mk > rs.prefix);
    const bool tie = i < end && !keep_all && mk == rs.prefix;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t bt = __ballot_sync(0xffffffffu, tie);
    const int gt_before = gt_run + __popc(bg & lt_mask);
    const int tie_before = tie_run + __popc(bt & lt_mask);
    if (gt) emit(gt_before + min(tie_before, rs.k_rem), i);
    else if (tie && tie_before < rs.k_rem) emit(gt_before + tie_before, i);
    gt_run += __popc(bg);
    tie_run += __popc(bt);
  }
  __syncthreads();
}

struct TopkArgs {
  const float* scores;
  int64_t ld;
  int32_t* sel;
  int32_t* nsel;
  uint32_t* cand_key;   // [T][max_ch][S-1]   (split rows only)
  int32_t* cand_idx;    // [T][max_ch][S-1]
  int32_t* cand_cnt;    // [T][max_ch]
  int chunk;            // candidates per chunk
  int max_ch;           // chunks per row in the workspace layout
};

// Writes the final selection of a row: kept[0..K) ascending, then the own block.
__device__ __forceinline__ void write_tail(int32_t* sel_row, int K, int S, int64_t bt) {
  for (int i = K + threadIdx.x; i < S; i += blockDim.x) sel_row[i] = (i == K) ? (int32_t)bt : -1;
}

__global__ void __launch_bounds__(topk::THREADS) topk_chunk_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));

  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int local = item - st.item0[si];
  const int64_t pos0 = st.pos0[si];
  const int q_len = st.q_len[si];
  const int64_t nb_seg = cdiv((pos0 + q_len - 1) / g.r, a.chunk);
  const int n_ch_seg = (int)(nb_seg > 1 ? nb_seg : 1);
  const int j = local / n_ch_seg, c = local - j * n_ch_seg;
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = pos0 + j;
  const int64_t bt = t / g.r;
  const int S = g.S, K = S - 1;
  int32_t* sel_row = a.sel + tok * S;

  if (bt + 1 <= S) {                           // every block in reach is kept
    if (c != 0) return;
    for (int i = threadIdx.x; i < S; i += blockDim.x) sel_row[i] = (i <= bt) ? i : -1;
    if (threadIdx.x == 0) a.nsel[tok] = (int32_t)(bt + 1);
    return;
  }
  const int n_ch_row = (int)cdiv(bt, a.chunk);
  if (c >= n_ch_row) return;
  const int64_t c0 = (int64_t)c * a.chunk;
  const int n = (int)((bt - c0) < a.chunk ? (bt - c0) : a.chunk);
  const float* row = a.scores + tok * a.ld + c0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = score_key(row[i]);
  __syncthreads();
  const bool keep_all = n <= K;
  RadixState rs{0u, 0u, 0};
  if (!keep_all) rs = radix_select(keys, n, K, sh);
  if (n_ch_row == 1) {
    compact_in_order(keys, n, rs, keep_all, sh, [&](int p, int i) { sel_row[p] = (int32_t)(c0 + i); });
    write_tail(sel_row, K, S, bt);
    if (threadIdx.x == 0) a.nsel[tok] = S;
  } else {
    const int64_t base = (tok * a.max_ch + c) * (int64_t)K;
    compact_in_order(keys, n, rs, keep_all, sh, [&](int p, int i) {
      a.cand_key[base + p] = keys[i];
      a.cand_idx[base + p] = (int32_t)(c0 + i);
    });
    if (threadIdx.x == 0) a.cand_cnt[tok * a.max_ch + c] = min(n, K);
  }
}

__global__ void __launch_bounds__(topk::THREADS) topk_merge_kernel(Geo g, SegTable st, TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  const int S = g.S, K = S - 1;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));
  int32_t* idx = reinterpret_cast<int32_t*>(keys + (size_t)a.max_ch * K);
  __shared__ int offs[64 + 1];

  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int j = item - st.item0[si];
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = st.pos0[si] + j;
  const int64_t bt = t / g.r;
  if (bt + 1 <= S) return;
  const int n_ch_row = (int)cdiv(bt, a.chunk);
  if (n_ch_row <= 1) return;
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int c = 0; c < n_ch_row; ++c) {
      offs[c] = acc;
      acc += a.cand_cnt[tok * a.max_ch + c];
    }
    offs[n_ch_row] = acc;
  }
  __syncthreads();
  const int n = offs[n_ch_row];
  for (int c = 0; c < n_ch_row; ++c) {
    const int64_t base = (tok * a.max_ch + c) * (int64_t)K;
    const int cnt = offs[c + 1] - offs[c];
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
      keys[offs[c] + i] = a.cand_key[base + i];
      idx[offs[c] + i] = a.cand_idx[base + i];
    }
  }
  __syncthreads();
  int32_t* sel_row = a.sel + tok * S;
  const RadixState rs = radix_select(keys, n, K, sh);
  compact_in_order(keys, n, rs, false, sh, [&](int p, int i) { sel_row[p] = idx[i]; });
  write_tail(sel_row, K, S, bt);
  if (threadIdx.x == 0) a.nsel[tok] = S;
}

inline size_t topk_chunk_smem(int chunk) { return sizeof(TopkShared) + sizeof(uint32_t) * (size_t)chunk; }
inline size_t topk_merge_smem(int max_ch, int K) {
  return sizeof(TopkShared) + (sizeof(uint32_t) + sizeof(int32_t)) * (size_t)max_ch * K;
}

}  // namespace qsa
