// topk.cuh -- per-query top-k block selection.
//
// Pages: each query keeps a budget of 2048 tokens (design report QSA item,
// K=2048; ms-swift best-practice page, model structure: budget 2048 tokens),
// i.e. S = 512 micro-blocks of r = 4.  Readings: the query's own block is
// always kept; the other S-1 are the best candidates b < floor(t/r) under
// the total order (score descending, block index ascending), -0 == +0.
//
// Algorithm (one CTA per row, or per row chunk for long rows; the row is
// streamed from global memory, so several CTAs fit on an SM).  Elements are
// ranked by the 64-bit composite (key << 32) | ~index, which orders them by
// score and then by lower block index, so every composite is distinct:
//   1. radix narrowing over the row: histograms of the next 11/11/10 key bits
//      over the elements still in the threshold bucket (warp-aggregated
//      shared atomics) locate the bucket holding the K-th largest element,
//      until that bucket fits a 4096-entry shared buffer;
//   2. gather: elements above the bucket are kept outright, the bucket's
//      elements are copied to the buffer as composites;
//   3. narrowing continues on the composites in shared memory (remaining key
//      bits, then index bits) until the bucket holds exactly the elements
//      still needed; every buffered composite at or above it is kept;
//   4. the kept block indices are sorted ascending (bitonic, 512 entries).
// If a bucket is still larger than the buffer after all 32 key bits (many
// exactly equal keys), the tied elements are taken in index order by an
// ordered ballot compaction instead.  Long rows are split into chunks whose
// local top K (exact under the same order) are merged by a second pass of
// the same routine over the chunk candidates.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {
namespace topk {
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int NBINS = 2048;
constexpr int CAP = 4096;                  // candidate buffer (composite keys)
constexpr int KMAX = kMaxBudgetBlocks;     // kept entries per row (S-1 <= 511)
constexpr int kChunkLarge = 1 << 30;       // no split
constexpr int kChunkSmall = 8192;
}

struct TopkShared {
  uint32_t hist[topk::NBINS];
  unsigned long long cand[topk::CAP];      // composites (key << 32) | ~index
  uint32_t kept[topk::KMAX];               // indices kept outright / final list
  int warp_a[topk::WARPS];
  int warp_b[topk::WARPS];
  int n_kept, n_cand;
  uint32_t sel_digit;
  int sel_above, sel_count;
};

// Source of one selection: element i has key(i) and index idx(i).
struct RowSrc {
  const float* scores;          // score row (keys from scores), or null
  const uint32_t* keys;         // candidate keys (merge), or null
  const int32_t* idx;           // candidate indices (merge)
  int64_t base;                 // index of element 0 (score rows)
  __device__ __forceinline__ uint32_t key(int i) const {
    return scores ? score_key(scores[i]) : keys[i];
  }
  __device__ __forceinline__ uint32_t index(int i) const {
    return scores ? (uint32_t)(base + i) : (uint32_t)idx[i];
  }
};

// Histogram of digit (key >> shift) & dmask over elements with (key & mask) == prefix.
__device__ void topk_hist(const RowSrc& src, int n, uint32_t prefix, uint32_t mask, int shift, uint32_t dmask,
                          TopkShared& sh) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < NBINS; i += THREADS) sh.hist[i] = 0;
  __syncthreads();
  for (int b = warp * 32; b < n; b += THREADS) {
    const int i = b + lane;
    const uint32_t key = i < n ? src.key(i) : 0u;
    const bool valid = i < n && (key & mask) == prefix;
    const uint32_t digit = (key >> shift) & dmask;
    const uint32_t peers = __match_any_sync(0xffffffffu, valid ? digit : 0xffffffffu);
    if (valid && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[digit], (uint32_t)__popc(peers));
  }
  __syncthreads();
}

// Finds the digit whose bucket holds the k_rem-th largest element: sets
// sh.sel_digit, sh.sel_above (count in higher buckets), sh.sel_count.
__device__ void topk_locate(int k_rem, TopkShared& sh) {
  using namespace topk;
  constexpr int PER = NBINS / THREADS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) local += sh.hist[threadIdx.x * PER + j];
  int suf = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  if (lane == 0) sh.warp_a[warp] = suf;
  __syncthreads();
  int above_warps = 0;
  for (int w = warp + 1; w < WARPS; ++w) above_warps += sh.warp_a[w];
  const int incl = suf + above_warps, excl = incl - local;
  if (excl < k_rem && k_rem <= incl) {
    int above = excl;
    for (int j = PER - 1; j >= 0; --j) {
      const int b = threadIdx.x * PER + j;
      const int c = (int)sh.hist[b];
      if (above + c >= k_rem) {
        sh.sel_digit = (uint32_t)b;
        sh.sel_above = above;
        sh.sel_count = c;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// Bitonic sort of a[0..n) (n a power of two), descending or ascending.
template <typename T>
__device__ void bitonic(T* a, int n, bool descending) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = ((i & k) == 0) != descending;
          const T x = a[i], y = a[p];
          if ((x > y) == up) {
            a[i] = y;
            a[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Finishes a selection whose candidates sh.cand[0..nc) are the composites of
// every element in the current bucket (key & mask == prefix) and k_rem of
// them are still needed: narrows on the remaining key bits, then on the
// index bits, until the bucket holds exactly the elements still needed, and
// appends every candidate at or above it to sh.kept.
__device__ void refine_and_keep(int nc, int k_rem, uint32_t prefix, uint32_t mask, TopkShared& sh) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long cprefix = (unsigned long long)prefix << 32, cmask = (unsigned long long)mask << 32;
  const int cshifts[6] = {53, 42, 32, 21, 10, 0};
  const int cwidths[6] = {11, 11, 10, 11, 11, 10};
  int q0 = 0;                               // first composite digit not yet resolved
  while (q0 < 3 && ((cmask >> cshifts[q0]) & 1ull)) ++q0;
  int count = nc;
  for (int q = q0; q < 6 && count != k_rem; ++q) {
    const unsigned long long dm = (1ull << cwidths[q]) - 1ull;
    for (int i = threadIdx.x; i < NBINS; i += THREADS) sh.hist[i] = 0;
    __syncthreads();
    for (int b = warp * 32; b < nc; b += THREADS) {
      const int i = b + lane;
      const unsigned long long c = i < nc ? sh.cand[i] : 0ull;
      const bool valid = i < nc && (c & cmask) == cprefix;
      const uint32_t digit = (uint32_t)((c >> cshifts[q]) & dm);
      const uint32_t peers = __match_any_sync(0xffffffffu, valid ? digit : 0xffffffffu);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[digit], (uint32_t)__popc(peers));
    }
    __syncthreads();
    topk_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    cprefix |= (unsigned long long)sh.sel_digit << cshifts[q];
    cmask |= dm << cshifts[q];
    count = sh.sel_count;
    __syncthreads();
  }
  for (int i = threadIdx.x; i < nc; i += THREADS) {
    const unsigned long long c = sh.cand[i];
    if ((c & cmask) >= cprefix) sh.kept[atomicAdd(&sh.n_kept, 1)] = 0xffffffffu - (uint32_t)(c & 0xffffffffull);
  }
  __syncthreads();
}

// Fast path for rows longer than the candidate buffer: a strided sample of
// the keys gives a threshold expected to admit about kSampleTarget elements;
// one pass collects every element at or above it.  If between K and CAP
// elements qualify, the K best are among them (at least K elements are at or
// above the threshold, so the K-th largest is too) and are found exactly on
// the buffered composites; otherwise returns false and nothing is kept.
constexpr int kSamples = 2048;
constexpr int kSampleTarget = 2048;

__device__ bool select_by_sample(const RowSrc& src, int n, int K, TopkShared& sh) {
  using namespace topk;
  uint32_t* samp = reinterpret_cast<uint32_t*>(sh.cand);      // reused before the candidates land
  const int m = min(kSamples, n / 4);
  for (int s = threadIdx.x; s < m; s += THREADS) samp[s] = src.key((int)((int64_t)s * n / m));
  __syncthreads();
  const int target = max(4 * K, kSampleTarget);
  const int rank = max(1, (int)((int64_t)m * target / n));
  // exact rank-th largest sample key
  const RowSrc ssrc{nullptr, samp, nullptr, 0};
  uint32_t prefix = 0, mask = 0;
  int k_rem = rank;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3; ++p) {
    const uint32_t dmask = (1u << widths[p]) - 1u;
    topk_hist(ssrc, m, prefix, mask, shifts[p], dmask, sh);
    topk_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    prefix |= sh.sel_digit << shifts[p];
    mask |= dmask << shifts[p];
    __syncthreads();
  }
  const uint32_t tau = prefix;
  if (threadIdx.x == 0) {
    sh.n_kept = 0;
    sh.n_cand = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += THREADS) {
    const uint32_t key = src.key(i);
    if (key >= tau) {
      const int slot = atomicAdd(&sh.n_cand, 1);
      if (slot < CAP) sh.cand[slot] = ((unsigned long long)key << 32) | (0xffffffffu - src.index(i));
    }
  }
  __syncthreads();
  const int nc = sh.n_cand;
  if (nc < K || nc > CAP) {
    __syncthreads();
    return false;
  }
  refine_and_keep(nc, K, 0u, 0u, sh);
  return true;
}

// Selects the K best elements of src[0..n) (K <= n) under (key desc, index
// asc).  On return sh.kept[0..K) holds their indices, in no particular order.
__device__ void topk_select(const RowSrc& src, int n, int K, TopkShared& sh) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (n > CAP && select_by_sample(src, n, K, sh)) return;
  uint32_t prefix = 0, mask = 0;
  int k_rem = K;
  int bucket = n;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3 && bucket > CAP; ++p) {
    const uint32_t dmask = (1u << widths[p]) - 1u;
    topk_hist(src, n, prefix, mask, shifts[p], dmask, sh);
    topk_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    prefix |= sh.sel_digit << shifts[p];
    mask |= dmask << shifts[p];
    bucket = sh.sel_count;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    sh.n_kept = 0;
    sh.n_cand = 0;
  }
  __syncthreads();
  if (bucket <= CAP) {
    // gather: above the bucket -> kept; in the bucket -> composite candidates
    for (int i = threadIdx.x; i < n; i += THREADS) {
      const uint32_t key = src.key(i);
      const uint32_t mk = key & mask;
      if (mk > prefix) {
        sh.kept[atomicAdd(&sh.n_kept, 1)] = src.index(i);
      } else if (mk == prefix) {
        sh.cand[atomicAdd(&sh.n_cand, 1)] = ((unsigned long long)key << 32) | (0xffffffffu - src.index(i));
      }
    }
    __syncthreads();
    refine_and_keep(sh.n_cand, k_rem, prefix, mask, sh);
  } else {
    // every element of the bucket has the same key: keep the k_rem lowest
    // indices among them, in index order, plus everything above the bucket.
    // Element order is index order for both sources.
    const int per = (int)cdiv(cdiv(n, WARPS), 32) * 32;
    const int beg = warp * per, end = min(n, beg + per);
    int n_gt = 0, n_tie = 0;
    for (int b = beg; b < end; b += 32) {
      const int i = b + lane;
      const uint32_t mk = i < end ? (src.key(i) & mask) : 0u;
      n_gt += __popc(__ballot_sync(0xffffffffu, i < end && mk > prefix));
      n_tie += __popc(__ballot_sync(0xffffffffu, i < end && mk == prefix));
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
    const uint32_t lt = (1u << lane) - 1u;
    for (int b = beg; b < end; b += 32) {
      const int i = b + lane;
      const uint32_t mk = i < end ? (src.key(i) & mask) : 0u;
      const bool gt = i < end && mk > prefix, tie = i < end && mk == prefix;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt), bt = __ballot_sync(0xffffffffu, tie);
      const int gb = gt_run + __popc(bg & lt), tb = tie_run + __popc(bt & lt);
      if (gt) sh.kept[gb + min(tb, k_rem)] = src.index(i);
      else if (tie && tb < k_rem) sh.kept[gb + tb] = src.index(i);
      gt_run += __popc(bg);
      tie_run += __popc(bt);
    }
    __syncthreads();
  }
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

// Sorts sh.kept[0..K) ascending and writes the final row: kept blocks, the
// own block, -1 padding.
__device__ void topk_write_final(TopkShared& sh, int K, int S, int64_t bt, int32_t* sel_row) {
  constexpr int P = topk::KMAX;
  for (int i = K + threadIdx.x; i < P; i += blockDim.x) sh.kept[i] = 0xffffffffu;
  __syncthreads();
  bitonic(sh.kept, P, false);
  for (int i = threadIdx.x; i < S; i += blockDim.x)
    sel_row[i] = i < K ? (int32_t)sh.kept[i] : (i == K ? (int32_t)bt : -1);
}

__global__ void __launch_bounds__(topk::THREADS) topk_chunk_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  __shared__ TopkShared sh;
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
  const RowSrc src{a.scores + tok * a.ld + c0, nullptr, nullptr, c0};
  const int kk = min(n, K);
  if (n <= K) {
    for (int i = threadIdx.x; i < n; i += THREADS) sh.kept[i] = (uint32_t)(c0 + i);
    __syncthreads();
  } else {
    topk_select(src, n, K, sh);
  }
  if (n_ch_row == 1) {
    topk_write_final(sh, K, S, bt, sel_row);
    if (threadIdx.x == 0) a.nsel[tok] = S;
  } else {
    const int64_t base = (tok * a.max_ch + c) * (int64_t)K;
    for (int i = threadIdx.x; i < kk; i += THREADS) {
      const uint32_t idx = sh.kept[i];
      a.cand_idx[base + i] = (int32_t)idx;
      a.cand_key[base + i] = score_key(a.scores[tok * a.ld + idx]);
    }
    if (threadIdx.x == 0) a.cand_cnt[tok * a.max_ch + c] = kk;
  }
}

// Merge of split rows.  Every chunk but a row's last holds at least
// kChunkSmall > S-1 elements and so stores exactly S-1 candidates; the
// chunk lists therefore lie back to back, in chunk (= index) order.
__global__ void __launch_bounds__(topk::THREADS) topk_merge_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  __shared__ TopkShared sh;
  const int S = g.S, K = S - 1;
  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int j = item - st.item0[si];
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = st.pos0[si] + j;
  const int64_t bt = t / g.r;
  if (bt + 1 <= S) return;
  const int n_ch_row = (int)cdiv(bt, a.chunk);
  if (n_ch_row <= 1) return;
  const int n = (n_ch_row - 1) * K + a.cand_cnt[tok * a.max_ch + n_ch_row - 1];
  const int64_t row_base = tok * a.max_ch * (int64_t)K;
  const RowSrc src{nullptr, a.cand_key + row_base, a.cand_idx + row_base, 0};
  topk_select(src, n, K, sh);
  topk_write_final(sh, K, S, bt, a.sel + tok * S);
  if (threadIdx.x == 0) a.nsel[tok] = S;
}

inline size_t topk_chunk_smem(int) { return 0; }
inline size_t topk_merge_smem(int, int) { return 0; }

}  // namespace qsa
