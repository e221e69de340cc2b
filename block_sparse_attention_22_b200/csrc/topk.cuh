// topk.cuh -- per-query top-k block selection.
//
// Pages: each query keeps a budget of 2048 tokens (design report QSA item,
// K=2048; ms-swift best-practice page, model structure: budget 2048 tokens),
// i.e. S = 512 micro-blocks of r = 4.  Readings: the query's own block is
// always kept; the other S-1 are the best candidates b < floor(t/r) under
// the total order (score descending, block index ascending), -0 == +0.
//
// Many rows: one warp per row (topk_rows_kernel, below), with the rows it
// leaves selected by a 4-warp CTA each (~35 KB of shared memory, six CTAs per
// SM); 32 warps per row when rows are few and at most 32K blocks long; for
// few longer rows, 4096-score chunks sharing an exact histogram of the row
// (topk_hist_kernel, topk_hfilter_kernel, topk_hfinal_kernel).  The
// CTA-level selection of one row (topk_select) runs as follows.  Scores are compared as 32-bit keys
// whose unsigned order is the float order.  For a row of n candidates and
// K = S-1:
//   1. threshold: m = n/16 keys (1024 .. 8192, in runs of 8 neighbours spread
//      evenly over the row) are reduced by a radix select to the 16-bit
//      bucket of their rank-th largest, rank chosen so that about
//      kSampleTarget elements of the row are expected at or above the
//      bucket's lower edge (rows of at most CAP elements take every element);
//   2. filter: one pass over the row (16-byte loads, several per thread in
//      flight); each thread appends the elements at or above the threshold to
//      its own slots, spilling to shared overflow slots, with no coordination;
//   3. if between K and CAP elements were collected, the K-th largest of the
//      row is among them: a radix select over the candidates (8-bit digits,
//      starting below the bits all candidates share) finds its key T and how
//      many elements equal to T are needed; if fewer than all of the tied ones
//      are needed, a second radix select over the tied elements' indices keeps
//      the lowest ones;
//   4. the kept block indices are put in ascending order through a bitmap of
//      the row (set bits, then each thread emits the set bits of its words at
//      its prefix-count offset).
// If the sampled threshold admits fewer than K or more than CAP elements, an
// exact fallback runs: a radix select streamed over the whole row (four
// passes), then one ordered pass that keeps everything above T and the
// lowest-indexed elements equal to T.
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"

namespace qsa {
namespace topk {
constexpr int THREADS = 128;               // CTA of the per-row kernel (six CTAs per SM)
constexpr int kWideThreads = 1024;         // CTA of the kernel for few long rows (one row per SM)
constexpr int NBINS = 256;                 // one 8-bit digit per radix pass
constexpr int OVF = 1024;                  // shared overflow slots
constexpr int CAP = 4096;                  // candidates a row may collect (thread slots + overflow)
constexpr int KMAX = kMaxBudgetBlocks;     // kept entries per row (S-1 <= 511)
constexpr int kBufWords = 2 * CAP;         // candidate buffer, reused for the sample and the bitmap
constexpr int kMinSamples = 1024;
constexpr int kMaxSamples = kBufWords;
constexpr int kSampleGroup = 8;            // samples are runs of 8 neighbours (one 32-byte sector)
constexpr int kSampleTarget = 1536;        // expected elements at or above the sampled threshold
constexpr int kWideMaxBlocks = 32768;      // few rows up to this long: one wide CTA per row
constexpr int kWideStages = 8;             // cp.async slots per thread of the wide CTA
constexpr int kWideRingBytes = kWideStages * kWideThreads * 16;
constexpr int kFusedStride = 16;          // fused prefill selection: one sampled block in 16
// few long rows: an exact histogram of the top key bits, then a filter
constexpr int kHistBits = 12;              // sign, 8 exponent and 3 mantissa bits of the score
constexpr int kHistBins = 1 << kHistBits;
constexpr int kHistShift = 32 - kHistBits;
constexpr int kCoarseBins = 256;           // the top 8 key bits: 16 fine bins each
constexpr int kHistChunk = 4096;           // scores per CTA
constexpr int kHistThreads = 256;
constexpr int kHistPer = kHistChunk / (4 * kHistThreads);   // 16-byte groups per thread
}

// Per-CTA-size constants: each thread owns CAPL candidate slots.
template <int NT>
struct TopkCfg {
  static constexpr int THREADS = NT;
  static constexpr int WARPS = NT / 32;
  static constexpr int CAPL = (topk::CAP - topk::OVF) / NT;   // 24 at 128 threads, 3 at 1024
  static constexpr int U = NT >= 512 ? 4 : 8;                 // 16-byte loads in flight per thread
};

template <int NT>
struct alignas(16) TopkShared {
  uint32_t hist[topk::NBINS];
  uint32_t cbuf[topk::kBufWords];          // candidates | sample | bitmap
  uint32_t kept[topk::KMAX];               // kept indices / final sorted list
  int warp_a[NT / 32];
  int warp_b[NT / 32];
  uint32_t warp_c[NT / 32];
  int n_kept, n_ovf;
  uint32_t sel_digit;
  int sel_above, sel_count;
  // candidate slot s of thread t: lkey[s * NT + t]; overflow slot o: okey[o]
  static constexpr int kSlots = TopkCfg<NT>::CAPL * NT;
  __device__ __forceinline__ uint32_t* lkey() { return cbuf; }
  __device__ __forceinline__ uint32_t* lidx() { return cbuf + kSlots; }
  __device__ __forceinline__ uint32_t* okey() { return cbuf + 2 * kSlots; }
  __device__ __forceinline__ uint32_t* oidx() { return cbuf + 2 * kSlots + topk::OVF; }
};

// Source of one selection: element i has key(i) and index index(i); element
// order is index order.
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

// Float whose key is k (inverse of score_key on keys of finite floats); keys
// below that of -inf map to -inf.
__device__ __forceinline__ float key_to_float(uint32_t k) {
  if (k & 0x80000000u) return __uint_as_float(k & 0x7fffffffu);
  if (k < 0x007fffffu) return -__int_as_float(0x7f800000);
  return __uint_as_float(~k);
}

// ---------------------------------------------------------------- block reductions
template <int NT>
__device__ __forceinline__ int block_sum(int v, TopkShared<NT>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  if (lane == 0) sh.warp_b[warp] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int w = 0; w < TopkCfg<NT>::WARPS; ++w) t += sh.warp_b[w];
  __syncthreads();
  return t;
}

// Exclusive prefix sum of v over the block (thread order); *total = sum.
template <int NT>
__device__ __forceinline__ int block_exscan(int v, int* total, TopkShared<NT>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) sh.warp_b[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < TopkCfg<NT>::WARPS; ++w) {
    if (w < warp) before += sh.warp_b[w];
    all += sh.warp_b[w];
  }
  __syncthreads();
  *total = all;
  return before + incl - v;
}

template <int NT>
__device__ __forceinline__ void block_minmax(uint32_t& lo, uint32_t& hi, TopkShared<NT>& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  if (lane == 0) {
    sh.warp_c[warp] = lo;
    sh.warp_a[warp] = (int)hi;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < TopkCfg<NT>::WARPS; ++w) {
    lo = min(lo, sh.warp_c[w]);
    hi = max(hi, (uint32_t)sh.warp_a[w]);
  }
  __syncthreads();
}

// ---------------------------------------------------------------- radix helpers
template <int NT>
__device__ __forceinline__ void hist_clear(TopkShared<NT>& sh) {
  for (int i = threadIdx.x; i < topk::NBINS; i += NT) sh.hist[i] = 0;
}

// Adds element (key, valid) to the histogram of digit (key >> shift) & 255.
// The top digit of keys of similar magnitude is shared by most of a warp, so
// that pass aggregates equal digits into one shared atomic.
template <int NT>
__device__ __forceinline__ void hist_add(uint32_t key, bool valid, int shift, bool aggregate, TopkShared<NT>& sh) {
  const int lane = threadIdx.x & 31;
  const uint32_t digit = (key >> shift) & 255u;
  if (aggregate) {
    const uint32_t peers = __match_any_sync(0xffffffffu, valid ? digit : 0xffffffffu);
    if (valid && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[digit], (uint32_t)__popc(peers));
  } else if (valid) {
    atomicAdd(&sh.hist[digit], 1u);
  }
}

// Finds the digit whose bucket holds the k_rem-th largest element: sets
// sh.sel_digit, sh.sel_above (count in higher buckets), sh.sel_count.
// Ends with a barrier.
template <int NT>
__device__ void hist_locate(int k_rem, TopkShared<NT>& sh) {
  using namespace topk;
  constexpr int PER = NBINS >= NT ? NBINS / NT : 1;   // bins per thread
  constexpr int ACT = NBINS / PER;                    // threads holding bins
  constexpr int AW = (ACT + 31) / 32;                 // warps holding bins
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool act = (int)threadIdx.x < ACT;
  int local = 0;
  if (act) {
#pragma unroll
    for (int j = 0; j < PER; ++j) local += sh.hist[threadIdx.x * PER + j];
  }
  int suf = local;                       // sum over this and higher threads of the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  if (lane == 0 && warp < AW) sh.warp_a[warp] = suf;
  __syncthreads();
  if (act) {
    int above_warps = 0;
    for (int w = warp + 1; w < AW; ++w) above_warps += sh.warp_a[w];
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
  }
  __syncthreads();
}

// Radix select of the k-th largest value among the n values produced by
// val(i) that satisfy ok(i): 8-bit passes from the top down to bit
// last_shift.  Returns the value with the bits below last_shift cleared;
// *above = how many values are larger in the resolved bits, *equal = how
// many share them (with last_shift = 0: strictly larger, and equal).
template <int NT, class Val, class Ok>
__device__ uint32_t radix_select(int n, int k, Val val, Ok ok, int* above, int* equal, TopkShared<NT>& sh,
                                 int last_shift = 0) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t prefix = 0, mask = 0;
  int k_rem = k, n_above = 0, count = 0;
  for (int shift = 24; shift >= last_shift; shift -= 8) {
    hist_clear(sh);
    __syncthreads();
    for (int b = warp * 32; b < n; b += NT) {
      const int i = b + lane;
      const bool in = i < n && ok(i);
      const uint32_t v = in ? val(i) : 0u;
      hist_add(v, in && (v & mask) == prefix, shift, shift == 24, sh);
    }
    __syncthreads();
    hist_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    n_above += sh.sel_above;
    prefix |= sh.sel_digit << shift;
    mask |= 255u << shift;
    count = sh.sel_count;
    __syncthreads();
  }
  *above = n_above;
  *equal = count;
  return prefix;
}

// Appends idx to sh.kept when `take` (warp-aggregated; every lane calls it).
template <int NT>
__device__ __forceinline__ void keep_if(bool take, uint32_t idx, TopkShared<NT>& sh) {
  const int lane = threadIdx.x & 31;
  const uint32_t m = __ballot_sync(0xffffffffu, take);
  if (m == 0) return;
  int base = 0;
  if (lane == 0) base = atomicAdd(&sh.n_kept, __popc(m));
  base = __shfl_sync(0xffffffffu, base, 0);
  const int pos = base + __popc(m & ((1u << lane) - 1u));
  if (take && pos < topk::KMAX) sh.kept[pos] = idx;
}

// ---------------------------------------------------------------- candidates
// Each thread appends the candidates it finds to its own slots (no
// coordination); past CAPL they go to the shared overflow slots.  `cnt`
// counts every candidate of the thread.
template <int NT>
__device__ __forceinline__ void cand_append(uint32_t key, uint32_t idx, int& cnt, TopkShared<NT>& sh) {
  using namespace topk;
  if (cnt < TopkCfg<NT>::CAPL) {
    sh.lkey()[cnt * NT + threadIdx.x] = key;
    sh.lidx()[cnt * NT + threadIdx.x] = idx;
  } else {
    const int o = atomicAdd(&sh.n_ovf, 1);
    if (o < OVF) {
      sh.okey()[o] = key;
      sh.oidx()[o] = idx;
    }
  }
  ++cnt;
}

// Calls f(key, idx, valid) for this thread's candidates in a loop whose trip
// count is uniform across the warp (own slots, then a strided share of the
// overflow slots).
template <int NT, class F>
__device__ __forceinline__ void cand_for_each(int cnt, TopkShared<NT>& sh, F f) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int mine = min(cnt, TopkCfg<NT>::CAPL);
  const int wmax = __reduce_max_sync(0xffffffffu, mine);
  for (int s = 0; s < wmax; ++s) {
    const bool v = s < mine;
    f(v ? sh.lkey()[s * NT + threadIdx.x] : 0u, v ? sh.lidx()[s * NT + threadIdx.x] : 0u, v);
  }
  const int no = min(sh.n_ovf, OVF);
  for (int b = warp * 32; b < no; b += NT) {
    const int o = b + lane;
    const bool v = o < no;
    f(v ? sh.okey()[o] : 0u, v ? sh.oidx()[o] : 0u, v);
  }
}

// Radix select of the k-th largest of val(key, idx) over the candidates
// with ok(key, idx).  The passes start below the common high bits of the
// smallest and largest participating value.  Returns the value; *above =
// how many are larger, *equal = how many equal it.
template <int NT, class Val, class Ok>
__device__ uint32_t cand_radix(int cnt, int k, Val val, Ok ok, int* above, int* equal, TopkShared<NT>& sh) {
  uint32_t vmin = 0xffffffffu, vmax = 0u;
  int n_ok = 0;
  cand_for_each(cnt, sh, [&](uint32_t key, uint32_t idx, bool v) {
    if (v && ok(key, idx)) {
      const uint32_t x = val(key, idx);
      vmin = min(vmin, x);
      vmax = max(vmax, x);
      ++n_ok;
    }
  });
  block_minmax(vmin, vmax, sh);
  n_ok = block_sum(n_ok, sh);
  if (vmin == vmax) {
    *above = 0;
    *equal = n_ok;
    return vmin;
  }
  const int h = 31 - __clz(vmin ^ vmax);              // highest bit that differs
  uint32_t mask = h == 31 ? 0u : ~((2u << h) - 1u);   // bits above h: shared by all
  uint32_t prefix = vmin & mask;
  int k_rem = k, n_above = 0, count = n_ok;
  for (int hi = h; hi >= 0; hi -= 8) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dm = (2u << (hi - lo)) - 1u;
    hist_clear(sh);
    __syncthreads();
    cand_for_each(cnt, sh, [&](uint32_t key, uint32_t idx, bool v) {
      if (v && ok(key, idx)) {
        const uint32_t x = val(key, idx);
        if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> lo) & dm], 1u);
      }
    });
    __syncthreads();
    hist_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    n_above += sh.sel_above;
    prefix |= sh.sel_digit << lo;
    mask |= dm << lo;
    count = sh.sel_count;
    __syncthreads();
  }
  *above = n_above;
  *equal = count;
  return prefix;
}

// Exact selection over the collected candidates, which hold every element of
// the row whose key is >= the K-th largest key: appends the indices of the K
// best (key desc, index asc) to sh.kept.
template <int NT>
__device__ void select_candidates(int cnt, int K, TopkShared<NT>& sh) {
  int above, equal;
  const uint32_t T = cand_radix(
      cnt, K, [](uint32_t k, uint32_t) { return k; }, [](uint32_t, uint32_t) { return true; }, &above, &equal,
      sh);
  const int need = K - above;                // elements equal to T to keep (>= 1)
  uint32_t imax = 0xffffffffu;                // keep ties with index <= imax
  if (need < equal) {
    // the need lowest indices among the ties: the need-th largest of ~index
    int a2, e2;
    const uint32_t inv = cand_radix(
        cnt, need, [](uint32_t, uint32_t i) { return ~i; }, [T](uint32_t k, uint32_t) { return k == T; }, &a2,
        &e2, sh);
    imax = ~inv;
  }
  cand_for_each(cnt, sh, [&](uint32_t k, uint32_t i, bool v) {
    keep_if(v && (k > T || (k == T && i <= imax)), i, sh);
  });
  __syncthreads();
}

// Exact fallback streamed over the whole source (any n >= K): four radix
// passes over global memory, then one pass in element (= index) order that
// keeps every element above T and the lowest-indexed ones equal to T.  Src
// provides key(i) and index(i) (a score row, or scores computed on the fly).
template <int NT, class Src>
__device__ void select_streamed(const Src& src, int n, int K, TopkShared<NT>& sh) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int above, equal;
  const uint32_t T = radix_select(
      n, K, [&](int i) { return src.key(i); }, [](int) { return true; }, &above, &equal, sh);
  const int need = K - above;
  // ties in index order: warp w owns a contiguous range of elements
  const int per = (int)cdiv(cdiv(n, TopkCfg<NT>::WARPS), 32) * 32;
  const int beg = warp * per, end = min(n, beg + per);
  int n_tie = 0;
  for (int b = beg; b < end; b += 32) {
    const int i = b + lane;
    n_tie += __popc(__ballot_sync(0xffffffffu, i < end && src.key(i) == T));
  }
  if (lane == 0) sh.warp_b[warp] = n_tie;
  __syncthreads();
  int tie_run = 0;
  for (int w = 0; w < warp; ++w) tie_run += sh.warp_b[w];
  const uint32_t lt = (1u << lane) - 1u;
  for (int b = beg; b < end; b += 32) {
    const int i = b + lane;
    const uint32_t k = i < end ? src.key(i) : 0u;
    const bool tie = i < end && k == T;
    const uint32_t bt = __ballot_sync(0xffffffffu, tie);
    const bool take = (i < end && k > T) || (tie && tie_run + __popc(bt & lt) < need);
    keep_if(take, take ? src.index(i) : 0u, sh);
    tie_run += __popc(bt);
  }
  __syncthreads();
}

// Filter pass of a score row: every element with score >= tau (as floats,
// which matches key >= key(tau)) becomes a candidate of the thread that
// reads it.  16-byte streaming loads over the aligned middle of the row.
template <int NT>
__device__ void filter_scores(const float* row, int64_t base, int n, float tau, int& cnt, TopkShared<NT>& sh) {
  using namespace topk;
  const int align_head = (int)(((16 - ((uintptr_t)row & 15)) & 15) / 4);
  const int head = align_head < n ? align_head : n;
  const int nvec = (n - head) / 4;
  const int tail0 = head + nvec * 4;
  if (threadIdx.x < head) {
    const float s = row[threadIdx.x];
    if (s >= tau) cand_append(score_key(s), (uint32_t)(base + threadIdx.x), cnt, sh);
  } else if (threadIdx.x >= 32 && threadIdx.x < 32 + n - tail0) {
    const int i = tail0 + (int)threadIdx.x - 32;
    const float s = row[i];
    if (s >= tau) cand_append(score_key(s), (uint32_t)(base + i), cnt, sh);
  }
  const float4* v4 = reinterpret_cast<const float4*>(row + head);
  constexpr int U = TopkCfg<NT>::U;
  for (int v0 = threadIdx.x; v0 < nvec; v0 += U * NT) {
    float4 x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * NT;
      x[u] = v < nvec ? __ldg(v4 + v) : make_float4(NAN, NAN, NAN, NAN);   // NaN never passes
    }
    // hits of this thread's 4U elements as a bit mask; most threads have
    // none or one, so the appends loop over set bits, re-reading the value
    // from L1 instead of selecting it among registers
    uint32_t hm = 0;
#pragma unroll
    for (int u = 0; u < U; ++u)
      hm |= ((x[u].x >= tau) ? 1u : 0u) << (4 * u) | ((x[u].y >= tau) ? 2u : 0u) << (4 * u) |
            ((x[u].z >= tau) ? 4u : 0u) << (4 * u) | ((x[u].w >= tau) ? 8u : 0u) << (4 * u);
    while (hm) {
      const int b = __ffs(hm) - 1;
      hm &= hm - 1u;
      const int i = head + 4 * (v0 + (b >> 2) * NT) + (b & 3);
      cand_append(score_key(__ldg(row + i)), (uint32_t)(base + i), cnt, sh);
    }
  }
}

// filter_scores for the wide CTA: each thread streams its 16-byte pieces of
// the row through R private shared-memory slots with cp.async, so R pieces
// per thread are in flight without holding registers (a single CTA must keep
// ~100 KB in flight to stream a long row at a useful rate).
template <int NT, int R>
__device__ void filter_scores_staged(const float* row, int64_t base, int n, float tau, int& cnt, TopkShared<NT>& sh,
                                     float4* ring) {
  const int align_head = (int)(((16 - ((uintptr_t)row & 15)) & 15) / 4);
  const int head = align_head < n ? align_head : n;
  const int nvec = (n - head) / 4;
  const int tail0 = head + nvec * 4;
  if ((int)threadIdx.x < head) {
    const float s = row[threadIdx.x];
    if (s >= tau) cand_append(score_key(s), (uint32_t)(base + threadIdx.x), cnt, sh);
  } else if (threadIdx.x >= 32 && (int)threadIdx.x < 32 + n - tail0) {
    const int i = tail0 + (int)threadIdx.x - 32;
    const float s = row[i];
    if (s >= tau) cand_append(score_key(s), (uint32_t)(base + i), cnt, sh);
  }
  const float4* v4 = reinterpret_cast<const float4*>(row + head);
  const int mine = (int)threadIdx.x < nvec ? (nvec - (int)threadIdx.x + NT - 1) / NT : 0;
#pragma unroll
  for (int k = 0; k < R - 1; ++k) {
    if (k < mine) sm100::cp_async16(sm100::smem_u32(ring + k * NT + threadIdx.x), v4 + threadIdx.x + k * NT, 16);
    sm100::cp_async_commit();
  }
  for (int k = 0; k < mine; ++k) {
    const int kn = k + R - 1;
    if (kn < mine)
      sm100::cp_async16(sm100::smem_u32(ring + (kn % R) * NT + threadIdx.x), v4 + threadIdx.x + (int64_t)kn * NT, 16);
    sm100::cp_async_commit();
    sm100::cp_async_wait<R - 1>();              // this thread's piece k has landed
    const float4 x = ring[(k % R) * NT + threadIdx.x];
    const uint32_t i0 = (uint32_t)(base + head + 4 * ((int)threadIdx.x + k * NT));
    if (x.x >= tau) cand_append(score_key(x.x), i0 + 0, cnt, sh);
    if (x.y >= tau) cand_append(score_key(x.y), i0 + 1, cnt, sh);
    if (x.z >= tau) cand_append(score_key(x.z), i0 + 2, cnt, sh);
    if (x.w >= tau) cand_append(score_key(x.w), i0 + 3, cnt, sh);
  }
  sm100::cp_async_wait_all();
}

// Sampled threshold of src[0..n) (n > CAP): m keys in runs of kSampleGroup
// neighbours spread evenly over the source are reduced to the lower edge of
// a 16-bit-wide bucket holding their rank-th largest, rank chosen so that
// about kSampleTarget elements of the source are expected at or above it.
// The two 8-bit radix passes start below the high bits all samples share (so
// their digits spread over the histogram instead of piling onto a few
// bins).  The result depends only on the source, so CTAs sharing a row agree
// on it.  Ends with a barrier.
template <int NT>
__device__ uint32_t sampled_threshold(const RowSrc& src, int n, TopkShared<NT>& sh,
                                      int max_samples = topk::kMaxSamples, int target = topk::kSampleTarget) {
  using namespace topk;
  const int m0 = n / 16 < kMinSamples ? kMinSamples : (n / 16 > max_samples ? max_samples : n / 16);
  const int groups = m0 / kSampleGroup;
  const int m = groups * kSampleGroup;
  uint32_t vmin = 0xffffffffu, vmax = 0u;
  // group gi starts at gi*(n-8)/(groups-1) <= n-8, so every position is < n
#pragma unroll 8
  for (int s = threadIdx.x; s < m; s += NT) {
    const int gi = s / kSampleGroup, j = s - gi * kSampleGroup;
    const int64_t pos = (int64_t)gi * (n - kSampleGroup) / (groups - 1) + j;
    const uint32_t k = src.key((int)pos);
    sh.cbuf[s] = k;
    vmin = min(vmin, k);
    vmax = max(vmax, k);
  }
  block_minmax(vmin, vmax, sh);
  const int rank = max(1, (int)((int64_t)m * target / n));
  if (vmin == vmax) return vmin;
  const int h = 31 - __clz(vmin ^ vmax);
  uint32_t mask = h == 31 ? 0u : ~((2u << h) - 1u);
  uint32_t prefix = vmin & mask;
  int k_rem = rank;
  for (int hi = h, pass = 0; hi >= 0 && pass < 2; hi -= 8, ++pass) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dm = (2u << (hi - lo)) - 1u;
    hist_clear(sh);
    __syncthreads();
    for (int s = threadIdx.x; s < m; s += NT) {
      const uint32_t x = sh.cbuf[s];
      if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> lo) & dm], 1u);
    }
    __syncthreads();
    hist_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    prefix |= sh.sel_digit << lo;
    mask |= dm << lo;
    __syncthreads();
  }
  return prefix;
}

// Selects the K best elements of src[0..n) (K <= n) under (key desc, index
// asc).  On return sh.kept[0..K) holds their indices, in no particular order.
template <int NT>
__device__ void topk_select(const RowSrc& src, int n, int K, TopkShared<NT>& sh, float4* ring = nullptr) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    sh.n_kept = 0;
    sh.n_ovf = 0;
  }
  const uint32_t tkey = n > CAP ? sampled_threshold(src, n, sh) : 0u;   // 1. (every key is >= 0)
  __syncthreads();
  // 2. filter
  int cnt = 0;
  if (src.scores) {
    if (ring)
      filter_scores_staged<NT, topk::kWideStages>(src.scores, src.base, n, key_to_float(tkey), cnt, sh, ring);
    else
      filter_scores(src.scores, src.base, n, key_to_float(tkey), cnt, sh);
  } else {
    // candidate lists of a merge: batches of loads in flight, then the appends
    constexpr int B = 8;
    for (int i0 = threadIdx.x; i0 < n; i0 += B * NT) {
      uint32_t k[B], ix[B];
#pragma unroll
      for (int u = 0; u < B; ++u) {
        const int i = i0 + u * NT;
        k[u] = i < n ? __ldcs(src.keys + i) : 0u;
        ix[u] = i < n ? (uint32_t)__ldcs(src.idx + i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < B; ++u)
        if (i0 + u * NT < n && k[u] >= tkey) cand_append(k[u], ix[u], cnt, sh);
    }
  }
  __syncthreads();
  const int nc = block_sum(cnt, sh);
  if (nc >= K && sh.n_ovf <= OVF) {
    select_candidates(cnt, K, sh);              // 3.
  } else {
    count_fallback();
    select_streamed(src, n, K, sh);             // exact fallback
  }
  (void)lane;
  (void)warp;
}

// Bitonic sort of a[0..n) (n a power of two), ascending.
__device__ void bitonic_asc(uint32_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = (i & k) == 0;
          const uint32_t x = a[i], y = a[p];
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

struct TopkArgs {
  const float* scores;
  int64_t ld;
  int32_t* sel;
  int32_t* nsel;
  int chunk;            // scores per chunk CTA (few long rows)
  // few long rows (histogram path); hrec and hhist start zeroed
  int32_t* hrec;        // [T][kRecWords] list counters and the row's threshold bin
  uint32_t* hhist;      // [T][kHistBins + kCoarseBins] row histograms of the top 12 and 8 key bits
  int32_t* hsure;       // [T][KMAX] elements above the threshold bin
  uint32_t* hkey;       // [T][CAP] keys of the threshold bin's elements
  int32_t* hidx;        // [T][CAP] their block indices
};

// Puts sh.kept[0..K) (distinct indices in [lo, hi)) in ascending order.  A
// bitmap of the range in the candidate buffer orders them when it fits
// (rows up to 2^18 blocks); otherwise a bitonic sort does.
template <int NT>
__device__ void topk_sort_kept(TopkShared<NT>& sh, int K, int64_t lo, int64_t hi) {
  using namespace topk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t span = hi - lo;
  if (span > (int64_t)kBufWords * 32) {
    constexpr int P = KMAX;
    for (int i = K + threadIdx.x; i < P; i += blockDim.x) sh.kept[i] = 0xffffffffu;
    __syncthreads();
    bitonic_asc(sh.kept, P);
    return;
  }
  uint32_t* bm = sh.cbuf;
  const int nw = (int)((span + 31) >> 5);
  for (int w = threadIdx.x; w < nw; w += NT) bm[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += NT) {
    const uint32_t off = (uint32_t)(sh.kept[i] - lo);
    atomicOr(&bm[off >> 5], 1u << (off & 31));
  }
  __syncthreads();
  // warp w owns the words [beg, end); its lanes read 32 consecutive words at
  // a time (no bank conflicts) and a warp scan of their popcounts places
  // each word's set bits
  constexpr int WARPS = TopkCfg<NT>::WARPS;
  const int per = (int)cdiv(cdiv(nw, WARPS), 32) * 32;
  const int beg = min(nw, warp * per), end = min(nw, beg + per);
  int cnt = 0;
  for (int w = beg + lane; w < end; w += 32) cnt += __popc(bm[w]);
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) sh.warp_a[warp] = cnt;
  __syncthreads();
  int run = 0;
  for (int w = 0; w < warp; ++w) run += sh.warp_a[w];
  for (int w0 = beg; w0 < end; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bits = w < end ? bm[w] : 0u;
    const int c = __popc(bits);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = run + incl - c;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (pos < KMAX) sh.kept[pos] = (uint32_t)(lo + ((int64_t)w << 5) + b);
      ++pos;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncthreads();
}

// Writes the final row: kept blocks ascending, the own block, -1 padding.
template <int NT>
__device__ void topk_write_final(TopkShared<NT>& sh, int K, int S, int64_t bt, int32_t* sel_row) {
  topk_sort_kept(sh, K, 0, bt);
  for (int i = threadIdx.x; i < S; i += blockDim.x)
    sel_row[i] = i < K ? (int32_t)sh.kept[i] : (i == K ? (int32_t)bt : -1);
}

// Few rows, each up to kWideMaxBlocks blocks: one CTA of kWideThreads per
// row, streaming the row through cp.async slots.
__global__ void __launch_bounds__(topk::kWideThreads, 1) topk_wide_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  pdl_wait();
  pdl_trigger();
  __shared__ TopkShared<topk::kWideThreads> sh;
  extern __shared__ float4 ring[];              // kWideRingBytes
  const int S = g.S, K = S - 1;
  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int j = item - st.item0[si];
  const int64_t tok = st.q_offset[si] + j;
  const int64_t bt = (st.pos0[si] + j) / g.r;
  int32_t* sel_row = a.sel + tok * S;
  if (bt + 1 <= S) {
    for (int i = threadIdx.x; i < S; i += blockDim.x) sel_row[i] = (i <= bt) ? i : -1;
    if (threadIdx.x == 0) a.nsel[tok] = (int32_t)(bt + 1);
    return;
  }
  const RowSrc src{a.scores + tok * a.ld, nullptr, nullptr, 0};
  topk_select(src, (int)bt, K, sh, ring);
  topk_write_final(sh, K, S, bt, sel_row);
  if (threadIdx.x == 0) a.nsel[tok] = S;
}

// One chunk of a row (few long rows).
struct TopkItem {
  int64_t tok, bt, c0;
  int n, c, n_ch_row;
  bool all;            // every block in reach is kept (short context)
  bool skip;           // nothing to do for this item
};

__device__ __forceinline__ TopkItem topk_item(const Geo& g, const SegTable& st, const TopkArgs& a, int item) {
  TopkItem it;
  const int si = find_segment(st, item);
  const int local = item - st.item0[si];
  const int64_t pos0 = st.pos0[si];
  const int q_len = st.q_len[si];
  const int64_t nb_seg = cdiv((pos0 + q_len - 1) / g.r, a.chunk);
  const int n_ch_seg = (int)(nb_seg > 1 ? nb_seg : 1);
  const int j = local / n_ch_seg;
  it.c = local - j * n_ch_seg;
  it.tok = st.q_offset[si] + j;
  it.bt = (pos0 + j) / g.r;
  it.all = it.bt + 1 <= g.S;
  it.n_ch_row = it.all ? 1 : (int)cdiv(it.bt, a.chunk);
  it.c0 = (int64_t)it.c * a.chunk;
  it.n = it.all ? 0 : (int)((it.bt - it.c0) < a.chunk ? (it.bt - it.c0) : a.chunk);
  it.skip = it.all ? it.c != 0 : it.c >= it.n_ch_row;
  return it;
}

// Few long rows (decode: a handful of rows of 32K to millions of blocks).
// Three launches, each a stage of the whole batch:
//   topk_hist_kernel (one CTA per 4096-score chunk of a row): the chunk's
//     histogram of the top 12 key bits, added into the row's histogram, and
//     its sums over 16 bins (the top 8 bits) into the row's coarse one;
//   topk_hfilter_kernel (one CTA per chunk): the bin B of the row's (S-1)-th
//     largest key (from the row's coarse histogram of the top 8 key bits,
//     then the 16 fine bins of one coarse bin, found by every chunk CTA while
//     its chunk loads), then the chunk's elements in bins above B ("sure":
//     all kept) and in B ("tied bin") appended to the row's two lists, each
//     CTA reserving its ranges with one atomic per list;
//   topk_hfinal_kernel (one CTA of kWideThreads per row): the sure elements
//     and the best (key desc, index asc) of the tied bin (a radix select
//     over the bin), ordered through a bitmap of the row.  A tied bin larger
//     than its list sends the row to the exact streamed fallback.
// Per token row the workspace holds a record (two list counters, cleared by
// the launcher with the histogram; B and the counts), the histogram, the
// sure list (S-1 entries) and the tied-bin list (CAP pairs).
namespace topk {
enum : int { kRecSure = 0, kRecTie, kRecBin, kRecAbove, kRecCount, kRecWords = 8 };

// The chunk's scores, kHistPer 16-byte groups per thread (coalesced), in
// registers; elements past n read as -inf and are flagged invalid.
struct HistChunk {
  float v[kHistPer * 4];
  __device__ __forceinline__ void load(const float* row, int n) {
    const bool vec = ((uintptr_t)row & 15) == 0;
#pragma unroll
    for (int k = 0; k < kHistPer; ++k) {
      const int i = (k * kHistThreads + (int)threadIdx.x) * 4;
      if (vec && i + 4 <= n) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(row + i));
        v[4 * k] = x.x;
        v[4 * k + 1] = x.y;
        v[4 * k + 2] = x.z;
        v[4 * k + 3] = x.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[4 * k + j] = i + j < n ? __ldcg(row + i + j) : -INFINITY;
      }
    }
  }
  __device__ __forceinline__ static int index(int e) {       // element e of this thread
    return ((e >> 2) * kHistThreads + (int)threadIdx.x) * 4 + (e & 3);
  }
};

// The fine bin of a row histogram gh (kHistBins fine bins, then kCoarseBins
// coarse bins, in global memory) that holds the k-th largest element: first
// the coarse bin from the 256 coarse counts (one per thread), then, by warp 0,
// the fine bin among that coarse bin's 16.  *bin, *above = elements in
// higher fine bins, *count = elements in that bin.  Ends with a barrier.
template <int NT>
__device__ void hist_row_locate(const uint32_t* gh, int k, uint32_t* bin, int* above, int* count,
                                TopkShared<NT>& sh) {
  static_assert(NT == kCoarseBins, "one coarse bin per thread");
  constexpr int WARPS = TopkCfg<NT>::WARPS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = (int)__ldcg(gh + kHistBins + threadIdx.x);
  int suf = c;                                   // this and higher lanes of the warp
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  if (lane == 0) sh.warp_a[warp] = suf;
  __syncthreads();
  int higher = 0;
  for (int w = warp + 1; w < WARPS; ++w) higher += sh.warp_a[w];
  const int ex = higher + suf - c;               // elements in higher coarse bins
  if (ex < k && k <= ex + c) {
    sh.sel_digit = threadIdx.x;
    sh.sel_above = ex;
  }
  __syncthreads();
  if (warp == 0) {
    const int cb = (int)sh.sel_digit, cab = sh.sel_above;
    const int f = lane < 16 ? (int)__ldcg(gh + cb * 16 + lane) : 0;
    int fs = f;                                  // fine bins >= this one, within the coarse bin
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_down_sync(0xffffffffu, fs, off);
      if (lane + off < 32) fs += v;
    }
    const int fex = cab + fs - f;
    if (lane < 16 && fex < k && k <= fex + f) {
      sh.sel_digit = (uint32_t)(cb * 16 + lane);
      sh.sel_above = fex;
      sh.sel_count = f;
    }
  }
  __syncthreads();
  *bin = sh.sel_digit;
  *above = sh.sel_above;
  *count = sh.sel_count;
  __syncthreads();
}
}  // namespace topk

__global__ void __launch_bounds__(topk::kHistThreads) topk_hist_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist[kHistBins];
  const TopkItem it = topk_item(g, st, a, blockIdx.x);
  if (it.skip || it.all) return;
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads) hist[b] = 0u;
  HistChunk ch;
  ch.load(a.scores + it.tok * a.ld + it.c0, it.n);
  __syncthreads();
#pragma unroll
  for (int e = 0; e < kHistPer * 4; ++e)
    if (HistChunk::index(e) < it.n) atomicAdd(&hist[score_key(ch.v[e]) >> kHistShift], 1u);
  __syncthreads();
  uint32_t* gh = a.hhist + it.tok * (kHistBins + kCoarseBins);
  for (int b = threadIdx.x; b < kHistBins; b += kHistThreads) {
    const uint32_t c = hist[b];
    if (c) atomicAdd(&gh[b], c);
  }
  // coarse bin t: fine bins [16 t, 16 t + 16)
  static_assert(kHistThreads == kCoarseBins, "one coarse bin per thread");
  uint32_t cs = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) cs += hist[threadIdx.x * 16 + ((j + threadIdx.x) & 15)];
  if (cs) atomicAdd(&gh[kHistBins + threadIdx.x], cs);
}

__global__ void __launch_bounds__(topk::kHistThreads, 4) topk_hfilter_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  constexpr int NT = kHistThreads;
  constexpr int E = kHistPer * 4;
  pdl_wait();
  pdl_trigger();
  __shared__ TopkShared<NT> sh;
  __shared__ int s_base_sure, s_base_tie;
  const int S = g.S, K = S - 1;
  const TopkItem it = topk_item(g, st, a, blockIdx.x);
  if (it.skip) return;
  int32_t* sel_row = a.sel + it.tok * S;
  if (it.all) {
    for (int i = threadIdx.x; i < S; i += NT) sel_row[i] = (i <= it.bt) ? i : -1;
    if (threadIdx.x == 0) a.nsel[it.tok] = (int32_t)(it.bt + 1);
    return;
  }
  HistChunk ch;
  ch.load(a.scores + it.tok * a.ld + it.c0, it.n);          // in flight while the threshold is found
  uint32_t B;
  int above, count;
  hist_row_locate(a.hhist + it.tok * (kHistBins + kCoarseBins), K, &B, &above, &count, sh);
  int32_t* rec = a.hrec + it.tok * kRecWords;
  if (it.c == 0 && threadIdx.x == 0) {
    rec[kRecBin] = (int32_t)B;
    rec[kRecAbove] = above;
    rec[kRecCount] = count;
  }
  if (count > CAP) return;                                  // the final kernel falls back
  uint32_t is_sure = 0u, is_tie = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t bin = score_key(ch.v[e]) >> kHistShift;
    const bool in = HistChunk::index(e) < it.n;
    is_sure |= (uint32_t)(in && bin > B) << e;
    is_tie |= (uint32_t)(in && bin == B) << e;
  }
  int tot_sure, tot_tie;
  const int ex_sure = block_exscan(__popc(is_sure), &tot_sure, sh);
  const int ex_tie = block_exscan(__popc(is_tie), &tot_tie, sh);
  if (threadIdx.x == 0) {
    s_base_sure = tot_sure ? atomicAdd(rec + kRecSure, tot_sure) : 0;
    s_base_tie = tot_tie ? atomicAdd(rec + kRecTie, tot_tie) : 0;
  }
  __syncthreads();
  int32_t* sure = a.hsure + it.tok * KMAX;
  uint32_t* tkey = a.hkey + it.tok * CAP;
  int32_t* tidx = a.hidx + it.tok * CAP;
  int ps = s_base_sure + ex_sure, pt = s_base_tie + ex_tie;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = HistChunk::index(e);
    if ((is_sure >> e) & 1u) {
      if (ps < KMAX) sure[ps] = (int32_t)(it.c0 + i);
      ++ps;
    } else if ((is_tie >> e) & 1u) {
      if (pt < CAP) {
        tkey[pt] = score_key(ch.v[e]);
        tidx[pt] = (int32_t)(it.c0 + i);
      }
      ++pt;
    }
  }
}

// One CTA per row: the sure elements, then the best K - above of the tied bin.
__global__ void __launch_bounds__(topk::kWideThreads, 1) topk_hfinal_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  constexpr int NT = kWideThreads;
  pdl_wait();
  pdl_trigger();
  __shared__ TopkShared<NT> sh;
  const int S = g.S, K = S - 1;
  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int j = item - st.item0[si];
  const int64_t tok = st.q_offset[si] + j;
  const int64_t bt = (st.pos0[si] + j) / g.r;
  if (bt + 1 <= S) return;                                  // written by the filter kernel
  const int32_t* rec = a.hrec + tok * kRecWords;
  const int above = __ldcg(rec + kRecAbove), count = __ldcg(rec + kRecCount);
  if (threadIdx.x == 0) {
    sh.n_kept = 0;
    sh.n_ovf = 0;
  }
  __syncthreads();
  if (count <= CAP) {
    int cnt = 0;
    for (int i = threadIdx.x; i < count; i += NT)
      cand_append(__ldcg(a.hkey + tok * CAP + i), (uint32_t)__ldcg(a.hidx + tok * CAP + i), cnt, sh);
    for (int i = threadIdx.x; i < above; i += NT) sh.kept[i] = (uint32_t)__ldcg(a.hsure + tok * KMAX + i);
    if (threadIdx.x == 0) sh.n_kept = above;
    __syncthreads();
    select_candidates(cnt, K - above, sh);
  } else {
    const RowSrc row{a.scores + tok * a.ld, nullptr, nullptr, 0};
    count_fallback();
    select_streamed(row, (int)bt, K, sh);
  }
  topk_write_final(sh, K, S, bt, a.sel + tok * S);
  if (threadIdx.x == 0) a.nsel[tok] = S;
}

// ---------------------------------------------------------------- many rows: one warp per row
// The 4-warp CTA per row above spends most of a row in barrier-separated
// phases with no loads in flight.  Here each warp selects its own row with
// warp-synchronous steps only, so an SM has 24 rows in flight (4 warps x 6
// CTAs) whose load phases overlap each other's selection phases.  The number
// of rows in flight sets the speed: each row is a chain of dependent steps,
// and its loads go through cp.async (16-byte loads into registers stalled in
// the L1 miss path at about 2 TB/s over all SMs, however many were in flight).
//   1. rows of at most CAPW candidates take them all; longer rows take the
//      lower edge of the 16-bit bucket of the rank-th largest of m = n/16
//      sampled keys (runs of 8 neighbours on 16-byte boundaries, copied to
//      shared memory all at once), rank chosen so that about TARGET elements
//      of the row are expected at or above it;
//   2. filter: the row streams through a ring of RS slots of 32 x U 16-byte
//      pieces per warp; the lanes' hits are compacted into the warp's list by
//      a warp prefix sum, in ascending block order;
//   3. if the list holds K..CAPW elements: exact radix select (8-bit digits
//      below the common high bits, then lowest indices among the ties);
//   4. the kept elements, read from the list in its order, are already in
//      ascending block order.
// A row whose list holds fewer than K or more than CAPW elements is marked
// (nsel = -1) and selected exactly by topk_rows_fallback_kernel.  Rows of
// more than 64K blocks are marked -2 and left to that kernel's 4-warp CTAs:
// one warp keeps too few loads in flight to stream them.
namespace topk_w {
constexpr int WARPS = 4;
constexpr int THREADS = 32 * WARPS;
constexpr int CAPW = 1024;                 // candidates a row may collect
constexpr int BUFW = 2 * CAPW;             // sample keys held in shared memory
constexpr int TARGET = 768;                // expected elements at or above the sampled threshold
constexpr int MIN_S = 512;
constexpr int MAX_S = 16384;               // samples beyond BUFW are re-read from the row each pass
constexpr int U = 2;                       // 16-byte loads in flight per lane (at most 4: a byte each)
constexpr int RS = 2;                      // ring slots of U x 32 16-byte pieces per warp
constexpr int CTAS = 6;                    // resident CTAs per SM (shared memory, 80 registers)
constexpr int64_t kMaxRowBlocks = 65536;   // longer rows go to 4-warp CTAs; 16-bit candidate indices
static_assert(U <= 4, "a packed count holds one byte per load row");
static_assert(kMaxRowBlocks <= 65536, "candidate indices are held in 16 bits");
static_assert(RS * U * 32 * 16 + CAPW * 6 <= BUFW * 4, "the ring and the candidates fit the sample space");
}

// Per warp: the sample keys (step 1) share their space with the filter's
// ring and the candidate list (steps 2-4).  Candidate indices are below
// kMaxRowBlocks = 2^16, so 16 bits hold them.
struct alignas(16) WarpRowShared {
  uint32_t hist[topk::NBINS];
  union {
    uint32_t sample[topk_w::BUFW];
    struct {
      float4 ring[topk_w::RS][topk_w::U * 32];
      uint32_t key[topk_w::CAPW];
      uint16_t idx[topk_w::CAPW];
    } f;
  };
};

// Bin holding the k-th largest counted value: each lane owns 8 consecutive
// bins; suffix sums run from the top bin down.  Returns the digit; *above =
// count in higher bins, *count = the bin's count.  Warp-uniform results.
__device__ __forceinline__ uint32_t warp_hist_locate(const uint32_t* hist, int k, int* above, int* count) {
  const int lane = threadIdx.x & 31;
  uint32_t b[8];
  int local = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    b[j] = hist[lane * 8 + j];
    local += (int)b[j];
  }
  int suf = local;                              // this lane and the lanes above it
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_down_sync(0xffffffffu, suf, off);
    if (lane + off < 32) suf += v;
  }
  const int excl = suf - local;                 // lanes above
  uint32_t digit = 0;
  int ab = 0, cnt = 0;
  const bool mine = excl < k && k <= suf;
  if (mine) {
    int run = excl;
    for (int j = 7; j >= 0; --j) {
      if (run + (int)b[j] >= k) {
        digit = (uint32_t)(lane * 8 + j);
        ab = run;
        cnt = (int)b[j];
        break;
      }
      run += (int)b[j];
    }
  }
  const int src = max(0, __ffs(__ballot_sync(0xffffffffu, mine)) - 1);
  *above = __shfl_sync(0xffffffffu, ab, src);
  *count = __shfl_sync(0xffffffffu, cnt, src);
  return __shfl_sync(0xffffffffu, digit, src);
}

// Radix select over n values val(i) (those with ok(i)) held by the warp:
// passes of 8-bit digits from the highest bit where min and max differ; at
// most `max_passes` passes (2: a 16-bit bucket).  Returns the prefix; *above
// and *equal as in cand_radix.
template <class Val, class Ok>
__device__ uint32_t warp_radix(int n, int k, Val val, Ok ok, int* above, int* equal, uint32_t* hist,
                               int max_passes = 4) {
  const int lane = threadIdx.x & 31;
  uint32_t vmin = 0xffffffffu, vmax = 0u;
  int n_ok = 0;
  for (int i = lane; i < n; i += 32) {
    if (ok(i)) {
      const uint32_t x = val(i);
      vmin = min(vmin, x);
      vmax = max(vmax, x);
      ++n_ok;
    }
  }
  vmin = __reduce_min_sync(0xffffffffu, vmin);
  vmax = __reduce_max_sync(0xffffffffu, vmax);
  n_ok = __reduce_add_sync(0xffffffffu, n_ok);
  if (vmin == vmax) {
    *above = 0;
    *equal = n_ok;
    return vmin;
  }
  const int h = 31 - __clz(vmin ^ vmax);
  uint32_t mask = h == 31 ? 0u : ~((2u << h) - 1u);
  uint32_t prefix = vmin & mask;
  int k_rem = k, n_above = 0, count = n_ok;
  for (int hi = h, pass = 0; hi >= 0 && pass < max_passes; hi -= 8, ++pass) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dm = (2u << (hi - lo)) - 1u;
#pragma unroll
    for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      if (ok(i)) {
        const uint32_t x = val(i);
        if ((x & mask) == prefix) atomicAdd(&hist[(x >> lo) & dm], 1u);
      }
    }
    __syncwarp();
    int ab, cnt;
    const uint32_t d = warp_hist_locate(hist, k_rem, &ab, &cnt);
    k_rem -= ab;
    n_above += ab;
    prefix |= d << lo;
    mask |= dm << lo;
    count = cnt;
    __syncwarp();
  }
  *above = n_above;
  *equal = count;
  return prefix;
}

__global__ void __launch_bounds__(topk_w::THREADS, topk_w::CTAS) topk_rows_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  using namespace topk_w;
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) unsigned char topk_rows_smem[];
  WarpRowShared* shw = reinterpret_cast<WarpRowShared*>(topk_rows_smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WarpRowShared& sh = shw[warp];
  uint32_t* ckey = sh.f.key;
  uint16_t* cidx = sh.f.idx;
  const int n_items = st.item0[st.n];
  const int S = g.S, K = S - 1;
  const uint32_t below = (1u << lane) - 1u;
  for (int item = blockIdx.x * WARPS + warp; item < n_items; item += gridDim.x * WARPS) {
    const int si = find_segment(st, item);
    const int j = item - st.item0[si];
    const int64_t tok = st.q_offset[si] + j;
    const int64_t bt = ((int64_t)st.pos0[si] + j) / g.r;
    int32_t* sel_row = a.sel + tok * S;
    if (bt + 1 <= S) {
      for (int i = lane; i < S; i += 32) sel_row[i] = (i <= bt) ? i : -1;
      if (lane == 0) a.nsel[tok] = (int32_t)(bt + 1);
      continue;
    }
    if (bt > kMaxRowBlocks) {
      if (lane == 0) a.nsel[tok] = -2;            // a long row: selected by a 4-warp CTA
      continue;
    }
    const int n = (int)bt;
    const float* row = a.scores + tok * a.ld;
    // the row as a ragged head, nvec 16-byte pieces and a ragged tail
    const int head = min(n, (int)(((16 - ((uintptr_t)row & 15)) & 15) / 4));
    const int nvec = (n - head) / 4;
    const int tail0 = head + nvec * 4;
    const float4* v4 = reinterpret_cast<const float4*>(row + head);
    // 1. threshold
    uint32_t tkey = 0u;
    if (n > CAPW) {
      const int m0 = n / 16 < MIN_S ? MIN_S : (n / 16 > MAX_S ? MAX_S : n / 16);
      const int groups = m0 / kSampleGroup;
      const int m = groups * kSampleGroup;
      // group gi: the 8 elements of pieces q, q+1 with q = gi*(nvec-2)/(groups-1)
      // (nvec >= 255 here; gi < 2048 and nvec <= 16384 keep the product below 2^25)
      const uint32_t qspan = (uint32_t)(nvec - 2), den = (uint32_t)(groups - 1);
      const int rank = max(1, (int)((int64_t)m * TARGET / n));
      int ab, eq;
      if (m <= BUFW) {
        // every lane's groups in flight at once: two 16-byte copies each
        for (int gi = lane; gi < groups; gi += 32) {
          const uint32_t q = (uint32_t)gi * qspan / den;
          sm100::cp_async16(sm100::smem_u32(sh.sample + gi * kSampleGroup), v4 + q, 16);
          sm100::cp_async16(sm100::smem_u32(sh.sample + gi * kSampleGroup + 4), v4 + q + 1, 16);
        }
        sm100::cp_async_wait_all();
        __syncwarp();
        tkey = warp_radix(
            m, rank, [&](int i) { return score_key(__uint_as_float(sh.sample[i])); }, [](int) { return true; }, &ab,
            &eq, sh.hist, 2);
      } else {
        auto sample = [&](int s_i) -> uint32_t {
          const uint32_t gi = (uint32_t)s_i / kSampleGroup, jj = (uint32_t)s_i % kSampleGroup;
          return score_key(row[head + 4 * (gi * qspan / den) + jj]);
        };
        tkey = warp_radix(m, rank, sample, [](int) { return true; }, &ab, &eq, sh.hist, 2);
      }
      __syncwarp();
    }
    const float tau = key_to_float(tkey);
    // 2. filter into the warp's list in ascending block order: the ragged
    // head, then per iteration U rows of 32 16-byte loads (byte u of a packed
    // count holds row u's hits, so one warp scan gives every row's offsets),
    // then the ragged tail
    int nc = 0;                                   // warp-uniform count (may exceed CAPW)
    auto append_one = [&](int e) {                // one element per lane, e < 0: none
      const float v = e >= 0 ? row[e] : 0.f;
      const bool hit = e >= 0 && v >= tau;
      const uint32_t mb = __ballot_sync(0xffffffffu, hit);
      const int pos = nc + __popc(mb & below);
      if (hit && pos < CAPW) {
        ckey[pos] = score_key(v);
        cidx[pos] = (uint16_t)e;
      }
      nc += __popc(mb);
    };
    append_one(lane < head ? lane : -1);
    const int iters = (nvec + 32 * U - 1) / (32 * U);
    // iteration `it` of the row through ring slot it % RS: each lane copies
    // its own U pieces and later reads back only those (no warp barrier)
    auto issue = [&](int it) {
      float4* slot = sh.f.ring[it % RS];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int vi = it * 32 * U + u * 32 + lane;
        if (vi < nvec) sm100::cp_async16(sm100::smem_u32(slot + u * 32 + lane), v4 + vi, 16);
      }
      sm100::cp_async_commit();
    };
#pragma unroll
    for (int k = 0; k < RS - 1; ++k) issue(k);
    for (int it = 0; it < iters; ++it) {
      const int b = it * 32 * U;
      issue(it + RS - 1);                         // the slot read in the previous iteration
      sm100::cp_async_wait<RS - 1>();             // this lane's pieces of iteration `it` have landed
      float4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int vi = b + u * 32 + lane;
        x[u] = vi < nvec ? sh.f.ring[it % RS][u * 32 + lane] : make_float4(NAN, NAN, NAN, NAN);   // NaN never passes
      }
      uint32_t hm[U];                             // the lane's hits in piece u, a bit per element
      uint32_t packed = 0u;                       // a byte per row: at most 4 x 32 = 128
#pragma unroll
      for (int u = 0; u < U; ++u) {
        hm[u] = (uint32_t)(x[u].x >= tau) | (uint32_t)(x[u].y >= tau) << 1 | (uint32_t)(x[u].z >= tau) << 2 |
                (uint32_t)(x[u].w >= tau) << 3;
        packed |= (uint32_t)__popc(hm[u]) << (8 * u);
      }
      uint32_t incl = packed;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
      const uint32_t excl = incl - packed;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        int o = nc + (int)((excl >> (8 * u)) & 255u);
        const uint32_t i0 = (uint32_t)(head + 4 * (b + u * 32 + lane));
        // one trip per hit of the lane (few pass the threshold), in element order
        for (uint32_t bits = hm[u]; bits; bits &= bits - 1u) {
          const int c = __ffs(bits) - 1;
          const float v = c == 0 ? x[u].x : c == 1 ? x[u].y : c == 2 ? x[u].z : x[u].w;
          if (o < CAPW) {
            ckey[o] = score_key(v);
            cidx[o] = (uint16_t)(i0 + c);
          }
          ++o;
        }
        nc += (int)((tot >> (8 * u)) & 255u);
      }
    }
    sm100::cp_async_wait_all();
    append_one(lane < n - tail0 ? tail0 + lane : -1);
    __syncwarp();
    if (nc < K || nc > CAPW) {
      if (lane == 0) {
        a.nsel[tok] = -1;                         // exact selection by the fallback kernel
        atomicAdd(&g_qsa_select_fallbacks, 1ull);
      }
      continue;
    }
    // 3. exact selection among the nc candidates
    int above, equal;
    const uint32_t T = warp_radix(
        nc, K, [&](int i) { return ckey[i]; }, [](int) { return true; }, &above, &equal, sh.hist);
    const int need = K - above;
    uint32_t imax = 0xffffffffu;
    if (need < equal) {
      int a2, e2;
      imax = ~warp_radix(
          nc, need, [&](int i) { return ~(uint32_t)cidx[i]; }, [&](int i) { return ckey[i] == T; }, &a2, &e2, sh.hist);
    }
    // 4. the list is in ascending block order, so the kept candidates are
    // written in order as they are found, then the own block
    int nk = 0;
    for (int b = 0; b < nc; b += 32) {
      const int i = b + lane;
      const bool take = i < nc && (ckey[i] > T || (ckey[i] == T && (uint32_t)cidx[i] <= imax));
      const uint32_t mb = __ballot_sync(0xffffffffu, take);
      const int pos = nk + __popc(mb & below);
      if (take && pos < K) sel_row[pos] = (int32_t)cidx[i];
      nk += __popc(mb);
    }
    for (int i = K + lane; i < S; i += 32) sel_row[i] = i == K ? (int32_t)bt : -1;
    if (lane == 0) a.nsel[tok] = S;
    __syncwarp();                                 // shared state is reused by the next row
  }
}

// Rows topk_rows_kernel marked (nsel = -1 or -2): selection by a 4-warp CTA
// (sampled threshold, filter, candidate selection, or the streamed fallback).
// Launched without programmatic chaining and with no early trigger: its CTAs
// mostly skip rows, and a dependent kernel made resident early would take
// the SMs its remaining CTAs need.
__global__ void __launch_bounds__(topk::THREADS, 6) topk_rows_fallback_kernel(Geo g, SegTable st, TopkArgs a) {
  using namespace topk;
  __shared__ TopkShared<topk::THREADS> sh;
  const int n_items = st.item0[st.n];
  const int S = g.S, K = S - 1;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int si = find_segment(st, item);
    const int j = item - st.item0[si];
    const int64_t tok = st.q_offset[si] + j;
    const int mark = a.nsel[tok];
    if (mark != -1 && mark != -2) continue;      // uniform across the CTA
    const int64_t bt = ((int64_t)st.pos0[si] + j) / g.r;
    const RowSrc src{a.scores + tok * a.ld, nullptr, nullptr, 0};
    topk_select(src, (int)bt, K, sh);
    topk_write_final(sh, K, S, bt, a.sel + tok * S);
    if (threadIdx.x == 0) a.nsel[tok] = S;
    __syncthreads();
  }
}

// ---------------------------------------------------------------- fused prefill selection
// Many rows of prefill-like segments skip the score matrix:
//   1. the indexer scores an evenly spaced sample, pooled block j*stride;
//   2. topk_tau_kernel: per row, the threshold key below which about
//      kSampleTarget elements of the row are expected (the lower edge of the
//      16-bit bucket of the sample's matching rank), and a zeroed count;
//   3. the indexer in filter mode appends every candidate with score >= tau
//      (the float of that key) to the row's list (up to CAP entries; the
//      count keeps counting);
//   4. topk_cand_kernel: when the list holds between K and CAP elements it
//      holds every element of the row at or above the K-th largest, so the
//      exact candidate selection gives the row's answer; otherwise an exact
//      streamed selection runs over scores recomputed on CUDA cores.
// Rows with n <= CAP take tau = 0 (every key passes); rows that keep every
// block take tau = ~0 and need no candidates.
struct FusedSelArgs {
  const float* samples;          // [T][ld_s] sample scores (row j = block j*stride)
  int64_t ld_s;
  int stride;
  float* tau;                    // [T] threshold (-inf: keep all, NaN: none)
  const float* cand_score;       // [T][CAP]
  const int32_t* cand_idx;       // [T][CAP]
  int32_t* cand_cnt;             // [T]
  int32_t* sel;                  // [T][S]
  int32_t* nsel;                 // [T]
  // exact fallback: scores recomputed from the indexer inputs
  const __nv_bfloat16* q_idx;    // [T][4][DI]
  const float* w;                // [T][4]
  const __nv_bfloat16* khat;     // [n_slots][n_cap/r][DI]
};

// Lower edge of the 16-bit bucket (below the bits all keys share) holding
// the rank-th largest key of row[0..n); at least `rank` keys are >= it.
// Keys are staged in shared memory when they fit.  Ends with a barrier.
template <int NT>
__device__ uint32_t rank_threshold(const float* row, int n, int rank, TopkShared<NT>& sh) {
  using namespace topk;
  const bool staged = n <= kBufWords;
  uint32_t vmin = 0xffffffffu, vmax = 0u;
  for (int i = threadIdx.x; i < n; i += NT) {
    const uint32_t k = score_key(row[i]);
    if (staged) sh.cbuf[i] = k;
    vmin = min(vmin, k);
    vmax = max(vmax, k);
  }
  block_minmax(vmin, vmax, sh);
  if (vmin == vmax) return vmin;
  const int h = 31 - __clz(vmin ^ vmax);
  uint32_t mask = h == 31 ? 0u : ~((2u << h) - 1u);
  uint32_t prefix = vmin & mask;
  int k_rem = rank;
  for (int hi = h, pass = 0; hi >= 0 && pass < 2; hi -= 8, ++pass) {
    const int lo = hi >= 7 ? hi - 7 : 0;
    const uint32_t dm = (2u << (hi - lo)) - 1u;
    hist_clear(sh);
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
      const uint32_t x = staged ? sh.cbuf[i] : score_key(row[i]);
      if ((x & mask) == prefix) atomicAdd(&sh.hist[(x >> lo) & dm], 1u);
    }
    __syncthreads();
    hist_locate(k_rem, sh);
    k_rem -= sh.sel_above;
    prefix |= sh.sel_digit << lo;
    mask |= dm << lo;
    __syncthreads();
  }
  return prefix;
}

struct FusedRow {
  int64_t tok, t, bt, slot;
};

__device__ __forceinline__ FusedRow fused_row(const Geo& g, const SegTable& st, int item) {
  FusedRow r;
  const int si = find_segment(st, item);
  const int j = item - st.item0[si];
  r.tok = st.q_offset[si] + j;
  r.t = (int64_t)st.pos0[si] + j;
  r.bt = r.t / g.r;
  r.slot = st.slot[si];
  return r;
}

// NT threads per row: 128 when rows are many (six CTAs per SM), 1024 when
// they are few (decode).
template <int NT>
__global__ void __launch_bounds__(NT, NT >= 512 ? 1 : 6) topk_tau_kernel(Geo g, SegTable st, FusedSelArgs a) {
  using namespace topk;
  pdl_wait();
  pdl_trigger();
  __shared__ TopkShared<NT> sh;
  const int n_items = st.item0[st.n];
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const FusedRow r = fused_row(g, st, item);
    uint32_t tkey;
    if (r.bt + 1 <= g.S) {
      tkey = 0xffffffffu;                        // every block is kept: no candidates needed (NaN)
    } else if (r.bt <= CAP) {
      tkey = 0u;                                 // every element fits the list (-inf)
    } else {
      const int n = (int)r.bt;
      const int n_s = (int)cdiv(n, a.stride);    // samples j*stride < n
      const int rank = max(1, (int)((int64_t)n_s * kSampleTarget / n));
      tkey = rank_threshold(a.samples + r.tok * a.ld_s, n_s, rank, sh);
    }
    if (threadIdx.x == 0) {
      a.tau[r.tok] = key_to_float(tkey);         // score >= it  <=>  key >= tkey
      a.cand_cnt[r.tok] = 0;
    }
    __syncthreads();                             // shared state is reused by the next item
  }
}

// Scores of one row computed on CUDA cores for the exact fallback: element i
// is block i, s = sum_h w_h ReLU(q~_h . k^_i) with q~ (rotated, rounded to
// bf16 like the tensor-core path) staged in shared memory as fp32.
struct ComputedRow {
  const float* qt;               // [4][DI] shared
  const __nv_bfloat16* kh;       // the slot's k^ rows
  float4 w;
  int DI;
  __device__ __forceinline__ uint32_t key(int i) const {
    const uint4* kr = reinterpret_cast<const uint4*>(kh + (int64_t)i * DI);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < DI / 8; ++c) {
      const uint4 raw = kr[c];
      const __nv_bfloat16* kv = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = __bfloat162float(kv[e]);
#pragma unroll
        for (int h = 0; h < 4; ++h) acc[h] = fmaf(qt[h * DI + 8 * c + e], x, acc[h]);
      }
    }
    float s = 0.f;
    s = fmaf(w.x, fmaxf(acc[0], 0.f), s);
    s = fmaf(w.y, fmaxf(acc[1], 0.f), s);
    s = fmaf(w.z, fmaxf(acc[2], 0.f), s);
    s = fmaf(w.w, fmaxf(acc[3], 0.f), s);
    return score_key(s);
  }
  __device__ __forceinline__ uint32_t index(int i) const { return (uint32_t)i; }
};

template <int NT>
__global__ void __launch_bounds__(NT, NT >= 512 ? 1 : 6) topk_cand_kernel(Geo g, SegTable st, FusedSelArgs a) {
  using namespace topk;
  pdl_wait();
  pdl_trigger();
  __shared__ TopkShared<NT> sh;
  const int n_items = st.item0[st.n];
  const int S = g.S, K = S - 1;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const FusedRow r = fused_row(g, st, item);
    int32_t* sel_row = a.sel + r.tok * S;
    if (r.bt + 1 <= S) {
      for (int i = threadIdx.x; i < S; i += blockDim.x) sel_row[i] = (i <= r.bt) ? i : -1;
      if (threadIdx.x == 0) a.nsel[r.tok] = (int32_t)(r.bt + 1);
      continue;
    }
    if (threadIdx.x == 0) {
      sh.n_kept = 0;
      sh.n_ovf = 0;
    }
    const int nc = a.cand_cnt[r.tok];
    __syncthreads();
    if (nc >= K && nc <= CAP) {
      // at most CAP/NT per thread: CAPL own slots, the rest (<= OVF in all) in overflow
      int cnt = 0;
      const int64_t base = r.tok * (int64_t)CAP;
      for (int i = threadIdx.x; i < nc; i += NT)
        cand_append(score_key(a.cand_score[base + i]), (uint32_t)a.cand_idx[base + i], cnt, sh);
      __syncthreads();
      select_candidates(cnt, K, sh);
    } else {
      count_fallback();
      float* qt = reinterpret_cast<float*>(sh.cbuf);        // unused by the streamed selection
      const int DI = g.DI, half = g.rope_half;
      const __nv_bfloat16* qr = a.q_idx + r.tok * 4 * (int64_t)DI;
      for (int e = threadIdx.x; e < 4 * DI; e += NT) {
        const int h = e / DI, d = e - h * DI;
        float v = __bfloat162float(qr[e]);
        if (d < 2 * half) {
          const int p = d < half ? d : d - half;
          float c, sn, o0, o1;
          rope_cs(g, r.t, p, c, sn);
          rope_pair(__bfloat162float(qr[h * DI + p]), __bfloat162float(qr[h * DI + p + half]), c, sn, o0, o1);
          v = __bfloat162float(__float2bfloat16_rn(d < half ? o0 : o1));
        }
        qt[e] = v;
      }
      __syncthreads();
      const float4 w4 = *reinterpret_cast<const float4*>(a.w + r.tok * 4);
      const ComputedRow src{qt, a.khat + r.slot * (g.n_cap / g.r) * (int64_t)DI, w4, DI};
      select_streamed(src, (int)r.bt, K, sh);
    }
    topk_write_final(sh, K, S, r.bt, sel_row);
    if (threadIdx.x == 0) a.nsel[r.tok] = S;
    __syncthreads();                             // shared state is reused by the next item
  }
}

}  // namespace qsa
