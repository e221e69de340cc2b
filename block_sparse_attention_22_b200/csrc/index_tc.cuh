// index_tc.cuh -- indexer scores on tcgen05 tensor cores (bf16 I/O).
//
// Design report summary page ("Qwen3.8-Next architecture design report"),
// QSA item: a 4-head MQA indexer scores every causal micro-block; scoring
// costs O(n^2/r).  With s(t,b) = sum_h w[t,h] * ReLU(q~[t,h] . k^[b]) this is
// a dense contraction of pooled keys against rotated queries:
//   ACC[b, (q,h)] = k^[b, :] . q~[q, h, :]      M = 128 blocks, N = 4*NQ, K = idx_dim
// followed by a per-block epilogue s = sum_h w[q,h] * max(ACC, 0).
//
// Work is the flat sequence of (segment, tile of NQ consecutive queries,
// 128-block k^ tile) triples, ordered by segment, query tile, k^ tile.  The
// kernel is persistent: CTA c takes the c-th of grid equal contiguous slices
// of that sequence (measured in k^ tiles plus a fixed weight per query tile
// for building its rotated queries), so every SM gets the same work and
// walks few query tiles (the rotated query tile is built once per query
// tile, not once per k^ tile).  The number of k^ tiles before query tile J of
// a segment has a closed form (a floor sum), which lets a CTA seek to its
// slice.
//
// The k^ tensor map is [slot][row][dim] with row j = pooled block j*stride:
// stride 1 scores every block; a larger stride scores an evenly spaced
// sample of them (the row threshold of the fused selection comes from it).
// In filter mode the epilogue writes no scores: it appends (key, block) for
// the candidates at or above the token's threshold key to the token's
// candidate list (warp-aggregated atomics on the list's count).
//
// NQ = 64 for prefill (N = 256; TMEM holds two 128x256 fp32 accumulators),
// NQ = 4 for decode (N = 16; the kernel then streams each sequence's k^ at
// HBM rate through a deeper ring).  Roles (one CTA per SM):
//   warp 0      TMA producer: k^ tiles (128 rows x idx_dim as 64-dim boxes)
//               into a ring of shared-memory stages;
//   warp 1      TMEM owner and single-thread MMA issuer;
//   warps 2..   at each new query tile: q~ = RoPE_t(q_idx) rounded to bf16
//               into the swizzled B tile (fp32 arithmetic in the same fixed
//               order as the key pooling; the partner of a rotated pair comes
//               from the neighbouring lane), then per k^ tile the epilogue:
//               4 warps per TMEM lane quadrant, each reading its share of the
//               columns into registers, releasing the accumulator, and
//               writing scores[t][b] for b < floor(t/r) as 128-byte rows.
// Every mbarrier wait is bounded.
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"

namespace qsa {
namespace tc_index {
constexpr int kTileRows = 128;             // k^ blocks per tile (MMA M)
constexpr int kMaxRopeHalf = 32;           // rotated pairs per vector (rope_dims <= 64)
}

template <int NQ>
struct IndexTcCfg {
  static constexpr int N = 4 * NQ;                         // MMA N = queries x 4 heads
  static constexpr int kEpiWarps = NQ >= 16 ? 8 : 4;       // 2 per TMEM lane quadrant for 16+ queries
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kThreads = 64 + kEpiThreads;
  static constexpr int kColsPerWarp = N / (kEpiWarps / 4);  // 64 (16 queries) or 16 (4 queries)
  static constexpr int kStages = NQ >= 64 ? 4 : 6;
  static constexpr int kABytes = 128 * 128 * 2;            // one k^ tile, idx_dim 128
  static constexpr int kBBytes = N * 128 * 2;              // rotated queries, 2 slabs
  static constexpr int kOffB = kStages * kABytes;
  static constexpr int kOffW = kOffB + kBBytes;            // w[NQ][4] fp32
  static constexpr int kOffCS = kOffW + ((NQ * 16 + 1023) / 1024) * 1024;   // cos/sin[NQ][half]
  static constexpr int kOffTau = kOffCS + ((NQ * tc_index::kMaxRopeHalf * 8 + 1023) / 1024) * 1024;   // float[NQ]
  static constexpr int kOffBar = kOffTau + ((NQ * 4 + 1023) / 1024) * 1024;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 2 * N < 32 ? 32 : 2 * N;
  static constexpr uint32_t kIdesc = sm100::idesc_bf16(128, N, false, false);
  static constexpr int kRotTasks = (N * 16 + kEpiThreads - 1) / kEpiThreads;   // 16-byte chunks per thread
};

struct IndexTcArgs {
  const __nv_bfloat16* q_idx;   // [T][4][DI]
  const float* w;               // [T][4]
  float* scores;                // [T][ld] (score mode)
  int64_t ld;
  int stride;                   // pooled blocks per scored row: 1, or the sample stride
  // filter mode (tau != null): instead of writing scores, the (score, block)
  // pairs of every candidate with score >= tau[token] are appended to the
  // token's list; cand_cnt counts them all (entries past cand_cap are
  // dropped, and the count tells the selection so)
  const float* tau;             // [T]; -inf keeps every candidate, NaN none
  float* cand_score;            // [T][cand_cap]
  int32_t* cand_idx;            // [T][cand_cap]
  int32_t* cand_cnt;            // [T], zero on entry
  int cand_cap;
  // queries already rotated (q_idx holds q~ rows): the query tile skips the
  // rotation; row_map (or null): score row of query row i is row_map[i]
  int prerotated;
  const int32_t* row_map;
};

struct IndexTcCtl {
  uint64_t a_full[8];
  uint64_t a_empty[8];
  uint64_t b_ready;
  uint64_t acc_full[2];
  uint64_t acc_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// sum_{i=0}^{n-1} floor((a*i + b) / m) for n >= 0, m >= 1, a >= 0, b >= 0.
// Each round strips the integer parts of a/m and b/m, then counts the
// lattice points under the line the other way round:
//   S(n, m, a, b) = K*n - S(K, a, m, m - b + a - 1),  K = floor((a(n-1) + b)/m),
// whose (m, a) pair shrinks like Euclid's algorithm.
__host__ __device__ inline int64_t floor_sum(int64_t n, int64_t m, int64_t a, int64_t b) {
  int64_t total = 0, sign = 1;
  while (n > 0) {
    if (a >= m) {
      total += sign * (a / m) * (n * (n - 1) / 2);
      a %= m;
    }
    if (b >= m) {
      total += sign * (b / m) * n;
      b %= m;
    }
    const int64_t K = (a * (n - 1) + b) / m;
    if (K == 0) break;
    total += sign * K * n;
    sign = -sign;
    const int64_t nb = m - b + a - 1;
    n = K;
    const int64_t nm = a;
    a = m;
    m = nm;
    b = nb;
  }
  return total;
}

// k^ tiles scored by query tile qt of a segment (the blocks its last query
// scores, floor(t_last / r), in tiles of 128 scored rows; with stride s a row
// is every s-th block, so a tile spans 128 s blocks).
// The segment's scored blocks are [blk_lo, limit): tiles start at tile
// floor(blk_lo / 128 s); limit = blk_cap when > 0, else the causal limit
// (every query of a capped segment scores the same blocks).  First blocks
// past 0 and caps are for the decode-like tiles (NQ < 64) only.
template <int NQ>
__host__ __device__ inline int index_qtile_tiles(int64_t pos0, int q_len, int qt, int r, int stride, int blk_lo = 0,
                                                 int blk_cap = 0) {
  const int64_t P = (int64_t)tc_index::kTileRows * stride;
  const int64_t t_last = pos0 + (int64_t)min(NQ * (qt + 1), q_len) - 1;
  const int64_t n = cdiv(blk_cap > 0 ? (int64_t)blk_cap : t_last / r, P) - blk_lo / P;
  return n > 0 ? (int)n : 0;
}

// Balancing weight of a query tile's prologue (building its rotated B tile),
// in k^ tiles: the slices are equal in k^ tiles + kPrologueUnits per query
// tile, so CTAs whose slice crosses many short early query tiles of a
// prefill get fewer k^ tiles.
template <int NQ>
constexpr int index_prologue_units() { return NQ >= 64 ? 6 : 2; }

// Work units (k^ tiles plus prologue weights) of the full query tiles
// 0..J-1 of a segment, where with P = 128 s blocks per tile the k^ tiles of
// full query tile j are
//   ceil(floor((pos0 + NQ j + NQ - 1) / r) / P) = floor((pos0 + NQ - 1 + (P-1) r + NQ j) / (P r)).
// With a first block, every full query tile has floor(blk_lo / P) tiles
// fewer (its causal limit is at least blk_lo: its queries lie past the
// blocks it skips); with a cap, every query tile has the same count.
template <int NQ>
__host__ __device__ inline int64_t index_units_before(int64_t pos0, int J, int r, int stride, int blk_lo = 0,
                                                      int blk_cap = 0) {
  const int64_t P = (int64_t)tc_index::kTileRows * stride;
  const int64_t W = index_prologue_units<NQ>();
  if (blk_cap > 0) return (int64_t)J * (index_qtile_tiles<NQ>(pos0, NQ, 0, r, stride, blk_lo, blk_cap) + W);
  return floor_sum(J, P * r, NQ, pos0 + NQ - 1 + (P - 1) * r) - (int64_t)(blk_lo / P) * J + W * J;
}

// All work units of a segment.
template <int NQ>
inline int64_t index_tc_units(int q_len, int64_t pos0, int r, int stride = 1, int blk_lo = 0, int blk_cap = 0) {
  if (q_len <= 0) return 0;
  const int nqt = (int)cdiv(q_len, NQ);
  return index_units_before<NQ>(pos0, nqt - 1, r, stride, blk_lo, blk_cap) + index_prologue_units<NQ>() +
         index_qtile_tiles<NQ>(pos0, q_len, nqt - 1, r, stride, blk_lo, blk_cap);
}

// Position in the flat sequence of work units: per segment, per query tile,
// kPrologueUnits weights then one unit per k^ tile.  A CTA processes the k^
// tiles whose units fall in its slice.
struct IndexCursor {
  int si, qt, tile, nt;
  int64_t left;        // units left in this CTA's slice, the current tile included
};

// Moves to the next query tile that has k^ tiles (consuming its prologue
// weight) while the current one is exhausted.
template <int NQ>
__device__ __forceinline__ void index_skip(const Geo& g, const SegTable& st, int stride, IndexCursor& c) {
  while (c.left > 0 && c.tile >= c.nt) {
    c.tile = 0;
    if (++c.qt >= (int)cdiv(st.q_len[c.si], NQ)) {
      c.qt = 0;
      ++c.si;
    }
    c.nt = index_qtile_tiles<NQ>(st.pos0[c.si], st.q_len[c.si], c.qt, g.r, stride, st.blk_lo[c.si],
                                 st.blk_cap[c.si]);
    c.left -= index_prologue_units<NQ>();
  }
}

template <int NQ>
__device__ __forceinline__ void index_seek(const Geo& g, const SegTable& st, int stride, int64_t L, int64_t R,
                                           IndexCursor& c) {
  constexpr int W = index_prologue_units<NQ>();
  c.left = R - L;
  if (c.left <= 0) return;
  c.si = find_segment(st, (int)L);
  const int64_t local = L - st.item0[c.si];
  const int64_t pos0 = st.pos0[c.si];
  const int nqt = (int)cdiv(st.q_len[c.si], NQ);
  const int blo = st.blk_lo[c.si], bcap = st.blk_cap[c.si];
  int lo = 0, hi = nqt - 1;                       // largest J with units_before(J) <= local
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (index_units_before<NQ>(pos0, mid, g.r, stride, blo, bcap) <= local) lo = mid; else hi = mid - 1;
  }
  c.qt = lo;
  const int64_t o = local - index_units_before<NQ>(pos0, lo, g.r, stride, blo, bcap);
  c.nt = index_qtile_tiles<NQ>(pos0, st.q_len[c.si], lo, g.r, stride, blo, bcap);
  if (o < W) {                                    // the slice starts inside the prologue weight
    c.left -= W - o;
    c.tile = 0;
  } else {
    c.tile = (int)(o - W);
  }
  index_skip<NQ>(g, st, stride, c);
}

template <int NQ>
__device__ __forceinline__ void index_advance(const Geo& g, const SegTable& st, int stride, IndexCursor& c) {
  --c.left;
  ++c.tile;
  index_skip<NQ>(g, st, stride, c);
}

template <int NQ>
__global__ void __launch_bounds__(IndexTcCfg<NQ>::kThreads, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap tm_khat, Geo g, SegTable st, IndexTcArgs a) {
  using namespace tc_index;
  using namespace sm100;
  using C = IndexTcCfg<NQ>;
  extern __shared__ unsigned char smem_raw[];
  // 1 KiB-aligned base, offset from the shared array itself so that accesses
  // through it stay shared-memory accesses (not generic ones)
  unsigned char* smem = smem_raw + ((1024u - (sm100::smem_u32(smem_raw) & 1023u)) & 1023u);
  IndexTcCtl& ctl = *reinterpret_cast<IndexTcCtl*>(smem + C::kOffBar);
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t total = st.item0[st.n];
  const int64_t L = total * blockIdx.x / gridDim.x, R = total * (blockIdx.x + 1) / gridDim.x;
  if (L >= R) return;                                          // uniform across the CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&ctl.a_full[i], 1);
      mbar_init(&ctl.a_empty[i], 1);
    }
    mbar_init(&ctl.b_ready, C::kEpiWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.acc_full[i], 1);
      mbar_init(&ctl.acc_free[i], C::kEpiWarps);
    }
    mbar_init(&ctl.mma_done, 1);
    ctl.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_khat);
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const uint32_t smem_base = smem_u32(smem);
  pdl_wait();                                   // the previous kernel's results are visible from here
  pdl_trigger();

  IndexCursor cur;
  index_seek<NQ>(g, st, a.stride, L, R, cur);

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      for (int i = 0; cur.left > 0; ++i, index_advance<NQ>(g, st, a.stride, cur)) {
        const int s = i % C::kStages;
        if (!mbar_wait(&ctl.a_empty[s], (uint32_t)(((i / C::kStages) & 1) ^ 1), abort_flag)) break;
        mbar_expect_tx(&ctl.a_full[s], (uint32_t)(kTileRows * g.DI * 2));
        // tensor map [slot][scored row][dim]: rows past the slot's last read as zero
        const int64_t lo_tile = NQ < 64 ? (int64_t)st.blk_lo[cur.si] / ((int64_t)kTileRows * a.stride) : 0;
        const int32_t y = (int32_t)((lo_tile + cur.tile) * kTileRows);
        for (int slab = 0; slab < g.DI / 64; ++slab)
          tma_load_3d(smem + s * C::kABytes + slab * 16384, &tm_khat, 64 * slab, y, st.slot[cur.si], &ctl.a_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int nqt_seen = 0;
      for (int i = 0; ok && cur.left > 0; ++i, index_advance<NQ>(g, st, a.stride, cur)) {
        if (i == 0 || cur.tile == 0) {                 // a new rotated query tile in B
          if (!(ok = mbar_wait(&ctl.b_ready, (uint32_t)(nqt_seen & 1), abort_flag))) break;
          ++nqt_seen;
        }
        const int s = i % C::kStages, ab = i & 1;
        if (!(ok = mbar_wait(&ctl.acc_free[ab], (uint32_t)(((i >> 1) & 1) ^ 1), abort_flag))) break;
        if (!(ok = mbar_wait(&ctl.a_full[s], (uint32_t)((i / C::kStages) & 1), abort_flag))) break;
        tc_fence_after();
        const uint32_t a_addr = smem_base + s * C::kABytes;
        const uint32_t b_addr = smem_base + C::kOffB;
        const int ksteps = g.DI / 16;
        for (int kk = 0; kk < ksteps; ++kk) {
          const int slab = kk >> 2, sub = kk & 3;
          const uint64_t da = desc_sw128(a_addr + slab * 16384 + sub * 32, 16, 1024);
          const uint64_t db = desc_sw128(b_addr + slab * (C::N * 128) + sub * 32, 16, 1024);
          umma_bf16(tmem + ab * C::N, da, db, C::kIdesc, kk != 0);
        }
        umma_commit(&ctl.a_empty[s]);
        umma_commit(&ctl.acc_full[ab]);
      }
      umma_commit(&ctl.mma_done);
      volatile int never = 0;
      mbar_wait(&ctl.mma_done, 0, &never);
    }
    __syncwarp();
  } else {
    // ============================================================ q~ tiles and epilogue
    const int et = threadIdx.x - 64;                // 0 .. kEpiThreads-1
    const int DI = g.DI, half = g.rope_half;
    const int chunks = DI / 8;                      // 16-byte chunks per q~ row
    float* ws = reinterpret_cast<float*>(smem + C::kOffW);
    float2* cs = reinterpret_cast<float2*>(smem + C::kOffCS);
    float* taus = reinterpret_cast<float*>(smem + C::kOffTau);
    const int quad = warp & 3;
    const int cq = (warp - 2) >> 2;                 // column share within the quadrant
    constexpr int kCols = C::kColsPerWarp;
    constexpr int kQ = kCols / 4;                   // queries per warp share
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(cq * kCols);
    // pairs are whole 16-byte chunks when half is a multiple of 8: the partner
    // chunk then sits hc lanes away in the same warp
    const int hc = (half % 8 == 0) ? half / 8 : -1;

    int64_t tok0 = 0, t_first = 0;
    int nq = 0;
    int blo = 0, row0 = 0;                          // the segment's first scored block, and its tile row
    for (int i = 0; cur.left > 0; ++i, index_advance<NQ>(g, st, a.stride, cur)) {
      if (i == 0 || cur.tile == 0) {
        // ---------------------------------------------- new query tile
        const int q0 = cur.qt * NQ;
        tok0 = st.q_offset[cur.si] + q0;
        t_first = (int64_t)st.pos0[cur.si] + q0;
        nq = min(NQ, st.q_len[cur.si] - q0);
        if constexpr (NQ < 64) {                    // first blocks past 0: decode-like tiles only
          blo = st.blk_lo[cur.si];
          row0 = blo / (kTileRows * a.stride) * kTileRows;
        }
        named_bar_sync(1, C::kEpiThreads);          // every share is done with the previous w, cos/sin
        const bool rotate = !(NQ == 16 && a.prerotated);
        for (int k = et; rotate && k < nq * half; k += C::kEpiThreads) {
          const int q = k / half, p = k - q * half;
          float c, sn;
          rope_cs(g, t_first + q, p, c, sn);
          cs[k] = make_float2(c, sn);
        }
        for (int k = et; k < NQ * 4; k += C::kEpiThreads) ws[k] = (k >> 2) < nq ? a.w[tok0 * 4 + k] : 0.f;
        if (a.tau)
          for (int k = et; k < NQ; k += C::kEpiThreads) taus[k] = k < nq ? a.tau[tok0 + k] : __int_as_float(0x7fffffff);
        else if (NQ == 16 && a.row_map)     // score mode: the tau area holds the score rows
          for (int k = et; k < NQ; k += C::kEpiThreads)
            reinterpret_cast<int32_t*>(taus)[k] = k < nq ? a.row_map[tok0 + k] : 0;
        named_bar_sync(1, C::kEpiThreads);
        // rotated queries: row n = q*4 + h of the B tile (K-major, 128-byte swizzle).
        // The accumulators of the previous query tile were all observed full,
        // so no MMA still reads B.
        uint4 raw[C::kRotTasks];
#pragma unroll
        for (int k = 0; k < C::kRotTasks; ++k) {
          const int task = et + k * C::kEpiThreads;
          const int n = task / chunks, j = task - n * chunks;
          raw[k] = make_uint4(0, 0, 0, 0);
          if (n < C::N && (n >> 2) < nq)
            raw[k] = *reinterpret_cast<const uint4*>(a.q_idx + ((tok0 + (n >> 2)) * 4 + (n & 3)) * (int64_t)DI + 8 * j);
        }
#pragma unroll
        for (int k = 0; k < C::kRotTasks; ++k) {
          const int task = et + k * C::kEpiThreads;
          const int n = task / chunks, j = task - n * chunks;
          const int q = n >> 2;
          uint4 out = raw[k];
          if (NQ == 16 && a.prerotated) {
            // q~ rows as given (the shared-prefix tiles)
          } else if (hc > 0) {
            // partner chunk of a rotated pair: j + hc for first halves, j - hc for second halves
            const int src = j < hc ? lane + hc : (j < 2 * hc ? lane - hc : lane);
            uint4 pr;
            pr.x = __shfl_sync(0xffffffffu, raw[k].x, src);
            pr.y = __shfl_sync(0xffffffffu, raw[k].y, src);
            pr.z = __shfl_sync(0xffffffffu, raw[k].z, src);
            pr.w = __shfl_sync(0xffffffffu, raw[k].w, src);
            if (j < 2 * hc && n < C::N && q < nq) {
              const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw[k]);
              const __nv_bfloat16* y = reinterpret_cast<const __nv_bfloat16*>(&pr);
              __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(&out);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int p = 8 * (j < hc ? j : j - hc) + e;          // pair index
                const float2 t = cs[q * half + p];
                float o0, o1;
                if (j < hc) {
                  rope_pair(__bfloat162float(x[e]), __bfloat162float(y[e]), t.x, t.y, o0, o1);
                  o[e] = __float2bfloat16_rn(o0);
                } else {
                  rope_pair(__bfloat162float(y[e]), __bfloat162float(x[e]), t.x, t.y, o0, o1);
                  o[e] = __float2bfloat16_rn(o1);
                }
              }
            }
          } else if (n < C::N && q < nq && 8 * j < 2 * half) {
            // general pairing: fetch each partner element from the row in global memory
            const __nv_bfloat16* row = a.q_idx + ((tok0 + q) * 4 + (n & 3)) * (int64_t)DI;
            const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw[k]);
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(&out);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int d = 8 * j + e;
              if (d < 2 * half) {
                const int p = d < half ? d : d - half;
                const float2 t = cs[q * half + p];
                float o0, o1;
                rope_pair(__bfloat162float(row[p]), __bfloat162float(row[p + half]), t.x, t.y, o0, o1);
                o[e] = __float2bfloat16_rn(d < half ? o0 : o1);
              } else {
                o[e] = x[e];
              }
            }
          }
          if (n < C::N) {
            const int slab = j >> 3, jc = j & 7;
            const uint32_t addr = C::kOffB + slab * (C::N * 128) + (n >> 3) * 1024 + (n & 7) * 128 + ((jc ^ (n & 7)) << 4);
            *reinterpret_cast<uint4*>(smem + addr) = out;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.b_ready);
      }
      // -------------------------------------------------- epilogue of k^ tile cur.tile
      const int ab = i & 1;
      if (!mbar_wait_sleep(&ctl.acc_full[ab], (uint32_t)((i >> 1) & 1), abort_flag)) continue;
      tc_fence_after();
      float v[kCols];
#pragma unroll
      for (int c0 = 0; c0 < kCols; c0 += 16)
        tmem_ld16(lane_addr + ab * C::N + c0, *reinterpret_cast<float(*)[16]>(v + c0));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.acc_free[ab]);  // values are in registers: the MMA may reuse it

      const int64_t b0 = row0 + (int64_t)cur.tile * kTileRows;   // first scored row of the tile
      const int bl = quad * 32 + lane;                // scored row within the tile
      const int qb = cq * kQ;                         // first query of this share
      const int64_t t0 = t_first + qb;
      const int64_t blk = (b0 + bl) * a.stride;       // the pooled block of this row
      // block blk is a candidate of the query at t iff blk >= blk_lo and
      // (blk + 1) r <= t (lim + qq >= 0); in a capped segment (the 16-query
      // tiles of shared prefixes) iff blk < blk_cap instead
      int64_t lim = t0 - (blk + 1) * g.r;
      bool tile_in = ((b0 + kTileRows - 1) * a.stride + 1) * g.r <= t0;
      if constexpr (NQ < 64) {
        if (blk < blo) lim = -(int64_t)1 << 40;
        tile_in = tile_in && b0 * a.stride >= blo;
      }
      if constexpr (NQ == 16) {
        const int bcap = st.blk_cap[cur.si];
        if (bcap > 0) {
          lim = blk < bcap ? (int64_t)1 << 40 : -(int64_t)1 << 40;
          tile_in = (b0 + kTileRows - 1) * a.stride < bcap;
        }
      }
      const float4* w4 = reinterpret_cast<const float4*>(ws) + qb;
      float sc[kQ];
#pragma unroll
      for (int qq = 0; qq < kQ; ++qq) {
        const float4 wq = w4[qq];
        float s = 0.f;
        s = fmaf(wq.x, fmaxf(v[4 * qq + 0], 0.f), s);
        s = fmaf(wq.y, fmaxf(v[4 * qq + 1], 0.f), s);
        s = fmaf(wq.z, fmaxf(v[4 * qq + 2], 0.f), s);
        s = fmaf(wq.w, fmaxf(v[4 * qq + 3], 0.f), s);
        sc[qq] = s;
      }
      if (a.tau) {
        // filter mode: the warp's hits of query qq form ballot m_qq; lane qq
        // reserves them with one atomic on the query's count (the kQ round
        // trips of a tile overlap), then the hits of each query are stored at
        // consecutive positions
        static_assert(kQ <= 32, "one lane per query of the share");
        const bool full = qb + kQ <= nq && tile_in;
        uint32_t hits = 0, my_m = 0;
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq) {
          const bool pass = sc[qq] >= taus[qb + qq] && (full || (qb + qq < nq && lim + qq >= 0));
          const uint32_t m = __ballot_sync(0xffffffffu, pass);
          hits |= (pass ? 1u : 0u) << qq;
          if (lane == qq) my_m = m;
        }
        int my_base = 0;
        if (my_m) my_base = atomicAdd(&a.cand_cnt[tok0 + qb + lane], __popc(my_m));
        const uint32_t below = (1u << lane) - 1u;
        const int cap = a.cand_cap;
        float* ps = a.cand_score + (tok0 + qb) * (int64_t)cap;
        int32_t* pi = a.cand_idx + (tok0 + qb) * (int64_t)cap;
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq, ps += cap, pi += cap) {
          const uint32_t m = __shfl_sync(0xffffffffu, my_m, qq);
          const int pos = __shfl_sync(0xffffffffu, my_base, qq) + __popc(m & below);
          if (((hits >> qq) & 1u) && pos < cap) {
            ps[pos] = sc[qq];
            pi[pos] = (int32_t)blk;
          }
        }
      } else if (NQ == 16 && a.row_map) {
        const int32_t* rows = reinterpret_cast<const int32_t*>(taus) + qb;
#pragma unroll
        for (int qq = 0; qq < kQ; ++qq)
          if (qb + qq < nq && lim + qq >= 0) a.scores[(int64_t)rows[qq] * a.ld + b0 + bl] = sc[qq];
      } else {
        const int64_t ld = a.ld;
        float* p = a.scores + (tok0 + qb) * ld + b0 + bl;
        if (qb + kQ <= nq && tile_in) {
          // every block of the tile is a candidate of every query of the share
#pragma unroll
          for (int qq = 0; qq < kQ; ++qq, p += ld) *p = sc[qq];
        } else {
#pragma unroll
          for (int qq = 0; qq < kQ; ++qq, p += ld)
            if (qb + qq < nq && lim + qq >= 0) *p = sc[qq];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qsa
