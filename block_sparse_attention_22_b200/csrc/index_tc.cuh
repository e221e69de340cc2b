// index_tc.cuh -- indexer scores on tcgen05 tensor cores (bf16 I/O).
//
// Design report summary page ("Qwen3.8-Next architecture design report"),
// QSA item: a 4-head MQA indexer scores every causal micro-block; scoring
// costs O(n^2/r).  With s(t,b) = sum_h w[t,h] * ReLU(q~[t,h] . k^[b]) this is
// a dense contraction of pooled keys against rotated queries:
//   ACC[b, (q,h)] = k^[b, :] . q~[q, h, :]      M = 128 blocks, N = 4*NQ, K = idx_dim
// followed by a per-block epilogue s = sum_h w[q,h] * max(ACC, 0).
//
// A work item is (segment, tile of NQ consecutive query tokens, range of up to
// KT 128-block tiles).  NQ = 64 for prefill (N = 256; TMEM holds two 128x256
// fp32 accumulators), NQ = 4 for decode (N = 16; the kernel then streams the
// sequence's k^ at HBM rate).  Roles (10 warps, one CTA per SM):
//   warp 0      TMA producer: k^ tiles (128 rows x idx_dim, two 16 KiB boxes
//               for idx_dim 128) into a 4-stage ring;
//   warp 1      TMEM owner and single-thread MMA issuer;
//   warps 2..9  q~ = RoPE_t(q_idx) rounded to bf16, written once per item into
//               the swizzled B tile (fp32 arithmetic in the same fixed order
//               as the key pooling), then the epilogue: warp pair per TMEM lane
//               quadrant, each thread owns one block row and half of the
//               columns, and writes scores[t][b] for b < floor(t/r) as
//               coalesced 128-byte rows.
// Every mbarrier wait is bounded.
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"

namespace qsa {
namespace tc_index {
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kStages = 4;
constexpr int kTileRows = 128;             // k^ blocks per tile (MMA M)
constexpr int kMaxRopeHalf = 32;           // rotated pairs per vector (rope_dims <= 64)
}

template <int NQ>
struct IndexTcCfg {
  static constexpr int N = 4 * NQ;                         // MMA N = queries x 4 heads
  static constexpr int kKT = NQ >= 64 ? 16 : 64;           // tiles per work item
  static constexpr int kABytes = 128 * 128 * 2;            // one k^ tile, idx_dim 128
  static constexpr int kBBytes = N * 128 * 2;              // rotated queries, 2 slabs
  static constexpr int kOffB = tc_index::kStages * kABytes;
  static constexpr int kOffW = kOffB + kBBytes;            // w[NQ][4] fp32
  static constexpr int kOffLim = kOffW + NQ * 16;          // floor(t/r) per query (int64)
  static constexpr int kOffCS = kOffW + ((NQ * 24 + 1023) / 1024) * 1024;   // cos/sin[NQ][half][2]
  static constexpr int kOffBar = kOffCS + ((NQ * tc_index::kMaxRopeHalf * 8 + 1023) / 1024) * 1024;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 2 * N < 32 ? 32 : 2 * N;
  static constexpr uint32_t kIdesc = sm100::idesc_bf16(128, N, false, false);
};

struct IndexTcArgs {
  const __nv_bfloat16* q_idx;   // [T][4][DI]
  const float* w;               // [T][4]
  float* scores;                // [T][ld]
  int64_t ld;
};

struct IndexTcCtl {
  uint64_t a_full[tc_index::kStages];
  uint64_t a_empty[tc_index::kStages];
  uint64_t b_ready;
  uint64_t acc_full[2];
  uint64_t acc_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

// Item geometry shared by every role.
struct IndexItem {
  int si;
  int q0, nq;          // query tile within the segment
  int64_t pos0;        // position of the segment's first query
  int64_t tok0;        // token row of the tile's first query
  int64_t t_first, t_last;
  int tile0, ntiles;   // 128-block tiles [tile0, tile0+ntiles)
};

template <int NQ>
__device__ __forceinline__ bool index_item(const Geo& g, const SegTable& st, int item, IndexItem& it) {
  using C = IndexTcCfg<NQ>;
  it.si = find_segment(st, item);
  const int local = item - st.item0[it.si];
  const int q_len = st.q_len[it.si];
  it.pos0 = st.pos0[it.si];
  const int64_t nb_max = (it.pos0 + q_len - 1) / g.r;
  const int max_chunks = (int)cdiv(cdiv(nb_max, tc_index::kTileRows), C::kKT);
  if (max_chunks == 0) return false;
  const int qt = local / max_chunks, ch = local - qt * max_chunks;
  it.q0 = qt * NQ;
  it.nq = min(NQ, q_len - it.q0);
  it.tok0 = st.q_offset[it.si] + it.q0;
  it.t_first = it.pos0 + it.q0;
  it.t_last = it.t_first + it.nq - 1;
  const int64_t nb = it.t_last / g.r;                       // blocks the tile's last query scores
  const int nt = (int)cdiv(nb, tc_index::kTileRows);
  it.tile0 = ch * C::kKT;
  it.ntiles = min(C::kKT, nt - it.tile0);
  return it.ntiles > 0;
}

template <int NQ>
__global__ void __launch_bounds__(tc_index::kThreads, 1)
    index_tc_kernel(const __grid_constant__ CUtensorMap tm_khat, Geo g, SegTable st, IndexTcArgs a) {
  using namespace tc_index;
  using namespace sm100;
  using C = IndexTcCfg<NQ>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  IndexTcCtl& ctl = *reinterpret_cast<IndexTcCtl*>(smem + C::kOffBar);
  volatile int* abort_flag = &ctl.abort;
  float* ws = reinterpret_cast<float*>(smem + C::kOffW);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  IndexItem it;
  if (!index_item<NQ>(g, st, blockIdx.x, it)) return;          // uniform across the CTA
  const int64_t kh_row0 = (int64_t)st.slot[it.si] * (g.n_cap / g.r);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&ctl.a_full[i], 1);
      mbar_init(&ctl.a_empty[i], 1);
    }
    mbar_init(&ctl.b_ready, kEpiWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.acc_full[i], 1);
      mbar_init(&ctl.acc_free[i], kEpiWarps);
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

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      for (int i = 0; i < it.ntiles; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&ctl.a_empty[s], (uint32_t)(((i / kStages) & 1) ^ 1), abort_flag)) break;
        mbar_expect_tx(&ctl.a_full[s], (uint32_t)(kTileRows * g.DI * 2));
        const int32_t y = (int32_t)(kh_row0 + (int64_t)(it.tile0 + i) * kTileRows);
        for (int slab = 0; slab < g.DI / 64; ++slab)
          tma_load_2d(smem + s * C::kABytes + slab * 16384, &tm_khat, 64 * slab, y, &ctl.a_full[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&ctl.b_ready, 0, abort_flag);
      tc_fence_after();
      for (int i = 0; i < it.ntiles && ok; ++i) {
        const int s = i % kStages, ab = i & 1;
        if (!(ok = mbar_wait(&ctl.acc_free[ab], (uint32_t)(((i >> 1) & 1) ^ 1), abort_flag))) break;
        if (!(ok = mbar_wait(&ctl.a_full[s], (uint32_t)((i / kStages) & 1), abort_flag))) break;
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
    // ============================================================ q~ tile, then epilogue
    const int e = warp - 2;                         // 0..7
    const int et = threadIdx.x - 64;                // 0..255
    const int DI = g.DI, half = g.rope_half;
    // cos/sin of every (query position, rotated pair) of the tile, once
    float2* cs = reinterpret_cast<float2*>(smem + C::kOffCS);
    for (int k = et; k < it.nq * half; k += 32 * kEpiWarps) {
      const int q = k / half, i = k - q * half;
      float c, sn;
      rope_cs(g, it.t_first + q, i, c, sn);
      cs[k] = make_float2(c, sn);
    }
    named_bar_sync(1, 32 * kEpiWarps);
    // rotated queries: row n = q*4 + h of the B tile (K-major, 128-byte swizzle)
    for (int n = et; n < C::N; n += 32 * kEpiWarps) {
      const int q = n >> 2, h = n & 3;
      const bool live = q < it.nq;
      const __nv_bfloat16* src = a.q_idx + ((it.tok0 + q) * 4 + h) * (int64_t)DI;
      for (int j = 0; j < DI / 8; ++j) {            // 16-byte chunk j: dims 8j .. 8j+7
        __align__(16) __nv_bfloat16 out[8];
        if (live) {
          const uint4 raw = *reinterpret_cast<const uint4*>(src + 8 * j);
          const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int d = 8 * j + k;
            float v = __bfloat162float(x[k]);
            if (d < 2 * half) {
              const int i = d < half ? d : d - half;
              const float xa = __bfloat162float(src[i]), xb = __bfloat162float(src[i + half]);
              const float2 t = cs[q * half + i];
              float o0, o1;
              rope_pair(xa, xb, t.x, t.y, o0, o1);
              v = d < half ? o0 : o1;
            }
            out[k] = __float2bfloat16_rn(v);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) out[k] = __float2bfloat16_rn(0.f);
        }
        const int slab = j >> 3, jc = j & 7;
        const uint32_t addr = C::kOffB + slab * (C::N * 128) + (n >> 3) * 1024 + (n & 7) * 128 + ((jc ^ (n & 7)) << 4);
        *reinterpret_cast<uint4*>(smem + addr) = *reinterpret_cast<const uint4*>(out);
      }
    }
    for (int i = et; i < NQ * 4; i += 32 * kEpiWarps)
      ws[i] = (i >> 2) < it.nq ? a.w[it.tok0 * 4 + i] : 0.f;
    int64_t* lim = reinterpret_cast<int64_t*>(smem + C::kOffLim);   // blocks each query scores
    for (int q = et; q < NQ; q += 32 * kEpiWarps) lim[q] = q < it.nq ? (it.t_first + q) / g.r : 0;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.b_ready);
    named_bar_sync(1, 32 * kEpiWarps);              // w[] visible to every epilogue thread

    // epilogue: warp pair per lane quadrant; each warp takes half of the columns
    const int quad = warp & 3;
    const int colhalf = e >> 2;                      // 0 or 1
    constexpr int kCols = C::N / 2;                  // columns per warp
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    for (int i = 0; i < it.ntiles; ++i) {
      const int ab = i & 1;
      mbar_wait(&ctl.acc_full[ab], (uint32_t)((i >> 1) & 1), abort_flag);
      tc_fence_after();
      const int64_t b = (int64_t)(it.tile0 + i) * kTileRows + quad * 32 + lane;
      constexpr int kChunk = kCols >= 32 ? 32 : (kCols >= 16 ? 16 : 8);   // TMEM columns per load
      for (int c0 = 0; c0 < kCols; c0 += kChunk) {
        float v[32];
        if constexpr (kChunk == 32) {
          tmem_ld16(lane_addr + ab * C::N + colhalf * kCols + c0, *reinterpret_cast<float(*)[16]>(v));
          tmem_ld16(lane_addr + ab * C::N + colhalf * kCols + c0 + 16, *reinterpret_cast<float(*)[16]>(v + 16));
        } else if constexpr (kChunk == 16) {
          tmem_ld16(lane_addr + ab * C::N + colhalf * kCols + c0, *reinterpret_cast<float(*)[16]>(v));
        } else {
          tmem_ld8(lane_addr + ab * C::N + colhalf * kCols + c0, *reinterpret_cast<float(*)[8]>(v));
        }
        tmem_wait_ld();
#pragma unroll
        for (int qq = 0; qq < kChunk / 4; ++qq) {
          const int q = (colhalf * kCols + c0) / 4 + qq;
          if (q < it.nq && b < lim[q]) {
            float sc = 0.f;
#pragma unroll
            for (int h = 0; h < 4; ++h) sc = fmaf(ws[q * 4 + h], fmaxf(v[qq * 4 + h], 0.f), sc);
            a.scores[(it.tok0 + q) * a.ld + b] = sc;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.acc_free[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int NQ>
inline int64_t index_tc_items(int q_len, int pos0, int r) {
  using C = IndexTcCfg<NQ>;
  if (q_len <= 0) return 0;
  const int64_t nb_max = ((int64_t)pos0 + q_len - 1) / r;
  return cdiv(q_len, NQ) * cdiv(cdiv(nb_max, tc_index::kTileRows), C::kKT);
}

}  // namespace qsa
