// attn_union_tc.cuh -- sparse GQA attention over the union of neighbouring
// queries' kept blocks (tcgen05 tensor cores, bf16 I/O).
//
// Miles docs "Qwen3.8-Flash-Next", section 1: query t attends only the key
// tokens its selection kept; the result here is that of attn_tc.cuh.  What
// changes is the unit of work.  Neighbouring query tokens whose indexer
// queries are close keep mostly the same blocks, and a per-query gather then
// moves the same K/V rows once per query.  Here a tile of mq consecutive
// query tokens of one segment (mq * hpg <= 128 query rows of one KV group)
// gathers the ascending union of its members' kept blocks once.  A 32-bit
// mask per union block (bit i: member i kept the block) and each member's
// causal limit decide which keys a query row attends; every other key gets
// probability zero.  The design report's QSA item gives the blocks (r = 4
// tokens) and the budget.
//
// Two kernels:
//   union_build_kernel  one CTA per tile: a bitmap of the members' kept
//                       blocks, its popcount prefix, the ascending union
//                       list and the member masks.
//   attn_union_kernel   persistent, one CTA per SM, unit = (tile, KV group):
//       S[row, key] = Q[row, :] . K_chunk[key, :]      (M=128 rows, N=64 keys, K=256)
//       O[row, :]  += P[row, key] . V_chunk[key, :]    (M=128, N=256 dims, K=64 keys)
//     row = member * hpg + head.  A chunk is 16 union blocks (64 keys).
//     Online softmax: a row's reference maximum moves only when a chunk's
//     maximum exceeds it by more than 8 (log2 units); then O and the row sum
//     so far are rescaled in TMEM (softmax is shift invariant and P stays
//     below 2^8 in between).
//
// Roles follow attn_tc.cuh (20 warps, warp w on sub-partition w % 4): nine
// cp.async producers gather the chunks' K and V into a 7-slot ring of 32 KiB
// slots (64 keys x 256 dims, 128-byte swizzled K-major) in the order the
// MMAs consume them (K0, K1, V0, K2, V1, ...); warp 0 issues the MMAs; eight
// softmax warps, two per TMEM lane quadrant, own one query row each (TMEM
// lane) and 32 of a chunk's 64 keys.  Q and P live in tensor memory as the A
// operands of their MMAs (bf16 pairs per 32-bit column): the softmax warps
// write each unit's Q rows there, and P over the first half of its chunk's S
// columns, which leaves shared memory to the K/V ring.  Every mbarrier wait
// is bounded; a timeout records an error and the CTA drains and returns.
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"
#include "attn_tc.cuh"

namespace qsa {
namespace tc_union {
constexpr int kMaxMembers = 32;            // bits of a union mask
constexpr int kBlk = 16;                   // union blocks per chunk
constexpr int kKeys = 64;                  // keys per chunk
constexpr int kSlots = 7;                  // ring slots: one chunk's K or V each
constexpr int kSlotBytes = 32768;          // 64 keys x 256 dims, 4 slabs of 8 KiB
constexpr int kOffBar = kSlots * kSlotBytes;               // 229376
constexpr int kCtlBytes = 1280;
constexpr int kSmemBytes = kOffBar + kCtlBytes + 1024;     // + alignment slack: 231680
constexpr uint32_t kTmemCols = 512;        // S (then P over its first 32): 2 x 64 columns at 0
constexpr uint32_t kTmemQ = 128;           // Q: 128 rows x 256 dims as 128 columns of bf16 pairs
constexpr uint32_t kTmemO = 256;           // O: 256 columns
constexpr uint32_t kIdescS = sm100::idesc_bf16(128, kKeys, false, false);
constexpr uint32_t kIdescPV = sm100::idesc_bf16(128, 256, false, true);
constexpr int kBuildThreads = 256;
}  // namespace tc_union

// Tiles per segment of q_len query tokens.
__host__ __device__ inline int64_t union_tiles(int64_t q_len, int mq) { return (q_len + mq - 1) / mq; }

struct UnionBuildArgs {
  const int32_t* sel;       // [T][S]
  const int32_t* nsel;      // [T]
  int32_t* ulen;            // [tiles]: union length of each tile
  int32_t* ublk;            // [tiles][cap]: ascending union blocks
  uint32_t* umask;          // [tiles][cap]: member bits of each union block
  int64_t cap;              // entries per tile = mq * S
  int64_t tile_base;        // global number of this table's first tile
  int mq;                   // query tokens per tile
  int words;                // bitmap words held in shared memory
};

struct TileInfo {
  int64_t tok0;             // first member's token row
  int64_t t0;               // first member's position
  int nq;                   // members (<= mq)
  int64_t slot;
};

__device__ __forceinline__ TileInfo union_tile(const SegTable& st, int64_t tile, int mq) {
  TileInfo ti;
  const int si = find_segment(st, (int)tile);
  const int64_t q0 = (tile - st.item0[si]) * (int64_t)mq;
  ti.nq = (int)min((int64_t)mq, (int64_t)st.q_len[si] - q0);
  ti.tok0 = st.q_offset[si] + q0;
  ti.t0 = st.pos0[si] + q0;
  ti.slot = st.slot[si];
  return ti;
}

// One CTA per tile.  Blocks beyond the last member's own block, and entries
// the per-query path would reject, are left out (no member attends them).
__global__ void __launch_bounds__(tc_union::kBuildThreads)
    union_build_kernel(Geo g, SegTable st, UnionBuildArgs a) {
  using namespace tc_union;
  extern __shared__ uint32_t ush[];
  uint32_t* bits = ush;                         // [words] bitmap of kept blocks
  uint32_t* pre = ush + a.words;                // [words] union entries before word w
  uint32_t* msk = pre + a.words;                // [cap] member masks
  __shared__ uint32_t warp_tot[kBuildThreads / 32];
  __shared__ uint32_t total;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const TileInfo ti = union_tile(st, blockIdx.x, a.mq);
  const int64_t tlast = ti.t0 + ti.nq - 1;
  const int64_t nb = tlast / g.r + 1;                       // blocks 0..own block of the last member
  const int W = (int)((nb + 31) / 32);                      // <= a.words (host sizes it)
  for (int i = tid; i < W; i += blockDim.x) bits[i] = 0;
  for (int64_t i = tid; i < a.cap; i += blockDim.x) msk[i] = 0;
  __syncthreads();
  auto member_block = [&](int i, int j, int32_t& b) -> bool {
    b = a.sel[(ti.tok0 + i) * g.S + j];
    return block_row(b, 0, g) >= 0 && (int64_t)b < nb;
  };
  for (int i = 0; i < ti.nq; ++i) {
    const int n = min(max(a.nsel[ti.tok0 + i], 0), g.S);
    for (int j = tid; j < n; j += blockDim.x) {
      int32_t b;
      if (member_block(i, j, b)) atomicOr(&bits[b >> 5], 1u << (b & 31));
    }
  }
  __syncthreads();
  // exclusive popcount prefix: each thread a contiguous run of words
  const int per = (W + (int)blockDim.x - 1) / (int)blockDim.x;
  const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
  uint32_t cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
  uint32_t inc = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += v;
  }
  if (lane == 31) warp_tot[wid] = inc;
  __syncthreads();
  if (tid == 0) {
    uint32_t acc = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
      const uint32_t v = warp_tot[k];
      warp_tot[k] = acc;
      acc += v;
    }
    total = acc;
  }
  __syncthreads();
  uint32_t base = warp_tot[wid] + inc - cnt;
  int32_t* out = a.ublk + (a.tile_base + blockIdx.x) * a.cap;
  for (int w = w0; w < w1; ++w) {
    pre[w] = base;
    uint32_t x = bits[w];
    while (x) {
      const int bit = __ffs(x) - 1;
      out[base++] = w * 32 + bit;
      x &= x - 1;
    }
  }
  __syncthreads();
  for (int i = 0; i < ti.nq; ++i) {
    const int n = min(max(a.nsel[ti.tok0 + i], 0), g.S);
    for (int j = tid; j < n; j += blockDim.x) {
      int32_t b;
      if (member_block(i, j, b)) {
        const uint32_t idx = pre[b >> 5] + __popc(bits[b >> 5] & ((1u << (b & 31)) - 1u));
        atomicOr(&msk[idx], 1u << i);
      }
    }
  }
  __syncthreads();
  uint32_t* mout = a.umask + (a.tile_base + blockIdx.x) * a.cap;
  for (uint32_t k = tid; k < total; k += blockDim.x) mout[k] = msk[k];
  if (tid == 0) a.ulen[a.tile_base + blockIdx.x] = (int32_t)total;
}

struct AttnUnionArgs {
  const void* q;            // bf16 [T][H][D]
  const void* k;            // bf16 [n_slots][G][n_cap][D]
  const void* v;
  const int32_t* ulen;
  const int32_t* ublk;
  const uint32_t* umask;
  int64_t cap;
  int64_t tile_base;
  int64_t tiles;            // tiles in this table (units per group)
  int mq;
  void* o;                  // bf16 [T][H][D]
  float* lse;               // [T][H] or null
};

struct AttnUnionCtl {
  uint64_t slot_full[tc_union::kSlots];
  uint64_t slot_empty[tc_union::kSlots];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], p_free[2];   // P of a chunk written / its P.V finished (a rescale of O waits on it)
  uint64_t o_full, o_free;
  uint64_t mma_done;
  float red[128][2];        // a row's partial maximum / sum from each of its two softmax warps
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(AttnUnionCtl) <= tc_union::kCtlBytes, "control block");

// Ring position of chunk c's K (kind 0) or V (kind 1) within a unit of n
// chunks: K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1) -- the order in
// which the MMAs consume them, so slots free in ring order and each V chunk
// arrives one chunk later than with K(c), V(c) adjacent.
__device__ __forceinline__ int union_item(int c, int kind, int n) {
  if (kind == 0) return c == 0 ? 0 : 2 * c - 1;
  return c == n - 1 ? 2 * n - 1 : 2 * c + 2;
}

struct UnionUnit {
  TileInfo ti;
  int64_t tile;             // global tile number
  int grp;
  int len;                  // union length
  int nchunks;
};

__device__ __forceinline__ UnionUnit union_unit(const SegTable& st, const AttnUnionArgs& a, int64_t w) {
  UnionUnit u;
  u.grp = (int)(w / a.tiles);
  const int64_t tl = w - (int64_t)u.grp * a.tiles;
  u.ti = union_tile(st, tl, a.mq);
  u.tile = a.tile_base + tl;
  u.len = (int)min((int64_t)max(a.ulen[u.tile], 0), a.cap);
  u.nchunks = (u.len + tc_union::kBlk - 1) / tc_union::kBlk;
  return u;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = v[i];
    hi[i] = v[8 + i];
  }
  sm100::tmem_st8(taddr, lo);
  sm100::tmem_st8(taddr + 8, hi);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M=128 rows, 16-bit pairs along the
// columns) read from tensor memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u));
}

// 32 lanes x 32-bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// 2^x by the MUFU instruction (inputs here are <= 8 or -inf; results below
// 2^-126 flush to zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warp-uniform wait that suspends lane 0 in the barrier probe (no issue
// slots spent while the phase is open).
__device__ __forceinline__ bool warp_wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = sm100::mbar_wait_sleep(bar, parity, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__global__ void __launch_bounds__(tc_attn::kThreads, 1)
    attn_union_kernel(Geo g, SegTable st, AttnUnionArgs a) {
  using namespace tc_union;
  using namespace sm100;
  using tc_attn::kProducers;
  using tc_attn::kSoftmaxWarps;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  AttnUnionCtl& ctl = *reinterpret_cast<AttnUnionCtl*>(smem + kOffBar);
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = (int64_t)g.G * a.tiles;
  int ridx = 0;
  const tc_attn::Role role = tc_role(warp, ridx);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&ctl.slot_full[i], kProducers * 32);   // one cp.async completion arrival per producer lane
      mbar_init(&ctl.slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.s_free[i], kSoftmaxWarps);
      mbar_init(&ctl.p_full[i], kSoftmaxWarps);
      mbar_init(&ctl.p_free[i], 1);
    }
    mbar_init(&ctl.q_full, kSoftmaxWarps);
    mbar_init(&ctl.q_empty, 1);
    mbar_init(&ctl.o_full, 1);
    mbar_init(&ctl.o_free, kSoftmaxWarps);
    mbar_init(&ctl.mma_done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (role == tc_attn::kRoleMma) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (role == tc_attn::kRoleProducer) {
    // ============================================================ producers
    const int pw = ridx;                         // copies union blocks pw and pw + 9 of each chunk
    int64_t item = 0;                            // ring items issued so far (two per chunk)
    bool ok = true;
    const int r = (lane >> 3) & 3, jc = lane & 7;   // row of a block and 16-byte piece of a 128-byte line
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const UnionUnit u = union_unit(st, a, w);
      if (u.nchunks == 0) continue;
      const size_t kv_off = ((size_t)u.ti.slot * g.G + u.grp) * (size_t)g.n_cap * kHeadDim;
      const __nv_bfloat16* kg = (const __nv_bfloat16*)a.k + kv_off;
      const __nv_bfloat16* vg = (const __nv_bfloat16*)a.v + kv_off;
      const int32_t* ub = a.ublk + u.tile * a.cap;
      const int n = u.nchunks;
      // the chunk and tensor of ring position j (inverse of union_item)
      auto chunk_of = [&](int j) -> int {
        return (j == 0) ? 0 : (j == 2 * n - 1) ? n - 1 : (j & 1) ? (j + 1) / 2 : j / 2 - 1;
      };
      // lane i < 2: cache row of union block pw + 9 i of chunk c (entries checked by the union build)
      auto rows_of = [&](int c) -> int64_t {
        int64_t row = -1;
        if (lane < 2 && pw + kProducers * lane < kBlk) {
          const int pos = c * kBlk + pw + kProducers * lane;
          if (pos < u.len) row = (int64_t)ub[pos] * 4;
        }
        return row;
      };
      // the union entries are prefetched into L1 four ring positions ahead, so
      // that their load does not hold up each position's copies
      auto prefetch_rows = [&](int c) {
        if (lane < 2 && pw + kProducers * lane < kBlk) {
          const int pos = c * kBlk + pw + kProducers * lane;
          if (pos < u.len) asm volatile("prefetch.global.L1 [%0];" ::"l"(ub + pos));
        }
      };
      for (int j = 0; j < 4 && j < 2 * n; ++j) prefetch_rows(chunk_of(j));
      for (int j = 0; j < 2 * n && ok; ++j, ++item) {
        const int kind = (j == 0) ? 0 : (j == 2 * n - 1) ? 1 : (j & 1) ? 0 : 1;
        if (j + 4 < 2 * n) prefetch_rows(chunk_of(j + 4));
        const int64_t myrow = rows_of(chunk_of(j));
        {
          const int slot = (int)(item % kSlots);
          if (!(ok = warp_wait_sleep(&ctl.slot_empty[slot], (uint32_t)(((item / kSlots) & 1) ^ 1), abort_flag)))
            break;
          const __nv_bfloat16* base = kind == 0 ? kg : vg;
          const uint32_t dst0 = smem_u32(smem + slot * kSlotBytes);
#pragma unroll
          for (int bq = 0; bq < 2; ++bq) {
            const int b = pw + kProducers * bq;
            if (b >= kBlk) break;
            const int64_t row = __shfl_sync(0xffffffffu, myrow, bq);
            const int line = 4 * b + r;
            const uint32_t dst = dst0 + line * 128 + ((jc ^ (line & 7)) << 4);
            const __nv_bfloat16* src = base + 8 * jc + (row >= 0 ? (row + r) * kHeadDim : 0);
            const uint32_t nb = row >= 0 ? 16u : 0u;
#pragma unroll
            for (int s = 0; s < 4; ++s) cp_async16(dst + s * 8192, src + 64 * s, nb);   // dims 64 s + 8 jc .. +8
          }
          cp_async_mbar_arrive(&ctl.slot_full[slot]);    // completes once these copies land
        }
      }
    }
    cp_async_wait_all();                         // no copy of this warp outlives the CTA
  } else if (role == tc_attn::kRoleMma) {
    // ============================================================ MMA issuer
    // Per unit: S(0); then S(c), P.V(c-1) for c = 1..n-1; then P.V(n-1).
    int64_t gc = 0, uc = 0;                      // chunks and units so far
    const uint32_t sb = smem_u32(smem);
    bool ok = true;
    auto pv = [&](int64_t x, int cx, int n) -> bool {
      const int pb = (int)(x & 1);
      if (!warp_wait_sleep(&ctl.p_full[pb], (uint32_t)((x >> 1) & 1), abort_flag)) return false;
      if (cx == 0 && !warp_wait_sleep(&ctl.o_free, (uint32_t)((uc & 1) ^ 1), abort_flag)) return false;
      const int64_t it = 2 * gc + union_item(cx, 1, n);
      const int slot = (int)(it % kSlots);
      if (!warp_wait_sleep(&ctl.slot_full[slot], (uint32_t)((it / kSlots) & 1), abort_flag)) return false;
      tc_fence_after();
      if (lane == 0) {
        fence_proxy_async_smem();
        const uint32_t v_addr = sb + slot * kSlotBytes;
        for (int kk = 0; kk < 4; ++kk) {                 // 4 k-steps of 16 keys; P: 8 columns of bf16 pairs each
          const uint64_t db = desc_sw128(v_addr + kk * 2048, 8192, 1024);
          umma_bf16_ts(tmem + kTmemO, tmem + pb * kKeys + kk * 8, db, kIdescPV, (cx | kk) != 0);
        }
        umma_commit(&ctl.slot_empty[slot]);
        umma_commit(&ctl.p_free[pb]);
        if (cx == n - 1) umma_commit(&ctl.o_full);
      }
      __syncwarp();
      return true;
    };
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const UnionUnit u = union_unit(st, a, w);
      if (u.nchunks == 0) continue;
      if (!(ok = warp_wait_sleep(&ctl.q_full, (uint32_t)(uc & 1), abort_flag))) break;
      const int n = u.nchunks;
      for (int c = 0; c < n && ok; ++c) {
        const int64_t x = gc + c;
        const int b = (int)(x & 1);
        if (!(ok = warp_wait_sleep(&ctl.s_free[b], (uint32_t)(((x >> 1) & 1) ^ 1), abort_flag))) break;
        const int64_t it = 2 * gc + union_item(c, 0, n);
        const int slot = (int)(it % kSlots);
        if (!(ok = warp_wait_sleep(&ctl.slot_full[slot], (uint32_t)((it / kSlots) & 1), abort_flag))) break;
        tc_fence_after();
        if (lane == 0) {
          fence_proxy_async_smem();
          const uint32_t k_addr = sb + slot * kSlotBytes;
          for (int kk = 0; kk < 16; ++kk) {             // 16 k-steps of 16 dims; Q: 8 columns each
            const int slab = kk >> 2, sub = kk & 3;
            const uint64_t db = desc_sw128(k_addr + slab * 8192 + sub * 32, 16, 1024);
            umma_bf16_ts(tmem + b * kKeys, tmem + kTmemQ + kk * 8, db, kIdescS, kk != 0);
          }
          umma_commit(&ctl.slot_empty[slot]);
          umma_commit(&ctl.s_full[b]);
          if (c == u.nchunks - 1) umma_commit(&ctl.q_empty);
        }
        __syncwarp();
        if (c > 0) ok = pv(x - 1, c - 1, n);
      }
      if (!ok) break;
      ok = pv(gc + n - 1, n - 1, n);
      gc += u.nchunks;
      ++uc;
    }
    // every MMA issued above has finished before TMEM is freed
    if (lane == 0) {
      umma_commit(&ctl.mma_done);
      volatile int never = 0;
      mbar_wait(&ctl.mma_done, 0, &never);
    }
    __syncwarp();
  } else if (role == tc_attn::kRoleSoftmax) {
    // ============================================================ softmax + epilogue
    const int quad = warp & 3;                   // TMEM lane quadrant of this warp
    const int half = ridx;                       // keys 32 half .. +31 of a chunk; O dims 128 half .. +127
    const int li = quad * 32 + lane;             // TMEM lane = query row
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t sb = smem_u32(smem);
    const float tau2 = g.scale * 1.4426950408889634f;
    const int qi = li / g.hpg, hh = li - qi * g.hpg;   // member and head of this row
    int64_t gc = 0, uc = 0;
    // No early exit: the two warps of a quadrant meet at a named barrier per chunk.
    for (int64_t w = blockIdx.x; w < n_units; w += gridDim.x) {
      const UnionUnit u = union_unit(st, a, w);
      if (u.nchunks == 0) continue;
      const bool active = qi < u.ti.nq;
      const int64_t t = u.ti.t0 + qi;
      const int32_t t4 = (int32_t)(t >> 2);                 // own block (r = 4)
      const uint32_t own_rows = (2u << (uint32_t)(t & 3)) - 1u;
      const int32_t* ub = a.ublk + u.tile * a.cap;
      const uint32_t* um = a.umask + u.tile * a.cap;
      // this unit's Q rows into TMEM, the A operand of S (bf16 pairs as they
      // lie in memory): row li = member qi, head hh; this thread dims
      // 128 half .. +127; rows of no member are zero.  The previous unit's
      // last S products have finished first.
      mbar_wait_sleep(&ctl.q_empty, (uint32_t)((uc & 1) ^ 1), abort_flag);
      {
        const uint4* qrow = reinterpret_cast<const uint4*>(
            (const __nv_bfloat16*)a.q + ((u.ti.tok0 + qi) * g.H + (int64_t)u.grp * g.hpg + hh) * kHeadDim + half * 128);
        tc_fence_after();
#pragma unroll
        for (int piece = 0; piece < 4; ++piece) {
          uint4 x[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) x[j] = active ? qrow[piece * 4 + j] : make_uint4(0, 0, 0, 0);
          const uint32_t v[16] = {x[0].x, x[0].y, x[0].z, x[0].w, x[1].x, x[1].y, x[1].z, x[1].w,
                                  x[2].x, x[2].y, x[2].z, x[2].w, x[3].x, x[3].y, x[3].z, x[3].w};
          tmem_st16u(lane_addr + kTmemQ + half * 64 + piece * 16, v);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.q_full);
      }
      float m = -INFINITY, l = 0.f;
      // this thread's 8 union entries of a chunk (blocks and member masks),
      // loaded one chunk ahead: entries c*16 + 8 half .. +7 (inside the
      // tile's lists, as nchunks*16 <= cap; entries past len are ignored)
      uint4 nb0, nb1, nm0, nm1;
      auto fetch = [&](int c) {
        const int pos0 = c * kBlk + half * 8;
        nb0 = *reinterpret_cast<const uint4*>(ub + pos0);
        nb1 = *reinterpret_cast<const uint4*>(ub + pos0 + 4);
        nm0 = *reinterpret_cast<const uint4*>(um + pos0);
        nm1 = *reinterpret_cast<const uint4*>(um + pos0 + 4);
      };
      fetch(0);
      for (int c = 0; c < u.nchunks; ++c, ++gc) {
        const int b = (int)(gc & 1);
        // whether this thread's row attends each key of its 8 union blocks
        // (a member keeps no block past its own block t4; of that one, rows 0..t%4)
        uint32_t vbits = 0;
        {
          const uint32_t bk[8] = {nb0.x, nb0.y, nb0.z, nb0.w, nb1.x, nb1.y, nb1.z, nb1.w};
          const uint32_t mk[8] = {nm0.x, nm0.y, nm0.z, nm0.w, nm1.x, nm1.y, nm1.z, nm1.w};
          const int pos0 = c * kBlk + half * 8;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (active && pos0 + k < u.len && ((mk[k] >> qi) & 1u)) {
              const int32_t bb = (int32_t)bk[k];
              const uint32_t rows = bb < t4 ? 0xFu : (bb == t4 ? own_rows : 0u);
              vbits |= rows << (4 * k);
            }
          }
        }
        if (c + 1 < u.nchunks) fetch(c + 1);
        mbar_wait_sleep(&ctl.s_full[b], (uint32_t)((gc >> 1) & 1), abort_flag);
        tc_fence_after();
        float s[32];                             // raw scores; keys this row does not attend: -inf
        {
          float s0[16], s1[16];
          tmem_ld16(lane_addr + b * kKeys + half * 32, s0);
          tmem_ld16(lane_addr + b * kKeys + half * 32 + 16, s1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            s[i] = ((vbits >> i) & 1u) ? s0[i] : -INFINITY;
            s[16 + i] = ((vbits >> (16 + i)) & 1u) ? s1[i] : -INFINITY;
          }
        }
        float pm = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) pm = fmaxf(pm, s[i]);
        ctl.red[li][half] = pm * tau2;
        named_bar_sync(1 + quad, 64);
        const float mc = fmaxf(ctl.red[li][0], ctl.red[li][1]);
        named_bar_sync(1 + quad, 64);            // both read before the next chunk writes
        float f = 1.f;
        bool need = false;
        if (mc > m + 8.f) {                      // false while both are -inf
          if (m != -INFINITY) {
            f = exp2f(m - mc);
            need = true;
          }
          m = mc;
        }
        l *= f;
        if (__any_sync(0xffffffffu, need)) {
          // O holds chunks 0..c-1 (c >= 1 here): wait for the last of their P.V products
          const int64_t xp = gc - 1;
          mbar_wait_sleep(&ctl.p_free[xp & 1], (uint32_t)((xp >> 1) & 1), abort_flag);
          tc_fence_after();
#pragma unroll 1
          for (int piece = 0; piece < 8; ++piece) {
            float o[16];
            const uint32_t addr = lane_addr + kTmemO + half * 128 + piece * 16;
            tmem_ld16(addr, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] *= f;
            tmem_st16(addr, o);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        // P = 2^(tau2 s - m): -inf scores give 0; a row with no attended key yet keeps m = -inf
        const float mb = m == -INFINITY ? 0.f : m;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(s[2 * i], tau2, -mb));
          const float p1 = ex2_approx(fmaf(s[2 * i + 1], tau2, -mb));
          l += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        // P over the first 32 of this chunk's 64 S columns: both warps of the
        // row have read S (the exchange above), and P.V(c-2), the last reader
        // of these columns, ran before S(c) in the MMA order
        tmem_st16u(lane_addr + b * kKeys + half * 16, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ctl.s_free[b]);
          mbar_arrive(&ctl.p_full[b]);
        }
      }
      // the row's denominator: both warps' partial sums
      ctl.red[li][half] = l;
      named_bar_sync(1 + quad, 64);
      const float lt = ctl.red[li][0] + ctl.red[li][1];
      named_bar_sync(1 + quad, 64);
      mbar_wait_sleep(&ctl.o_full, (uint32_t)(uc & 1), abort_flag);
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      __nv_bfloat16* orow = (__nv_bfloat16*)a.o +
                            ((u.ti.tok0 + qi) * g.H + (int64_t)u.grp * g.hpg + hh) * kHeadDim + half * 128;
#pragma unroll 1
      for (int piece = 0; piece < 8; ++piece) {
        float o[16];
        tmem_ld16(lane_addr + kTmemO + half * 128 + piece * 16, o);
        tmem_wait_ld();
        if (active) {
          uint4 v0, v1;
          v0.x = pack_bf16x2(o[0] * inv, o[1] * inv);
          v0.y = pack_bf16x2(o[2] * inv, o[3] * inv);
          v0.z = pack_bf16x2(o[4] * inv, o[5] * inv);
          v0.w = pack_bf16x2(o[6] * inv, o[7] * inv);
          v1.x = pack_bf16x2(o[8] * inv, o[9] * inv);
          v1.y = pack_bf16x2(o[10] * inv, o[11] * inv);
          v1.z = pack_bf16x2(o[12] * inv, o[13] * inv);
          v1.w = pack_bf16x2(o[14] * inv, o[15] * inv);
          *reinterpret_cast<uint4*>(orow + piece * 16) = v0;
          *reinterpret_cast<uint4*>(orow + piece * 16 + 8) = v1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.o_free);
      ++uc;
      if (active && half == 0 && a.lse)
        a.lse[(u.ti.tok0 + qi) * g.H + (int64_t)u.grp * g.hpg + hh] = (m + log2f(lt)) * 0.6931471805599453f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (role == tc_attn::kRoleMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace qsa
