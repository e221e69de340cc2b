// attn_tc.cuh -- sparse GQA attention on tcgen05 tensor cores (bf16 I/O).
//
// Miles docs "Qwen3.8-Flash-Next", section 1: attention reads only the kept
// key tokens; 24 heads in 2 query groups, head dim 256.  The heads of a group
// share one selection, so a work unit is (query token, KV group): its hpg<=16
// heads against the group's kept blocks (up to 512 blocks = 2048 keys).
//
// The MMAs are swapped so that the gathered keys fill the 128-row M side:
//   S^T[key, head]  = K_chunk[key, :] . Q[head, :]       (M=128 keys, N=16, K=256)
//   O^T[d, head]   += V_chunk^T[d, key] . P^T[key, head]  (M=128 dims x2, N=16, K=128)
// A chunk is 32 kept blocks (128 keys).  Kept blocks are contiguous 4-row
// runs of the group's K/V cache; each is copied into the 128-byte-swizzled
// K-major layout the MMA reads (8-row atoms are filled by two blocks).
//
// Two-phase softmax per unit: every chunk's S^T goes to its own TMEM buffer
// (16 x 16 columns), the per-head maximum is taken over all of them but the
// last, then P = exp2(S - max) is written chunk by chunk and P.V accumulates
// straight into a TMEM output buffer.  The last chunk's maximum is folded in
// before the third P chunk: it replaces the running one only when it exceeds
// it by more than 8 (log2 units), and then O and the row sums so far are
// rescaled once in TMEM (softmax is shift invariant; P stays below 2^8).  So
// a unit's first P.V products need not wait for its last S.  K slots are
// freed as soon as their MMA has run, V slots as soon as their P is written,
// and the load stream waits on the softmax only between units.  Loads and MMAs walk one
// item sequence, K(0..n-1) then V(0..n-1) per unit; an item is two 32 KiB
// half-slots (128 keys x 128 dims) of a 6-slot ring.
//
// The gather is HBM/L2-bound and scattered (2 KiB per kept block and tensor),
// so it is issued as 16-byte cp.async copies by eight producer warps: on
// B200 a 4-row block only forms 512-byte TMA boxes, and the TMA request rate
// held such gathers near 1 TB/s, while wide cp.async issue reaches the
// memory system's rate.
//
// Roles (20 warps, persistent over work units, one CTA per SM; warp w runs
// on sub-partition w % 4):
//   9 producers  (three on each of sub-partitions 1..3): every half-slot is
//                shared, producer p copying kept blocks p, p+9, p+18, p+27
//                (one 512-byte row quad per instruction); each lane's
//                cp.async completion arrives on the slot's barrier, so
//                producers run ahead as far as the ring allows.  Producer 0
//                also loads each unit's Q tile with TMA.
//   warp 0       TMEM owner and single-thread MMA issuer, alone with two
//                softmax warps on sub-partition 0;
//   8 softmax    softmax and epilogue, two per TMEM lane quadrant: a thread
//                owns TMEM lane i (key i of a chunk for S; dims i and 128+i
//                for O) and 8 of the 16 heads;
//   warps 12, 16 idle.
// Every mbarrier wait is bounded (sm100::mbar_wait); a timeout records an
// error and the CTA's roles drain and return.
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"
#include "attn_simt.cuh"

namespace qsa {
namespace tc_attn {
constexpr int kProducers = 9;              // three on each of sub-partitions 1..3
constexpr int kSoftmaxWarps = 8;           // two per TMEM lane quadrant
constexpr int kWarps = 20;                 // + the MMA warp and two idle warps
constexpr int kThreads = 32 * kWarps;      // 640
enum Role { kRoleProducer, kRoleMma, kRoleSoftmax, kRoleIdle };
constexpr int kKeys = 128;                 // keys per chunk
constexpr int kBlk = 32;                   // blocks per chunk
constexpr int kSlots = 6;                  // 32 KiB K/V half-chunk slots
constexpr int kSlotBytes = 32768;
constexpr int kQBytes = 8192;              // 16 heads x 256 dims, 4 slabs x 2 KiB
constexpr int kPBytes = 4096;              // 16 heads x 128 keys, 2 slabs x 2 KiB
constexpr int kN = 16;                     // heads per MMA tile
constexpr int kHH = 8;                     // heads per softmax thread
constexpr int kOffQ = kSlots * kSlotBytes;                 // 196608
constexpr int kOffP = kOffQ + 2 * kQBytes;                 // 212992
constexpr int kOffBar = kOffP + 2 * kPBytes;               // 221184
constexpr int kSmemBytes = kOffBar + 1024 + 1024;          // + control block + alignment slack
constexpr int kMaxChunks = kMaxBudgetBlocks / 32;   // 16 S buffers
constexpr uint32_t kTmemCols = 512;        // S: 16 x 16 cols at 0; O: 2 x 32 cols at 256
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kIdescS = sm100::idesc_bf16(128, kN, false, false);
constexpr uint32_t kIdescPV = sm100::idesc_bf16(128, kN, true, false);
}

struct AttnTcArgs {
  const void* k;           // bf16 [n_slots][G][n_cap][D]
  const void* v;
  const int32_t* sel;
  const int32_t* nsel;
  void* o;                 // bf16 [T][H][D]
  float* lse;              // [T][H] or null
  float* part_o;           // split partials (n_split > 1)
  float* part_ml;
  int n_split;
  int blocks_per_split;    // multiple of 32
  int64_t units_per_group; // = st.item0[st.n]
};

struct AttnTcCtl {
  uint64_t slot_full[tc_attn::kSlots];
  uint64_t slot_empty[tc_attn::kSlots];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[tc_attn::kMaxChunks], s_free[tc_attn::kMaxChunks];
  uint64_t p_full[2], p_free[2];
  uint64_t o_full[2], o_free[2];
  uint64_t mma_done;
  float red[2][4][16];
  uint32_t tmem_base;
  int abort;
};

struct TcUnit {
  int64_t tok;
  int64_t t;
  int64_t slot;
  int64_t pslot;   // slot of the blocks below pblk (a shared prefix)
  int pblk;
  int grp;
  int split;
  int blk_begin;   // first position in the sel row
  int blk_end;     // one past the last
  int nchunks;
};

// Warp-uniform wait: lane 0 waits, every lane gets its verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = sm100::mbar_wait(bar, parity, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool warp_aborted(volatile int* abort_flag) {
  return __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
}

__device__ __forceinline__ TcUnit tc_unit(const Geo& g, const SegTable& st, const AttnTcArgs& a, int64_t w) {
  TcUnit u;
  u.grp = (int)(w / a.units_per_group);
  const int rem = (int)(w - (int64_t)u.grp * a.units_per_group);
  const int si = find_segment(st, rem);
  const int local = rem - st.item0[si];
  const int j = local / a.n_split;
  u.split = local - j * a.n_split;
  u.tok = st.q_offset[si] + j;
  u.t = (int64_t)st.pos0[si] + j;
  u.slot = st.slot[si];
  u.pslot = st.pslot[si];
  u.pblk = st.pblk[si];
  const int nsel = min(max(a.nsel[u.tok], 0), g.S);
  u.blk_begin = u.split * a.blocks_per_split;
  u.blk_end = min(nsel, u.blk_begin + a.blocks_per_split);
  u.nchunks = u.blk_end > u.blk_begin ? (int)cdiv(u.blk_end - u.blk_begin, tc_attn::kBlk) : 0;
  return u;
}

// Role of warp w.  Warp w runs on sub-partition w % 4 and may access TMEM
// lanes 32 (w % 4) .. +31.  Sub-partition 0 holds the MMA issuer and two
// softmax warps, each other sub-partition three producers and two softmax
// warps: an issuing tcgen05.mma holds its sub-partition for tens of cycles,
// and producers beside it would fall behind the others and hold up every
// shared half-slot.  `idx` is the producer number (0..8) or the softmax
// warp's head half (0, 1).
__device__ __forceinline__ tc_attn::Role tc_role(int w, int& idx) {
  using namespace tc_attn;
  const int q = w & 3, r = w >> 2;
  if (q == 0) {
    if (r == 0) {
      idx = 0;
      return kRoleMma;
    }
    idx = r - 1;
    return r <= 2 ? kRoleSoftmax : kRoleIdle;
  }
  if (r <= 2) {
    idx = (q - 1) * 3 + r;
    return kRoleProducer;
  }
  idx = r - 3;
  return kRoleSoftmax;
}

__global__ void __launch_bounds__(tc_attn::kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, Geo g, SegTable st, AttnTcArgs a) {
  using namespace tc_attn;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  AttnTcCtl& ctl = *reinterpret_cast<AttnTcCtl*>(smem + kOffBar);
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = (int64_t)g.G * a.units_per_group;
  int ridx = 0;
  const Role role = tc_role(warp, ridx);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&ctl.slot_full[i], kProducers * 32);   // one cp.async completion arrival per producer lane
      mbar_init(&ctl.slot_empty[i], 1);
    }
    for (int i = 0; i < kMaxChunks; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.s_free[i], kSoftmaxWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.q_full[i], 1);
      mbar_init(&ctl.q_empty[i], 1);
      mbar_init(&ctl.p_full[i], kSoftmaxWarps);
      mbar_init(&ctl.p_free[i], 1);
      mbar_init(&ctl.o_full[i], 1);
      mbar_init(&ctl.o_free[i], kSoftmaxWarps);
    }
    mbar_init(&ctl.mma_done, 1);
    ctl.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_q);
  }
  // zero both Q tiles: rows hpg..15 are never loaded and must read as zero
  for (int i = threadIdx.x; i < 2 * kQBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (role == kRoleMma) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  pdl_wait();                                   // the previous kernel's results are visible from here
  pdl_trigger();

  if (role == kRoleProducer) {
    // ============================================================ producers
    const int pw = ridx;                         // producer number: copies blocks pw, pw+9, pw+18, pw+27
    int64_t hs_next = 0, uc = 0;                 // half-slots issued so far (shared numbering)
    bool ok = true;
    const int r = (lane >> 3) & 3, jc = lane & 7;   // row of a block and 16-byte chunk of a line
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const TcUnit u = tc_unit(g, st, a, w);
      if (u.nchunks == 0) continue;
      if (pw == 0) {
        const int qb = (int)(uc & 1);
        if (!(ok = warp_wait(&ctl.q_empty[qb], (uint32_t)(((uc >> 1) & 1) ^ 1), abort_flag))) break;
        if (lane == 0) {
          mbar_expect_tx(&ctl.q_full[qb], (uint32_t)(g.hpg * 128 * 4));
          const int32_t qrow = (int32_t)(u.tok * g.H + (int64_t)u.grp * g.hpg);
          for (int s = 0; s < 4; ++s)
            tma_load_2d(smem + kOffQ + qb * kQBytes + s * 2048, &tm_q, 64 * s, qrow, &ctl.q_full[qb]);
        }
        __syncwarp();
      }
      ++uc;
      const __nv_bfloat16* kg = (const __nv_bfloat16*)a.k + (u.slot * g.G + u.grp) * g.n_cap * kHeadDim;
      const __nv_bfloat16* vg = (const __nv_bfloat16*)a.v + (u.slot * g.G + u.grp) * g.n_cap * kHeadDim;
      // rows below a shared prefix's end live in the prefix's slot: their
      // offset from the unit's own base shifts by whole slots
      const int64_t prow_end = (int64_t)u.pblk * g.r;
      const int64_t pshift = (u.pslot - u.slot) * g.G * g.n_cap;
      const int32_t* selrow = a.sel + u.tok * g.S;
      // rows (from the unit's own K/V base) of this warp's kept blocks pw + 9 i
      // of a chunk (lane i < 4); kNoRow for padding and rejected entries
      constexpr int64_t kNoRow = INT64_MIN / 2;
      auto rows_of = [&](int cc) -> int64_t {
        int64_t row = kNoRow;
        if (lane < 4 && cc < u.nchunks && pw + kProducers * lane < kBlk) {
          const int pos = u.blk_begin + cc * kBlk + pw + kProducers * lane;
          if (pos < u.blk_end) {
            const int64_t br = block_row(selrow[pos], 0, g);
            if (br >= 0) row = br < prow_end ? br + pshift : br;
          }
        }
        return row;
      };
      for (int kind = 0; kind < 2 && ok; ++kind) {     // all K chunks, then all V chunks
        for (int c = 0; c < u.nchunks && ok; ++c) {
          const int64_t myrow = rows_of(c);
          const __nv_bfloat16* base = kind == 0 ? kg : vg;
          for (int h = 0; h < 2 && ok; ++h) {
            const int64_t hs = hs_next++;
            const int slot = (int)(hs % kSlots);
            if (!(ok = warp_wait(&ctl.slot_empty[slot], (uint32_t)(((hs / kSlots) & 1) ^ 1), abort_flag))) break;
            const uint32_t dst0 = smem_u32(smem + slot * kSlotBytes);
#pragma unroll
            for (int bq = 0; bq < 4; ++bq) {
              const int b = pw + kProducers * bq;
              if (b >= kBlk) break;
              const int64_t row = __shfl_sync(0xffffffffu, myrow, bq);
              const int line = 4 * b + r;
              const uint32_t dst = dst0 + line * 128 + ((jc ^ (line & 7)) << 4);
              const __nv_bfloat16* src = base + 128 * h + 8 * jc + (row != kNoRow ? (row + r) * kHeadDim : 0);
              const uint32_t nb = row != kNoRow ? 16u : 0u;
              cp_async16(dst, src, nb);                       // dims 128h + 8jc .. +8
              cp_async16(dst + 16384, src + 64, nb);          // dims 128h + 64 + 8jc .. +8
            }
            cp_async_mbar_arrive(&ctl.slot_full[slot]);    // completes once these copies land
          }
        }
      }
    }
    cp_async_wait_all();                         // no copy of this warp outlives the CTA
  } else if (role == kRoleMma) {
    // ============================================================ MMA issuer
    // Whole warp in the loop; lane 0 issues the MMAs and commits.
    int64_t gp = 0, uc = 0, it = 0;
    uint32_t sbits = 0;                          // parity of each S buffer's next use
    const uint32_t smem_base = smem_u32(smem);
    bool ok = true;
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const TcUnit u = tc_unit(g, st, a, w);
      if (u.nchunks == 0) continue;
      const int qb = (int)(uc & 1), ob = (int)(uc & 1);
      if (!(ok = warp_wait(&ctl.q_full[qb], (uint32_t)((uc >> 1) & 1), abort_flag))) break;
      const uint32_t q_addr = smem_base + kOffQ + qb * kQBytes;
      // phase 1: S^T of every chunk into its own buffer
      for (int c = 0; c < u.nchunks && ok; ++c) {
        if (!(ok = warp_wait(&ctl.s_free[c], ((sbits >> c) & 1u) ^ 1u, abort_flag))) break;
        for (int half = 0; half < 2 && ok; ++half) {
          const int64_t i = 2 * it + half;
          const int slot = (int)(i % kSlots);
          if (!(ok = warp_wait(&ctl.slot_full[slot], (uint32_t)((i / kSlots) & 1), abort_flag))) break;
          tc_fence_after();
          if (lane == 0) {
            fence_proxy_async_smem();
            const uint32_t k_addr = smem_base + slot * kSlotBytes;
            for (int kk = 0; kk < 8; ++kk) {            // 8 k-steps of 16 dims per half
              const int slab = kk >> 2, sub = kk & 3;
              const uint64_t da = desc_sw128(k_addr + slab * 16384 + sub * 32, 16, 1024);
              const uint64_t db = desc_sw128(q_addr + (half * 2 + slab) * 2048 + sub * 32, 16, 1024);
              umma_bf16(tmem + c * kN, da, db, kIdescS, (half | kk) != 0);
            }
            umma_commit(&ctl.slot_empty[slot]);
          }
          __syncwarp();
        }
        if (!ok) break;
        ++it;
        sbits ^= 1u << c;
        if (lane == 0) umma_commit(&ctl.s_full[c]);
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&ctl.q_empty[qb]);
      // phase 2: O^T += V^T P^T over the chunks, straight into the unit's O buffer
      if (!(ok = warp_wait(&ctl.o_free[ob], (uint32_t)(((uc >> 1) & 1) ^ 1), abort_flag))) break;
      for (int c = 0; c < u.nchunks && ok; ++c, ++gp) {
        const int pb = (int)(gp & 1);
        if (!(ok = warp_wait(&ctl.p_full[pb], (uint32_t)((gp >> 1) & 1), abort_flag))) break;
        const uint32_t p_addr = smem_base + kOffP + pb * kPBytes;
        for (int half = 0; half < 2 && ok; ++half) {
          const int64_t i = 2 * it + half;
          const int slot = (int)(i % kSlots);
          if (!(ok = warp_wait(&ctl.slot_full[slot], (uint32_t)((i / kSlots) & 1), abort_flag))) break;
          tc_fence_after();
          if (lane == 0) {
            fence_proxy_async_smem();
            const uint32_t v_addr = smem_base + slot * kSlotBytes;
            for (int kk = 0; kk < 8; ++kk) {            // 8 k-steps of 16 keys
              const uint64_t da = desc_sw128(v_addr + kk * 2048, 16384, 1024);
              const uint64_t db = desc_sw128(p_addr + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
              umma_bf16(tmem + kTmemO + ob * 32 + half * kN, da, db, kIdescPV, (c | kk) != 0);
            }
            umma_commit(&ctl.slot_empty[slot]);
          }
          __syncwarp();
        }
        if (!ok) break;
        ++it;
        if (lane == 0) umma_commit(&ctl.p_free[pb]);
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&ctl.o_full[ob]);
      __syncwarp();
      ++uc;
    }
    // every MMA issued above has finished before TMEM is freed
    if (lane == 0) {
      umma_commit(&ctl.mma_done);
      volatile int never = 0;
      mbar_wait(&ctl.mma_done, 0, &never);
    }
    __syncwarp();
  } else if (role == kRoleSoftmax) {
    // ============================================================ softmax + epilogue
    const int quad = warp & 3;                          // TMEM lane quadrant this warp may access
    const int h0 = ridx * kHH;                          // first of this thread's 8 heads
    const int li = quad * 32 + lane;                    // TMEM lane: key of a chunk / dim
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t smem_base = smem_u32(smem);
    const float scale_log2 = g.scale * 1.4426950408889634f;
    const int nthr = 32 * kSoftmaxWarps;
    int64_t gp = 0, uc = 0;
    uint32_t sbits = 0;
    // No early exit in this role: its warps meet at named barriers, so they
    // must run the same iterations.  After an abort every wait returns at
    // once and the loop runs through without blocking.
    for (int64_t w = blockIdx.x; w < n_units; w += gridDim.x) {
      const TcUnit u = tc_unit(g, st, a, w);
      const int32_t* selrow = a.sel + u.tok * g.S;
      float m[kHH], l[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      // key validity of this thread's key in each chunk (kept block, causal within the own block)
      uint32_t vbits = 0;
      for (int c = 0; c < u.nchunks; ++c) {
        const int pos = u.blk_begin + c * kBlk + (li >> 2);
        if (pos < u.blk_end) {
          const int64_t row = block_row(selrow[pos], li & 3, g);
          if (row >= 0 && row <= u.t) vbits |= 1u << c;
        }
      }
      // phase 1: per-head maximum over every chunk but the last, so that the
      // first P chunks need not wait for the last S (folded in below)
      const int n_pre = u.nchunks > 1 ? u.nchunks - 1 : u.nchunks;
      for (int c = 0; c < n_pre; ++c) {
        mbar_wait(&ctl.s_full[c], (sbits >> c) & 1u, abort_flag);
        tc_fence_after();
        float s[kHH];
        tmem_ld8(lane_addr + c * kN + h0, s);
        tmem_wait_ld();
        if ((vbits >> c) & 1u) {
#pragma unroll
          for (int h = 0; h < kHH; ++h) m[h] = fmaxf(m[h], s[h] * scale_log2);
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1)
#pragma unroll
        for (int h = 0; h < kHH; ++h) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < kHH; ++h) ctl.red[0][quad][h0 + h] = m[h];
      named_bar_sync(1, nthr);
#pragma unroll
      for (int h = 0; h < kHH; ++h)
        m[h] = fmaxf(fmaxf(ctl.red[0][0][h0 + h], ctl.red[0][1][h0 + h]),
                     fmaxf(ctl.red[0][2][h0 + h], ctl.red[0][3][h0 + h]));
      // phase 2: P = exp2(S - max) per chunk, written as the B operand of P.V
      const int slab = li >> 6, kin = li & 63;
      const int fold_at = u.nchunks > 1 ? min(2, u.nchunks - 1) : -1;
      const int ob_u = (int)(uc & 1);                   // this unit's O buffer
      for (int c = 0; c < u.nchunks; ++c, ++gp) {
        if (c == fold_at) {
          // the last chunk's maximum: while it exceeds the running one by at
          // most 8 (log2 units) the running one stands -- softmax is shift
          // invariant and P stays below 2^8; beyond that, O and l of the
          // chunks already weighted are rescaled once
          const int cl = u.nchunks - 1;
          mbar_wait(&ctl.s_full[cl], (sbits >> cl) & 1u, abort_flag);
          tc_fence_after();
          float sl[kHH];
          tmem_ld8(lane_addr + cl * kN + h0, sl);
          tmem_wait_ld();
          float ml[kHH];
#pragma unroll
          for (int h = 0; h < kHH; ++h) ml[h] = ((vbits >> cl) & 1u) ? sl[h] * scale_log2 : -INFINITY;
#pragma unroll
          for (int off = 16; off; off >>= 1)
#pragma unroll
            for (int h = 0; h < kHH; ++h) ml[h] = fmaxf(ml[h], __shfl_xor_sync(0xffffffffu, ml[h], off));
          if (lane == 0)
#pragma unroll
            for (int h = 0; h < kHH; ++h) ctl.red[1][quad][h0 + h] = ml[h];
          named_bar_sync(1, nthr);
          float f[kHH];
          bool any = false;                             // uniform across the warp (same heads)
#pragma unroll
          for (int h = 0; h < kHH; ++h) {
            const float mf = fmaxf(fmaxf(ctl.red[1][0][h0 + h], ctl.red[1][1][h0 + h]),
                                   fmaxf(ctl.red[1][2][h0 + h], ctl.red[1][3][h0 + h]));
            f[h] = 1.f;
            if (mf > m[h] + 8.f) {
              f[h] = m[h] == -INFINITY ? 0.f : exp2f(m[h] - mf);
              m[h] = mf;
              any = true;
            }
          }
          if (any) {
            // O holds chunks 0..c-1: wait for the last of their P.V products
            const int64_t gprev = gp - 1;
            mbar_wait(&ctl.p_free[gprev & 1], (uint32_t)((gprev >> 1) & 1), abort_flag);
            tc_fence_after();
            float o0[kHH], o1[kHH];
            tmem_ld8(lane_addr + kTmemO + ob_u * 32 + h0, o0);
            tmem_ld8(lane_addr + kTmemO + ob_u * 32 + kN + h0, o1);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kHH; ++h) {
              o0[h] *= f[h];
              o1[h] *= f[h];
              l[h] *= f[h];
            }
            tmem_st8(lane_addr + kTmemO + ob_u * 32 + h0, o0);
            tmem_st8(lane_addr + kTmemO + ob_u * 32 + kN + h0, o1);
            tmem_wait_st();
            tc_fence_before();
          }
        }
        float s[kHH];
        tmem_ld8(lane_addr + c * kN + h0, s);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.s_free[c]);
        const bool valid = (vbits >> c) & 1u;
        const int pb = (int)(gp & 1);
        mbar_wait(&ctl.p_free[pb], (uint32_t)(((gp >> 1) & 1) ^ 1), abort_flag);
        const uint32_t p_lane = smem_base + kOffP + pb * kPBytes + slab * 2048 + (kin & 7) * 2;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          const int hh = h0 + h;
          const float p = (valid && m[h] != -INFINITY) ? exp2f(s[h] * scale_log2 - m[h]) : 0.f;
          l[h] += p;
          const uint32_t addr = p_lane + (hh >> 3) * 1024 + (hh & 7) * 128 + (((kin >> 3) ^ (hh & 7)) << 4);
          st_shared_u16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(p)));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.p_full[pb]);
      }
      sbits ^= (u.nchunks >= 32 ? 0xffffffffu : ((1u << u.nchunks) - 1u));
      // denominators over all keys
#pragma unroll
      for (int off = 16; off; off >>= 1)
#pragma unroll
        for (int h = 0; h < kHH; ++h) l[h] += __shfl_xor_sync(0xffffffffu, l[h], off);
      named_bar_sync(1, nthr);                // every thread has read red[0] (the maxima)
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < kHH; ++h) ctl.red[0][quad][h0 + h] = l[h];
      named_bar_sync(1, nthr);
#pragma unroll
      for (int h = 0; h < kHH; ++h)
        l[h] = ctl.red[0][0][h0 + h] + ctl.red[0][1][h0 + h] + ctl.red[0][2][h0 + h] + ctl.red[0][3][h0 + h];
      named_bar_sync(1, nthr);                // before red[] is reused
      // output: O^T from TMEM, normalised
      float o0[kHH], o1[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        o0[h] = 0.f;
        o1[h] = 0.f;
      }
      if (u.nchunks > 0) {
        const int ob = (int)(uc & 1);
        mbar_wait(&ctl.o_full[ob], (uint32_t)((uc >> 1) & 1), abort_flag);
        tc_fence_after();
        tmem_ld8(lane_addr + kTmemO + ob * 32 + h0, o0);
        tmem_ld8(lane_addr + kTmemO + ob * 32 + kN + h0, o1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.o_free[ob]);
        ++uc;
      }
      const int64_t unit = u.tok * g.G + u.grp;
      if (a.n_split == 1) {
        __nv_bfloat16* og = (__nv_bfloat16*)a.o + (u.tok * g.H + (int64_t)u.grp * g.hpg) * kHeadDim;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          if (h0 + h < g.hpg) {
            const float inv = 1.f / l[h];
            og[(h0 + h) * kHeadDim + li] = __float2bfloat16_rn(o0[h] * inv);
            og[(h0 + h) * kHeadDim + 128 + li] = __float2bfloat16_rn(o1[h] * inv);
          }
        }
        if (a.lse && li == 0) {
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (h0 + h < g.hpg)
              a.lse[u.tok * g.H + u.grp * g.hpg + h0 + h] = (m[h] + log2f(l[h])) * 0.6931471805599453f;
        }
      } else {
        const int64_t base = (unit * a.n_split + u.split) * g.hpg;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          if (h0 + h < g.hpg) {
            a.part_o[(base + h0 + h) * kHeadDim + li] = o0[h];
            a.part_o[(base + h0 + h) * kHeadDim + 128 + li] = o1[h];
          }
        }
        if (li == 0) {
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (h0 + h < g.hpg) {
              a.part_ml[(base + h0 + h) * 2] = u.nchunks ? m[h] * 0.6931471805599453f : -INFINITY;
              a.part_ml[(base + h0 + h) * 2 + 1] = l[h];
            }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (role == kRoleMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace qsa
