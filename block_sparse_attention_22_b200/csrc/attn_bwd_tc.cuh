// attn_bwd_tc.cuh -- backward of the sparse GQA attention on tcgen05 tensor
// cores (bf16 I/O).
//
// Miles docs "Qwen3.8-Flash-Next", section 1: the QSA attention kernel has a
// forward and a backward pass over the same kept tokens.  For one work unit
// (query token t, KV group) with its hpg <= 16 heads h and the kept keys j
// (block kept, j <= t), with tau = softmax scale and lse_h the forward's
// natural-log normaliser:
//   S^T[j, h]  = K_j . Q_h                     M=128 keys, N=16, K=256 dims
//   dP^T[j, h] = V_j . dO_h                    same shape
//   P = exp(tau S - lse_h), dS = P (dP - delta_h), delta_h = dO_h . O_h
//   dQ^T[d, h] += K^T[d, j] dS^T[j, h]         M=128 dims (x2), N=16, K=128 keys of a chunk
//   dV[j, d]    = P^T[j, h] dO[h, d]           M=128 keys, N=256 dims, K=16 heads
//   dK[j, d]    = dS^T[j, h] Q[h, d]           same shape
// and dq = tau dQ, dk += tau dK, dv += dV.  Keys are shared by many queries,
// so dK and dV of every chunk are added to the fp32 gradients in place, four
// elements per 16-byte atomic, rows of keys that are not attended skipped
// (their P and dS are zero).
//
// Same roles as the forward kernel (20 warps, one CTA per SM, persistent over
// units): nine cp.async producer warps gather each chunk's K rows (two 32 KiB
// half-slots) then its V rows into a 6-slot ring, producer 0 also loads the
// unit's Q and dO tiles with TMA; warp 0 owns TMEM and issues the MMAs; eight
// softmax/epilogue warps (a thread owns TMEM lane i -- key i of a chunk, or
// dim i of dQ -- and 8 of the 16 heads) turn S and dP into P^T and dS^T
// (bf16, in the layout the MMAs read) and drain dV, dK and dQ from TMEM.
// P^T and dS^T double as the MN-major A operand of the dV/dK products; the
// Q and dO tiles (64-dim slabs of 16 head rows) as their MN-major B operand.
// MMA order per chunk c: S(c); dQ, dV, dK of chunk c-1 (its dQ frees its K
// slots, which chunk c's V rows take in the 6-slot ring); dP(c).  A chunk's
// V slots are freed after its dP MMAs, so chunk c-1's softmax overlaps the
// S MMAs of chunk c.
// Every mbarrier wait is bounded (sm100::mbar_wait).
#pragma once
#include "qsa_internal.cuh"
#include "sm100.cuh"
#include "attn_tc.cuh"

namespace qsa {
namespace tc_bwd {
using tc_attn::kBlk;
using tc_attn::kProducers;
constexpr int kBlkPerProducer = (kBlk + kProducers - 1) / kProducers;   // kept blocks per producer and chunk
using tc_attn::kSoftmaxWarps;
using tc_attn::kThreads;
using tc_attn::kHH;
using tc_attn::kN;
constexpr int kSlots = 6;                  // 32 KiB K/V half-chunk slots
constexpr int kSlotBytes = 32768;
constexpr int kTileBytes = 8192;           // Q or dO: 16 heads x 256 dims, 4 slabs x 2 KiB
constexpr int kPBytes = 4096;              // P^T or dS^T of a chunk: 16 heads x 128 keys
constexpr int kOffQ = kSlots * kSlotBytes;             // 196608
constexpr int kOffDO = kOffQ + kTileBytes;             // 204800
constexpr int kOffP = kOffDO + kTileBytes;             // 212992: P^T[2]
constexpr int kOffDS = kOffP + 2 * kPBytes;            // 221184: dS^T[2]
constexpr int kOffBar = kOffDS + 2 * kPBytes;          // 229376
constexpr int kSmemBytes = kOffBar + 1024 + 1024;      // control block + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;             // S^T of chunk parity b: 16 columns at 16 b
constexpr uint32_t kTmemDP = 32;           // dP^T: 16 columns at 32 + 16 b
constexpr uint32_t kTmemDQ = 64;           // dQ^T: dims 0-127 at 64, 128-255 at 80
constexpr uint32_t kTmemKV = 256;          // dV or dK of a chunk: 256 columns
constexpr uint32_t kIdescS = sm100::idesc_bf16(128, kN, false, false);    // S^T, dP^T
constexpr uint32_t kIdescDQ = sm100::idesc_bf16(128, kN, true, false);    // A = K^T (MN-major)
constexpr uint32_t kIdescKV = sm100::idesc_bf16(128, 256, true, true);    // A = P^T / dS^T, B = dO / Q
}

struct AttnBwdTcArgs {
  const void* o;           // bf16 [T][H][D] forward output
  const float* lse;        // [T][H]
  const void* dout;        // bf16 [T][H][D]
  const void* k;           // bf16 [n_slots][G][n_cap][D]
  const void* v;
  const int32_t* sel;
  const int32_t* nsel;
  float* dq;               // [T][H][D], written
  float* dk;               // [n_slots][G][n_cap][D], accumulated
  float* dv;
  int64_t units_per_group; // query tokens of the launch
};

struct AttnBwdTcCtl {
  uint64_t slot_full[tc_bwd::kSlots];
  uint64_t slot_empty[tc_bwd::kSlots];
  uint64_t qd_full, qd_empty;
  uint64_t s_full[2], s_free[2], dp_full[2];
  uint64_t ps_full[2], ps_free[2];
  uint64_t kv_full, kv_free;
  uint64_t dq_full, dq_free;
  uint64_t mma_done;
  float delta[16];
  float lse2[16];          // lse_h * log2(e)
  uint32_t tmem_base;
  int abort;
};

struct BwdUnit {
  int64_t tok, t, slot;
  int grp;
  int nblk;                // kept blocks
  int nchunks;
};

__device__ __forceinline__ BwdUnit bwd_unit(const Geo& g, const SegTable& st, const AttnBwdTcArgs& a, int64_t w) {
  BwdUnit u;
  u.grp = (int)(w / a.units_per_group);
  const int rem = (int)(w - (int64_t)u.grp * a.units_per_group);
  const int si = find_segment(st, rem);
  const int j = rem - st.item0[si];
  u.tok = st.q_offset[si] + j;
  u.t = (int64_t)st.pos0[si] + j;
  u.slot = st.slot[si];
  u.nblk = min(max(a.nsel[u.tok], 0), g.S);
  u.nchunks = (int)cdiv(u.nblk, tc_bwd::kBlk);
  return u;
}

__global__ void __launch_bounds__(tc_bwd::kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do, Geo g,
                       SegTable st, AttnBwdTcArgs a) {
  using namespace tc_bwd;
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  AttnBwdTcCtl& ctl = *reinterpret_cast<AttnBwdTcCtl*>(smem + kOffBar);
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_units = (int64_t)g.G * a.units_per_group;
  int ridx = 0;
  const tc_attn::Role role = tc_role(warp, ridx);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&ctl.slot_full[i], kProducers * 32);   // one cp.async completion arrival per producer lane
      mbar_init(&ctl.slot_empty[i], 1);
    }
    mbar_init(&ctl.qd_full, 1);
    mbar_init(&ctl.qd_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.dp_full[i], 1);
      mbar_init(&ctl.s_free[i], kSoftmaxWarps);
      mbar_init(&ctl.ps_full[i], kSoftmaxWarps);
      mbar_init(&ctl.ps_free[i], 1);
    }
    mbar_init(&ctl.kv_full, 1);
    mbar_init(&ctl.kv_free, kSoftmaxWarps);
    mbar_init(&ctl.dq_full, 1);
    mbar_init(&ctl.dq_free, kSoftmaxWarps);
    mbar_init(&ctl.mma_done, 1);
    ctl.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
  }
  // zero Q and dO: rows hpg..15 are never loaded and must read as zero
  for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (role == tc_attn::kRoleMma) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  pdl_wait();
  pdl_trigger();

  if (role == tc_attn::kRoleProducer) {
    // ============================================================ producers
    const int pw = ridx;                         // copies blocks pw + kProducers i of a chunk
    int64_t hs_next = 0, uc = 0;
    bool ok = true;
    const int r = (lane >> 3) & 3, jc = lane & 7;   // row of a block and 16-byte chunk of a line
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const BwdUnit u = bwd_unit(g, st, a, w);
      if (u.nchunks == 0) continue;
      if (pw == 0) {
        if (!(ok = warp_wait(&ctl.qd_empty, (uint32_t)((uc & 1) ^ 1), abort_flag))) break;
        if (lane == 0) {
          mbar_expect_tx(&ctl.qd_full, (uint32_t)(g.hpg * 128 * 4 * 2));
          const int32_t qrow = (int32_t)(u.tok * g.H + (int64_t)u.grp * g.hpg);
          for (int s = 0; s < 4; ++s) {
            tma_load_2d(smem + kOffQ + s * 2048, &tm_q, 64 * s, qrow, &ctl.qd_full);
            tma_load_2d(smem + kOffDO + s * 2048, &tm_do, 64 * s, qrow, &ctl.qd_full);
          }
        }
        __syncwarp();
      }
      ++uc;
      const size_t kv_base = ((size_t)u.slot * g.G + u.grp) * (size_t)g.n_cap * kHeadDim;
      const __nv_bfloat16* kg = (const __nv_bfloat16*)a.k + kv_base;
      const __nv_bfloat16* vg = (const __nv_bfloat16*)a.v + kv_base;
      const int32_t* selrow = a.sel + u.tok * g.S;
      for (int c = 0; c < u.nchunks && ok; ++c) {
        int64_t myrow = -1;                      // rows of this warp's kept blocks (lane i < kBlkPerProducer)
        if (lane < kBlkPerProducer && pw + kProducers * lane < kBlk) {
          const int pos = c * kBlk + pw + kProducers * lane;
          if (pos < u.nblk) myrow = block_row(selrow[pos], 0, g);
        }
        for (int kind = 0; kind < 2 && ok; ++kind) {   // K rows, then V rows of the chunk
          const __nv_bfloat16* base = kind == 0 ? kg : vg;
          for (int h = 0; h < 2 && ok; ++h) {
            const int64_t hs = hs_next++;
            const int slot = (int)(hs % kSlots);
            if (!(ok = warp_wait(&ctl.slot_empty[slot], (uint32_t)(((hs / kSlots) & 1) ^ 1), abort_flag))) break;
            const uint32_t dst0 = smem_u32(smem + slot * kSlotBytes);
#pragma unroll
            for (int bq = 0; bq < kBlkPerProducer; ++bq) {
              const int b = pw + kProducers * bq;
              if (b >= kBlk) break;
              const int64_t row = __shfl_sync(0xffffffffu, myrow, bq);
              const int line = 4 * b + r;
              const uint32_t dst = dst0 + line * 128 + ((jc ^ (line & 7)) << 4);
              const __nv_bfloat16* src = base + 128 * h + 8 * jc + (row >= 0 ? (row + r) * kHeadDim : 0);
              const uint32_t nb = row >= 0 ? 16u : 0u;
              cp_async16(dst, src, nb);
              cp_async16(dst + 16384, src + 64, nb);
            }
            cp_async_mbar_arrive(&ctl.slot_full[slot]);
          }
        }
      }
    }
    cp_async_wait_all();
  } else if (role == tc_attn::kRoleMma) {
    // ============================================================ MMA issuer
    int64_t it = 0, uc = 0, gc = 0, kvn = 0;
    const uint32_t sb = smem_u32(smem);
    bool ok = true;
    // dQ, dV and dK of chunk cc (parity buffer bb), whose K rows are in
    // half-slots ks0 and ks0+1 of the ring; `first` starts dQ of the unit
    auto tail = [&](int64_t gcc, int64_t ks0, bool first) -> bool {
      const int bb = (int)(gcc & 1);
      if (!warp_wait(&ctl.ps_full[bb], (uint32_t)((gcc >> 1) & 1), abort_flag)) return false;
      tc_fence_after();
      const uint32_t ds_addr = sb + kOffDS + bb * kPBytes;
      const uint32_t p_addr = sb + kOffP + bb * kPBytes;
      for (int half = 0; half < 2; ++half) {
        const int slot = (int)((ks0 + half) % kSlots);
        if (lane == 0) {
          const uint32_t k_addr = sb + slot * kSlotBytes;
          for (int kk = 0; kk < 8; ++kk) {       // 8 k-steps of 16 keys
            const uint64_t da = desc_sw128(k_addr + kk * 2048, 16384, 1024);
            const uint64_t db = desc_sw128(ds_addr + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
            umma_bf16(tmem + kTmemDQ + half * kN, da, db, kIdescDQ, !(first && kk == 0));
          }
          umma_commit(&ctl.slot_empty[slot]);  // the K rows are no longer read
        }
        __syncwarp();
      }
      for (int which = 0; which < 2; ++which) {  // dV = P^T dO, then dK = dS^T Q
        if (!warp_wait(&ctl.kv_free, (uint32_t)((kvn & 1) ^ 1), abort_flag)) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = desc_sw128(which == 0 ? p_addr : ds_addr, 2048, 1024);
          const uint64_t db = desc_sw128(sb + (which == 0 ? kOffDO : kOffQ), 2048, 1024);
          umma_bf16(tmem + kTmemKV, da, db, kIdescKV, false);
          umma_commit(&ctl.kv_full);
        }
        __syncwarp();
        ++kvn;
      }
      if (lane == 0) umma_commit(&ctl.ps_free[bb]);
      __syncwarp();
      return true;
    };
    for (int64_t w = blockIdx.x; w < n_units && ok; w += gridDim.x) {
      if (warp_aborted(abort_flag)) break;
      const BwdUnit u = bwd_unit(g, st, a, w);
      if (u.nchunks == 0) continue;
      if (!(ok = warp_wait(&ctl.qd_full, (uint32_t)(uc & 1), abort_flag))) break;
      if (!(ok = warp_wait(&ctl.dq_free, (uint32_t)((uc & 1) ^ 1), abort_flag))) break;
      const uint32_t q_addr = sb + kOffQ, do_addr = sb + kOffDO;
      int64_t prev_ks = -1, prev_gc = -1;
      for (int c = 0; c < u.nchunks && ok; ++c, ++gc) {
        const int b = (int)(gc & 1);
        if (!(ok = warp_wait(&ctl.s_free[b], (uint32_t)(((gc >> 1) & 1) ^ 1), abort_flag))) break;
        const int64_t ks0 = it;
        // S^T = K Q^T; the previous chunk's dQ/dV/dK (its dQ frees its K
        // slots, which this chunk's V rows take); then dP^T = V dO^T
        for (int kind = 0; kind < 2 && ok; ++kind) {
          if (kind == 1 && prev_gc >= 0 && !(ok = tail(prev_gc, prev_ks, c == 1))) break;
          for (int half = 0; half < 2 && ok; ++half) {
            const int64_t i = it++;
            const int slot = (int)(i % kSlots);
            if (!(ok = warp_wait(&ctl.slot_full[slot], (uint32_t)((i / kSlots) & 1), abort_flag))) break;
            tc_fence_after();
            if (lane == 0) {
              fence_proxy_async_smem();
              const uint32_t a_addr = sb + slot * kSlotBytes;
              const uint32_t b_tile = kind == 0 ? q_addr : do_addr;
              const uint32_t d = tmem + (kind == 0 ? kTmemS : kTmemDP) + b * kN;
              for (int kk = 0; kk < 8; ++kk) {   // 8 k-steps of 16 dims per half
                const int slab = kk >> 2, sub = kk & 3;
                const uint64_t da = desc_sw128(a_addr + slab * 16384 + sub * 32, 16, 1024);
                const uint64_t db = desc_sw128(b_tile + (half * 2 + slab) * 2048 + sub * 32, 16, 1024);
                umma_bf16(d, da, db, kIdescS, (half | kk) != 0);
              }
              if (kind == 1) umma_commit(&ctl.slot_empty[slot]);   // V rows are read only here
            }
            __syncwarp();
          }
          if (ok && lane == 0) umma_commit(kind == 0 ? &ctl.s_full[b] : &ctl.dp_full[b]);
          __syncwarp();
        }
        if (!ok) break;
        prev_ks = ks0;
        prev_gc = gc;
      }
      if (!ok) break;
      if (!(ok = tail(prev_gc, prev_ks, u.nchunks == 1))) break;
      if (lane == 0) {
        umma_commit(&ctl.dq_full);
        umma_commit(&ctl.qd_empty);              // Q and dO are no longer read
      }
      __syncwarp();
      ++uc;
    }
    if (lane == 0) {
      umma_commit(&ctl.mma_done);
      volatile int never = 0;
      mbar_wait(&ctl.mma_done, 0, &never);
    }
    __syncwarp();
  } else if (role == tc_attn::kRoleSoftmax) {
    // ============================================================ softmax + epilogue
    const int quad = warp & 3;                          // TMEM lane quadrant of this warp
    const int h0 = ridx * kHH;                          // first of this thread's 8 heads
    const int li = quad * 32 + lane;                    // TMEM lane: key of a chunk / dim of dQ
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t sb = smem_u32(smem);
    const float tau2 = g.scale * 1.4426950408889634f;
    const int nthr = 32 * kSoftmaxWarps;
    const int sw = quad + 4 * ridx;                     // 0..7 among the softmax warps
    int64_t gc = 0, uc = 0, kvn = 0;
    // No early exit in this role: its warps meet at a named barrier each unit.
    for (int64_t w = blockIdx.x; w < n_units; w += gridDim.x) {
      const BwdUnit u = bwd_unit(g, st, a, w);
      if (u.nchunks == 0) continue;
      const int64_t hrow = u.tok * g.H + (int64_t)u.grp * g.hpg;
      // delta_h = dO_h . O_h and lse_h (log2 units) of the unit's heads
      for (int h = sw; h < kN; h += kSoftmaxWarps) {
        float s = 0.f;
        if (h < g.hpg) {
          const __nv_bfloat16* og = (const __nv_bfloat16*)a.o + (hrow + h) * kHeadDim;
          const __nv_bfloat16* dg = (const __nv_bfloat16*)a.dout + (hrow + h) * kHeadDim;
          for (int d = lane; d < kHeadDim; d += 32) s = fmaf(__bfloat162float(dg[d]), __bfloat162float(og[d]), s);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
          ctl.delta[h] = s;
          ctl.lse2[h] = h < g.hpg ? a.lse[hrow + h] * 1.4426950408889634f : 0.f;
        }
      }
      named_bar_sync(1, nthr);
      float dl[kHH], ls[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        dl[h] = ctl.delta[h0 + h];
        ls[h] = ctl.lse2[h0 + h];
      }
      named_bar_sync(1, nthr);                          // delta/lse are rewritten by the next unit
      const int32_t* selrow = a.sel + u.tok * g.S;
      const size_t kv_base = ((size_t)u.slot * g.G + u.grp) * (size_t)g.n_cap * kHeadDim;
      const int slab = li >> 6, kin = li & 63;
      const int ch = ridx;                              // dims 128 ch .. +127 of dV/dK rows
      for (int c = 0; c < u.nchunks; ++c, ++gc) {
        const int b = (int)(gc & 1);
        // this thread's key: kept, inside the chunk, not after t
        int64_t row = -1;
        {
          const int pos = c * kBlk + (li >> 2);
          if (pos < u.nblk) {
            const int64_t rr = block_row(selrow[pos], li & 3, g);
            if (rr >= 0 && rr <= u.t) row = rr;
          }
        }
        const bool valid = row >= 0;
        mbar_wait(&ctl.s_full[b], (uint32_t)((gc >> 1) & 1), abort_flag);
        mbar_wait(&ctl.dp_full[b], (uint32_t)((gc >> 1) & 1), abort_flag);
        tc_fence_after();
        float s[kHH], dp[kHH];
        tmem_ld8(lane_addr + kTmemS + b * kN + h0, s);
        tmem_ld8(lane_addr + kTmemDP + b * kN + h0, dp);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.s_free[b]);
        mbar_wait(&ctl.ps_free[b], (uint32_t)(((gc >> 1) & 1) ^ 1), abort_flag);
        const uint32_t p_lane = sb + kOffP + b * kPBytes + slab * 2048 + (kin & 7) * 2;
        const uint32_t d_lane = sb + kOffDS + b * kPBytes + slab * 2048 + (kin & 7) * 2;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          const int hh = h0 + h;
          const float p = (valid && hh < g.hpg) ? exp2f(s[h] * tau2 - ls[h]) : 0.f;
          const float ds = p * (dp[h] - dl[h]);
          const uint32_t off = (hh >> 3) * 1024 + (hh & 7) * 128 + (((kin >> 3) ^ (hh & 7)) << 4);
          st_shared_u16(p_lane + off, __bfloat16_as_ushort(__float2bfloat16_rn(p)));
          st_shared_u16(d_lane + off, __bfloat16_as_ushort(__float2bfloat16_rn(ds)));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.ps_full[b]);
        // dV, then dK, of this chunk's keys: added to the gradients in place
        for (int which = 0; which < 2; ++which, ++kvn) {
          mbar_wait(&ctl.kv_full, (uint32_t)(kvn & 1), abort_flag);
          tc_fence_after();
          float* dst = (which == 0 ? a.dv : a.dk) + kv_base + (valid ? row : 0) * kHeadDim + ch * 128;
          const float f = which == 0 ? 1.f : g.scale;
#pragma unroll 1
          for (int piece = 0; piece < 8; ++piece) {
            float x[16];
            tmem_ld16(lane_addr + kTmemKV + ch * 128 + piece * 16, x);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                atomicAdd(reinterpret_cast<float4*>(dst + piece * 16 + 4 * q4),
                          make_float4(x[4 * q4] * f, x[4 * q4 + 1] * f, x[4 * q4 + 2] * f, x[4 * q4 + 3] * f));
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.kv_free);
        }
      }
      // dq = tau dQ: lane li holds dims li and 128 + li of 8 heads
      mbar_wait(&ctl.dq_full, (uint32_t)(uc & 1), abort_flag);
      tc_fence_after();
      float q0[kHH], q1[kHH];
      tmem_ld8(lane_addr + kTmemDQ + h0, q0);
      tmem_ld8(lane_addr + kTmemDQ + kN + h0, q1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.dq_free);
      ++uc;
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        if (h0 + h < g.hpg) {
          float* out = a.dq + (hrow + h0 + h) * kHeadDim;
          out[li] = q0[h] * g.scale;
          out[128 + li] = q1[h] * g.scale;
        }
      }
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
