// attn_bwd.cuh -- backward of the sparse GQA attention on CUDA cores.
//
// Miles docs "Qwen3.8-Flash-Next", section 1: the QSA attention kernel has a
// forward and a backward pass over the same kept tokens.  For the loss
// sum_h dout_h . o_h, with P_hj = exp(scale q_h . k_j - lse_h) over the kept
// tokens j (block kept, j <= t), the derivative of softmax attention is
//   dp_hj = dout_h . v_j,  delta_h = dout_h . o_h (= sum_j P_hj dp_hj),
//   ds_hj = P_hj (dp_hj - delta_h),
//   dq_h = scale sum_j ds_hj k_j,  dk_j += scale sum_h ds_hj q_h,
//   dv_j += sum_h P_hj dout_h.
// One CTA per (query token, KV group): the group's heads share the kept
// keys, so each gathered K/V row serves all of them, and its dk/dv rows are
// summed over the heads before fp32 atomic adds, four elements per 16-byte
// atomic (keys are shared by many queries, so the key gradients are
// accumulated in place).
// lse is the forward's natural-log normaliser, so probabilities are
// recomputed without a second pass.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {
namespace bwd_attn {
constexpr int THREADS = 512;
constexpr int KC = 32;          // keys per chunk (8 blocks of 4)
constexpr int KPAD = kHeadDim + 1;
}

struct AttnBwdArgs {
  const void* q;          // [T][H][D] I/O dtype
  const void* o;          // [T][H][D] forward output
  const float* lse;       // [T][H] forward log-sum-exp (natural log)
  const void* dout;       // [T][H][D]
  const void* k;          // [slots][G][n_cap][D]
  const void* v;
  const int32_t* sel;
  const int32_t* nsel;
  float* dq;              // [T][H][D] fp32, written
  float* dk;              // [slots][G][n_cap][D] fp32, accumulated
  float* dv;
};

inline size_t attn_bwd_smem() {
  using namespace bwd_attn;
  return sizeof(float) * (2 * kMaxHpg * kHeadDim + 2 * KC * KPAD + 2 * kMaxHpg * KC + 2 * kMaxHpg);
}

template <typename T>
__global__ void __launch_bounds__(bwd_attn::THREADS) attn_bwd_kernel(Geo g, SegTable st, AttnBwdArgs a) {
  pdl_wait();
  pdl_trigger();
  using namespace bwd_attn;
  constexpr int D = kHeadDim;
  extern __shared__ float sm[];
  float* qs = sm;                              // [hpg][D]
  float* dos = qs + kMaxHpg * D;               // [hpg][D]
  float* kt = dos + kMaxHpg * D;               // [KC][KPAD]
  float* vt = kt + KC * KPAD;                  // [KC][KPAD]
  float* ps = vt + KC * KPAD;                  // [hpg][KC] probabilities
  float* dss = ps + kMaxHpg * KC;              // [hpg][KC] ds
  float* del = dss + kMaxHpg * KC;             // [hpg] delta
  float* lss = del + kMaxHpg;                  // [hpg] lse
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hpg = g.hpg;

  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int local = item - st.item0[si];
  const int j = local / g.G;
  const int grp = local - j * g.G;
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = (int64_t)st.pos0[si] + j;
  const int64_t slot = st.slot[si];
  const int nsel = min(max(a.nsel[tok], 0), g.S);
  const int32_t* sel = a.sel + tok * g.S;

  const int64_t hrow = tok * g.H + (int64_t)grp * hpg;     // first head row of the group
  const T* qg = (const T*)a.q + hrow * D;
  const T* dg = (const T*)a.dout + hrow * D;
  for (int e = tid; e < hpg * D; e += THREADS) {
    qs[e] = IO<T>::to_f(qg[e]);
    dos[e] = IO<T>::to_f(dg[e]);
  }
  if (warp < hpg) {
    // delta_h = dout_h . o_h
    const T* og = (const T*)a.o + (hrow + warp) * D;
    const T* dh = dg + (int64_t)warp * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s = fmaf(IO<T>::to_f(dh[d]), IO<T>::to_f(og[d]), s);
#pragma unroll
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      del[warp] = s;
      lss[warp] = a.lse[hrow + warp];
    }
  }
  const size_t kv_base = ((size_t)slot * g.G + grp) * (size_t)g.n_cap * D;
  const T* kg = (const T*)a.k + kv_base;
  const T* vg = (const T*)a.v + kv_base;
  float* dkg = a.dk + kv_base;
  float* dvg = a.dv + kv_base;

  float dq_acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) dq_acc[i] = 0.f;
  const int d_own = tid % D, h_base = (tid / D) * 8;
  __syncthreads();

  for (int c0 = 0; c0 < nsel; c0 += KC / 4) {
    const int nb = min(KC / 4, nsel - c0);
    // gather the chunk's K and V rows (zeros for padding or rejected indices)
    for (int e = tid; e < KC * D; e += THREADS) {
      const int kk = e / D, d = e % D;
      const int bi = kk >> 2;
      float xk = 0.f, xv = 0.f;
      if (bi < nb) {
        const int64_t row = block_row(sel[c0 + bi], kk & 3, g);
        if (row >= 0) {
          xk = IO<T>::to_f(kg[row * D + d]);
          xv = IO<T>::to_f(vg[row * D + d]);
        }
      }
      kt[kk * KPAD + d] = xk;
      vt[kk * KPAD + d] = xv;
    }
    __syncthreads();
    // probabilities and ds: one thread per (head, key)
    if (tid < hpg * KC) {
      const int h = tid / KC, kk = tid % KC, bi = kk >> 2;
      const int64_t row = bi < nb ? block_row(sel[c0 + bi], kk & 3, g) : -1;
      const bool valid = row >= 0 && row <= t;
      float s = 0.f, dp = 0.f;
      const float* qh = qs + h * D;
      const float* dh = dos + h * D;
      const float* kr = kt + kk * KPAD;
      const float* vr = vt + kk * KPAD;
#pragma unroll 8
      for (int d = 0; d < D; ++d) {
        s = fmaf(qh[d], kr[d], s);
        dp = fmaf(dh[d], vr[d], dp);
      }
      const float p = valid ? expf(s * g.scale - lss[h]) : 0.f;
      ps[h * KC + kk] = p;
      dss[h * KC + kk] = p * (dp - del[h]);
    }
    __syncthreads();
    // dq_h += scale * sum_j ds_hj k_j
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int h = h_base + i;
      if (h < hpg) {
        float acc = 0.f;
        const float* dsh = dss + h * KC;
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) acc = fmaf(dsh[kk], kt[kk * KPAD + d_own], acc);
        dq_acc[i] = fmaf(acc, g.scale, dq_acc[i]);
      }
    }
    // dk_j += scale * sum_h ds_hj q_h ; dv_j += sum_h P_hj dout_h  (attended keys only),
    // four dims per thread and one 16-byte atomic add per tensor
    for (int e = tid; e < KC * D / 4; e += THREADS) {
      const int kk = e / (D / 4), d = 4 * (e % (D / 4));
      const int bi = kk >> 2;
      const int64_t row = bi < nb ? block_row(sel[c0 + bi], kk & 3, g) : -1;
      if (row < 0 || row > t) continue;
      float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sv = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int h = 0; h < hpg; ++h) {
        const float ds = dss[h * KC + kk], p = ps[h * KC + kk];
        const float4 qv = *reinterpret_cast<const float4*>(qs + h * D + d);
        const float4 ov = *reinterpret_cast<const float4*>(dos + h * D + d);
        sk.x = fmaf(ds, qv.x, sk.x);
        sk.y = fmaf(ds, qv.y, sk.y);
        sk.z = fmaf(ds, qv.z, sk.z);
        sk.w = fmaf(ds, qv.w, sk.w);
        sv.x = fmaf(p, ov.x, sv.x);
        sv.y = fmaf(p, ov.y, sv.y);
        sv.z = fmaf(p, ov.z, sv.z);
        sv.w = fmaf(p, ov.w, sv.w);
      }
      sk.x *= g.scale;
      sk.y *= g.scale;
      sk.z *= g.scale;
      sk.w *= g.scale;
      atomicAdd(reinterpret_cast<float4*>(dkg + row * D + d), sk);
      atomicAdd(reinterpret_cast<float4*>(dvg + row * D + d), sv);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int h = h_base + i;
    if (h < hpg) a.dq[(hrow + h) * D + d_own] = dq_acc[i];
  }
}

}  // namespace qsa
