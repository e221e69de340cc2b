// attn_simt.cuh -- sparse GQA attention on CUDA cores (fp32 I/O path), and
// the split-K combine shared with the tensor-core kernel.
//
// Miles docs "Qwen3.8-Flash-Next", section 1: attention reads only the kept
// key tokens; 24 heads in 2 query groups, head dim 256.  Token j is attended
// iff its block floor(j/r) is kept and j <= t (the own block is causally
// masked).  One CTA per (query token, KV group, split): the group's heads
// share the selection, so every gathered K/V row is used by all of them.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {
namespace simt_attn {
constexpr int THREADS = 512;
constexpr int KC = 32;          // keys per chunk (8 blocks of 4)
constexpr int KPAD = kHeadDim + 1;
}

struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* sel;
  const int32_t* nsel;
  void* o;
  float* lse;
  float* part_o;      // [units][n_split][hpg][D] unnormalised partial outputs
  float* part_ml;     // [units][n_split][hpg][2]  (running max, sum)
  int n_split;        // 1: write o/lse directly
  int blocks_per_split;
};

template <typename T>
__global__ void __launch_bounds__(simt_attn::THREADS) attn_simt_kernel(Geo g, SegTable st, AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  using namespace simt_attn;
  constexpr int D = kHeadDim;
  extern __shared__ float sm[];
  float* qs = sm;                              // [hpg][D]
  float* kv = qs + kMaxHpg * D;                // [KC][KPAD]
  float* ps = kv + KC * KPAD;                  // [hpg][KC]
  float* mls = ps + kMaxHpg * KC;              // m[16], l[16], alpha[16]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hpg = g.hpg;

  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int local = item - st.item0[si];
  const int per_tok = g.G * a.n_split;
  const int j = local / per_tok;
  const int grp = (local / a.n_split) % g.G;
  const int split = local % a.n_split;
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = (int64_t)st.pos0[si] + j;
  const int64_t slot = st.slot[si];
  const int nsel = min(max(a.nsel[tok], 0), g.S);      // caller-supplied: clamp to the row
  const int32_t* sel = a.sel + tok * g.S;
  const int sb = split * a.blocks_per_split;
  const int se = min(nsel, sb + a.blocks_per_split);

  const T* qg = (const T*)a.q + (tok * g.H + (int64_t)grp * hpg) * D;
  for (int e = tid; e < hpg * D; e += THREADS) qs[e] = IO<T>::to_f(qg[e]);
  if (tid < kMaxHpg) {
    mls[tid] = -INFINITY;
    mls[16 + tid] = 0.f;
  }
  const size_t kv_base = ((size_t)slot * g.G + grp) * (size_t)g.n_cap * D;
  const T* kg = (const T*)a.k + kv_base;
  const T* vg = (const T*)a.v + kv_base;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const int d_own = tid % D, h_base = (tid / D) * 8;
  __syncthreads();

  for (int c0 = sb; c0 < se; c0 += KC / 4) {
    const int nb = min(KC / 4, se - c0);
    // gather K rows of up to 8 kept blocks
    for (int e = tid; e < KC * D; e += THREADS) {
      const int kk = e / D, d = e % D;
      const int bi = kk >> 2;
      float x = 0.f;
      if (bi < nb) {
        const int64_t row = block_row(sel[c0 + bi], kk & 3, g);
        if (row >= 0) x = IO<T>::to_f(kg[row * D + d]);
      }
      kv[kk * KPAD + d] = x;
    }
    __syncthreads();
    if (warp < hpg) {
      const int kk = lane, bi = kk >> 2;
      int64_t row = bi < nb ? block_row(sel[c0 + bi], kk & 3, g) : -1;
      if (row < 0) row = INT64_MAX;                   // padding or rejected index: masked
      float s = 0.f;
      const float* qh = qs + warp * D;
      const float* kr = kv + kk * KPAD;
#pragma unroll 8
      for (int d = 0; d < D; ++d) s = fmaf(qh[d], kr[d], s);
      s = (row <= t) ? s * g.scale : -INFINITY;
      float mx = s;
#pragma unroll
      for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = mls[warp];
      const float m_new = fmaxf(m_old, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : expf(m_old - m_new);
      const float p = (s == -INFINITY) ? 0.f : expf(s - m_new);
      float ps_sum = p;
#pragma unroll
      for (int off = 16; off; off >>= 1) ps_sum += __shfl_xor_sync(0xffffffffu, ps_sum, off);
      ps[warp * KC + kk] = p;
      __syncwarp();
      if (lane == 0) {
        mls[warp] = m_new;
        mls[16 + warp] = mls[16 + warp] * alpha + ps_sum;
        mls[32 + warp] = alpha;
      }
    }
    __syncthreads();
    // gather V rows
    for (int e = tid; e < KC * D; e += THREADS) {
      const int kk = e / D, d = e % D;
      const int bi = kk >> 2;
      float x = 0.f;
      if (bi < nb) {
        const int64_t row = block_row(sel[c0 + bi], kk & 3, g);
        if (row >= 0) x = IO<T>::to_f(vg[row * D + d]);
      }
      kv[kk * KPAD + d] = x;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int h = h_base + i;
      if (h < hpg) {
        float o = acc[i] * mls[32 + h];
        const float* ph = ps + h * KC;
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) o = fmaf(ph[kk], kv[kk * KPAD + d_own], o);
        acc[i] = o;
      }
    }
    __syncthreads();
  }

  const int64_t unit = tok * g.G + grp;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int h = h_base + i;
    if (h >= hpg) continue;
    const float m = mls[h], l = mls[16 + h];
    if (a.n_split == 1) {
      T* og = (T*)a.o + (tok * g.H + (int64_t)grp * hpg + h) * D;
      og[d_own] = IO<T>::from_f(acc[i] / l);
      if (a.lse && d_own == 0) a.lse[tok * g.H + grp * hpg + h] = m + logf(l);
    } else {
      const int64_t pidx = (unit * a.n_split + split) * hpg + h;
      a.part_o[pidx * D + d_own] = acc[i];
      if (d_own == 0) {
        a.part_ml[pidx * 2] = m;
        a.part_ml[pidx * 2 + 1] = l;
      }
    }
  }
}

// Log-sum-exp combine of split partials: one thread per (token, head, 4
// dims); the table's item0 counts tokens per segment.  The loops over splits
// are unrolled so their loads are in flight together.
template <typename T>
__global__ void __launch_bounds__(256) attn_combine_kernel(Geo g, SegTable st, AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int D = kHeadDim, V = 4;
  const int64_t total = (int64_t)st.item0[st.n] * g.H * (D / V);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(e % (D / V)) * V;
    const int64_t lh = e / (D / V);             // local token * H + head
    const int lt = (int)(lh / g.H);
    const int hh = (int)(lh % g.H);
    const int si = find_segment(st, lt);
    const int64_t tok = st.q_offset[si] + (lt - st.item0[si]);
    const int grp = hh / g.hpg, h = hh % g.hpg;
    const int64_t p0 = (tok * g.G + grp) * a.n_split * g.hpg + h;   // partial of split s: p0 + s*hpg
    float m = -INFINITY;
#pragma unroll 8
    for (int s = 0; s < a.n_split; ++s) m = fmaxf(m, a.part_ml[(p0 + (int64_t)s * g.hpg) * 2]);
    float l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int s = 0; s < a.n_split; ++s) {
      const int64_t p = p0 + (int64_t)s * g.hpg;
      const float2 ml = *reinterpret_cast<const float2*>(a.part_ml + p * 2);
      const float4 po = *reinterpret_cast<const float4*>(a.part_o + p * D + d);
      const float f = ml.x == -INFINITY ? 0.f : expf(ml.x - m);
      l += ml.y * f;
      o.x += po.x * f;
      o.y += po.y * f;
      o.z += po.z * f;
      o.w += po.w * f;
    }
    const int64_t th = tok * g.H + hh;
    T* out = (T*)a.o + th * D + d;
    out[0] = IO<T>::from_f(o.x / l);
    out[1] = IO<T>::from_f(o.y / l);
    out[2] = IO<T>::from_f(o.z / l);
    out[3] = IO<T>::from_f(o.w / l);
    if (a.lse && d == 0) a.lse[th] = m + logf(l);
  }
}

inline size_t attn_simt_smem() {
  using namespace simt_attn;
  return sizeof(float) * (kMaxHpg * kHeadDim + KC * KPAD + kMaxHpg * KC + 48);
}

}  // namespace qsa
