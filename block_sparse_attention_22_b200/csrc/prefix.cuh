// prefix.cuh -- rotated indexer queries of sequences that share a cached prefix.
//
// Release article on Qwen3.8-Flash-Next (tahou.com), section "GDN+QSA": the
// 1M-context figures assume a 90 % prefix-cache hit, i.e. many requests on
// one cached prefix.  When several decode queries share a prefix of P
// micro-blocks, their scores over the prefix blocks are one contraction
// against a single stream of the prefix's pooled keys: the indexer scores
// them as one capped segment (blocks [0, P), every query alike).  The
// queries of that segment come from different sequences, at different
// positions, so they are rotated here, each at its own position, into rows
// of the workspace (with their head weights and the row of their scores);
// the indexer then takes these rows as they are.
//
// The rotation is the indexer's own (the same fp32 operations, rounded to
// bf16 the same way), so a shared query's scores are bit-identical to those
// it would get alone.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {

struct PrefixRotArgs {
  const __nv_bfloat16* q_idx;   // [T][4][DI]
  const float* w;               // [T][4]
  __nv_bfloat16* q_rot;         // [V][4][DI]: virtual row v = item of the table
  float* w_rot;                 // [V][4]
  int32_t* row_map;             // [V]: the query's token row
};

// One CTA per (virtual row, indexer head); the table's items are the member
// queries of the shared segments, in order.
__global__ void __launch_bounds__(128) prefix_rotate_kernel(Geo g, SegTable st, PrefixRotArgs a) {
  pdl_wait();
  pdl_trigger();
  const int v = blockIdx.x >> 2, h = blockIdx.x & 3;
  const int si = find_segment(st, v);
  const int j = v - st.item0[si];
  const int64_t tok = st.q_offset[si] + j;
  const int64_t t = (int64_t)st.pos0[si] + j;
  const int DI = g.DI, half = g.rope_half;
  const __nv_bfloat16* x = a.q_idx + (tok * 4 + h) * (int64_t)DI;
  __nv_bfloat16* y = a.q_rot + ((int64_t)v * 4 + h) * DI;
  for (int d = threadIdx.x; d < DI; d += blockDim.x) {
    if (d < half) {
      float c, s, o0, o1;
      rope_cs(g, t, d, c, s);
      rope_pair(__bfloat162float(x[d]), __bfloat162float(x[d + half]), c, s, o0, o1);
      y[d] = __float2bfloat16_rn(o0);
      y[d + half] = __float2bfloat16_rn(o1);
    } else if (d >= 2 * half) {
      y[d] = x[d];
    }
  }
  if (threadIdx.x == 0) {
    a.w_rot[(int64_t)v * 4 + h] = a.w[tok * 4 + h];
    if (h == 0) a.row_map[v] = (int32_t)tok;
  }
}

}  // namespace qsa
