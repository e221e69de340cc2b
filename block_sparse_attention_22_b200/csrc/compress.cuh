// compress.cuh -- key pooling into micro-blocks + block rotary encoding.
//
// Design report summary page ("Qwen3.8-Next architecture design report"),
// QSA item: the indexer keys of each micro-block of r tokens are averaged,
// then position-encoded.  Here the encoding is the partial rotary encoding
// of the main attention (Miles docs "Qwen3.8-Flash-Next" section 1: rotary
// percent 0.25, base 1e7) at the block's first token position r*b.
//
// HBM-bound: reads r*DI elements and writes DI elements per block.  One
// thread per (block, dim); consecutive threads read consecutive dims, so a
// warp reads whole 64/128-byte row segments.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {

struct RangeTable {
  int32_t n;
  int32_t slot[kMaxSegs];
  int64_t b0[kMaxSegs];
  int64_t item0[kMaxSegs + 1];  // prefix of blocks per range
};

template <typename T>
// late_wait: the blocks pooled here are read by no kernel before the next
// one in the stream (decode-like batches: every query's candidates predate
// this step's blocks), so the pooling runs alongside the previous kernel and
// only its exit waits for that kernel, which keeps completion order.
__global__ void __launch_bounds__(256) compress_keys_kernel(Geo g, RangeTable rt, const T* __restrict__ k_idx,
                                                           T* __restrict__ khat, int late_wait) {
  if (!late_wait) pdl_wait();
  pdl_trigger();
  const int DI = g.DI, half = g.rope_half, r = g.r;
  const int64_t total = rt.item0[rt.n] * DI;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t item = e / DI;
    const int d = (int)(e - item * DI);
    if (d >= half && d < 2 * half) continue;     // written by the partner thread
    int lo = 0, hi = rt.n - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (rt.item0[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int64_t b = rt.b0[lo] + (item - rt.item0[lo]);
    const int64_t slot = rt.slot[lo];
    const T* rows = k_idx + (slot * g.n_cap + b * r) * DI;
    T* out = khat + (slot * (g.n_cap / r) + b) * DI;
    // mean over the r rows, summed in row order, in fp32
    float m0 = IO<T>::to_f(rows[d]);
    for (int j = 1; j < r; ++j) m0 = __fadd_rn(m0, IO<T>::to_f(rows[(int64_t)j * DI + d]));
    m0 = __fdiv_rn(m0, (float)r);
    if (d < half) {
      float m1 = IO<T>::to_f(rows[d + half]);
      for (int j = 1; j < r; ++j) m1 = __fadd_rn(m1, IO<T>::to_f(rows[(int64_t)j * DI + d + half]));
      m1 = __fdiv_rn(m1, (float)r);
      float c, s, o0, o1;
      rope_cs(g, b * r, d, c, s);
      rope_pair(m0, m1, c, s, o0, o1);
      out[d] = IO<T>::from_f(o0);
      out[d + half] = IO<T>::from_f(o1);
    } else {
      out[d] = IO<T>::from_f(m0);
    }
  }
  if (late_wait) pdl_wait();
}

template <typename T>
cudaError_t launch_compress(const Geo& g, const RangeTable& rt, const void* k_idx, void* khat,
                            cudaStream_t st, bool late_wait = false) {
  int64_t total = rt.item0[rt.n] * g.DI;
  if (total == 0) return cudaSuccess;
  int64_t blocks = cdiv(total, 256);
  if (blocks > 148 * 64) blocks = 148 * 64;
  count_launch();
  return launch_chained(compress_keys_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, st, g, rt, (const T*)k_idx,
                        (T*)khat, late_wait ? 1 : 0);
}

}  // namespace qsa
