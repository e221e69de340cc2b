// compress.cuh -- key pooling into micro-blocks + block rotary encoding.
//
// Design report summary page ("Qwen3.8-Next architecture design report"),
// QSA item: the indexer keys of each micro-block of r tokens are averaged,
// then position-encoded.  Here the encoding is the partial rotary encoding
// of the main attention (Miles docs "Qwen3.8-Flash-Next" section 1: rotary
// percent 0.25, base 1e7) at the block's first token position r*b.
//
// HBM-bound: reads r*DI elements and writes DI elements per block.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {

struct RangeTable {
  int32_t n;
  int32_t slot[kMaxSegs];
  int64_t b0[kMaxSegs];
  int64_t item0[kMaxSegs + 1];  // prefix of blocks per range
};

// One thread per 16-byte chunk of a block's row (8 bf16 or 4 fp32 dims): it
// loads that chunk of each of the r rows with one vector load per row (r
// loads in flight), so a warp reads whole rows in 16-byte pieces and writes
// its pooled chunk with one vector store.  The mean is formed in registers in
// the fixed order (rows summed in order, then divided by r, fp32, round to
// nearest); the rotate-half partner of a dim lives in another thread, so the
// means and the cos/sin pairs go through shared memory.
//
// late_wait: the blocks pooled here are read by no kernel before the next
// one in the stream (decode-like batches: every query's candidates predate
// this step's blocks), so the pooling runs alongside the previous kernel and
// only its exit waits for that kernel, which keeps completion order.
constexpr int kCompressThreads = 256;
constexpr int kCompressMaxDim = 128;

template <typename T>
__global__ void __launch_bounds__(kCompressThreads, 3) compress_keys_kernel(Geo g, RangeTable rt,
                                                                        const T* __restrict__ k_idx,
                                                                        T* __restrict__ khat, int late_wait) {
  constexpr int E = 16 / (int)sizeof(T);          // dims per 16-byte chunk
  // per block slot of this CTA: the means, and cos/sin of the rotated pairs
  __shared__ float s_mean[kCompressThreads * E];
  __shared__ float2 s_cs[kCompressThreads * E / 2];
  if (!late_wait) pdl_wait();
  pdl_trigger();
  const int DI = g.DI, half = g.rope_half, r = g.r;
  const int lpb = DI / E;                          // threads per block (8, 16 or 32)
  const int bpc = kCompressThreads / lpb;          // blocks per CTA pass
  const int jb = threadIdx.x / lpb;                // this thread's block slot
  const int c = threadIdx.x - jb * lpb;            // its chunk
  float* mean = s_mean + jb * DI;
  float2* cs = s_cs + jb * (DI / 2);
  const int64_t total = rt.item0[rt.n];
  const int64_t iters = cdiv(total, (int64_t)bpc * gridDim.x);
  for (int64_t it = 0; it < iters; ++it) {
    const int64_t item = (it * gridDim.x + blockIdx.x) * bpc + jb;
    const bool live = item < total;
    int64_t b = 0, slot = 0;
    if (live) {
      int lo = 0, hi = rt.n - 1;
      while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (rt.item0[mid] <= item) lo = mid; else hi = mid - 1;
      }
      b = rt.b0[lo] + (item - rt.item0[lo]);
      slot = rt.slot[lo];
      const T* rows = k_idx + (slot * g.n_cap + b * r) * DI + c * E;
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (j < r) v[j] = __ldg(reinterpret_cast<const uint4*>(rows + (int64_t)j * DI));
      float m[E];
      const T* x0 = reinterpret_cast<const T*>(&v[0]);
#pragma unroll
      for (int e = 0; e < E; ++e) m[e] = IO<T>::to_f(x0[e]);
#pragma unroll
      for (int j = 1; j < 4; ++j) {
        if (j < r) {
          const T* xj = reinterpret_cast<const T*>(&v[j]);
#pragma unroll
          for (int e = 0; e < E; ++e) m[e] = __fadd_rn(m[e], IO<T>::to_f(xj[e]));
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) mean[c * E + e] = __fdiv_rn(m[e], (float)r);
      // the block's rotated pairs, spread over its threads (the fp64 angle and
      // sincos are the costly part: one or two per thread, not eight)
      for (int i = c; i < half; i += lpb) {
        float cc, ss;
        rope_cs(g, b * r, i, cc, ss);
        cs[i] = make_float2(cc, ss);
      }
    }
    __syncthreads();
    if (live && c * E < 2 * half) {                // chunks holding rotated dims
      T out[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int d = c * E + e;
        float o = mean[d];
        if (d < half) {
          float o1;
          rope_pair(mean[d], mean[d + half], cs[d].x, cs[d].y, o, o1);
        } else if (d < 2 * half) {
          float o0;
          rope_pair(mean[d - half], mean[d], cs[d - half].x, cs[d - half].y, o0, o);
        }
        out[e] = IO<T>::from_f(o);
      }
      *reinterpret_cast<uint4*>(khat + (slot * (g.n_cap / r) + b) * DI + c * E) = *reinterpret_cast<uint4*>(out);
    } else if (live) {
      T out[E];
#pragma unroll
      for (int e = 0; e < E; ++e) out[e] = IO<T>::from_f(mean[c * E + e]);
      *reinterpret_cast<uint4*>(khat + (slot * (g.n_cap / r) + b) * DI + c * E) = *reinterpret_cast<uint4*>(out);
    }
    __syncthreads();
  }
  if (late_wait) pdl_wait();
}

template <typename T>
cudaError_t launch_compress(const Geo& g, const RangeTable& rt, const void* k_idx, void* khat,
                            cudaStream_t st, bool late_wait = false) {
  const int64_t total = rt.item0[rt.n];
  if (total == 0) return cudaSuccess;
  const int bpc = kCompressThreads / (g.DI / (16 / (int)sizeof(T)));
  int64_t blocks = cdiv(total, (int64_t)bpc);
  if (blocks > 148 * 16) blocks = 148 * 16;
  count_launch();
  return launch_chained(compress_keys_kernel<T>, dim3((unsigned)blocks), dim3(kCompressThreads), 0, st, g, rt,
                        (const T*)k_idx, (T*)khat, late_wait ? 1 : 0);
}

}  // namespace qsa
