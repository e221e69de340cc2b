// index_simt.cuh -- indexer scores on CUDA cores (fp32 I/O path).
//
// Design report summary page, QSA item: a 4-head MQA indexer scores every
// micro-block; DSA-style score s(t,b) = sum_h w[t,h] * ReLU(q~[t,h] . k^[b]).
// The rotated query q~ = RoPE_t(q_idx) is formed in the kernel with the same
// fp32 operation order as the key pooling and rounded to the I/O dtype.
//
// Tile: QT query tokens x BT blocks per CTA; one thread per block, QT*HI
// accumulators per thread; rotated queries live in shared memory.
#pragma once
#include "qsa_internal.cuh"

namespace qsa {

namespace simt_index {
constexpr int QT = 8;     // query tokens per tile
constexpr int BT = 256;   // blocks per tile (one per thread)
}

// Rotates QT query tokens of a segment into shared memory (fp32 copies of the
// I/O-dtype values).  Rows past the segment end are zero.
template <typename T>
__device__ void rotate_queries_to_smem(const Geo& g, const T* __restrict__ q_idx, int64_t tok0, int nq,
                                       int64_t pos_first, float* qr, int n_tok_tile) {
  const int DI = g.DI, HI = g.HI, half = g.rope_half;
  const int total = n_tok_tile * HI * DI;
  for (int e = threadIdx.x; e < total; e += blockDim.x) {
    const int qi = e / (HI * DI);
    const int rem = e - qi * HI * DI;
    const int d = rem % DI;
    if (qi >= nq) { qr[e] = 0.f; continue; }
    if (d >= half && d < 2 * half) continue;
    const T* src = q_idx + (tok0 + qi) * (int64_t)HI * DI + rem - d;
    if (d < half) {
      float c, s, o0, o1;
      rope_cs(g, pos_first + qi, d, c, s);
      rope_pair(IO<T>::to_f(src[d]), IO<T>::to_f(src[d + half]), c, s, o0, o1);
      qr[e] = IO<T>::to_f(IO<T>::from_f(o0));
      qr[e + half] = IO<T>::to_f(IO<T>::from_f(o1));
    } else {
      qr[e] = IO<T>::to_f(src[d]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(simt_index::BT) index_scores_simt_kernel(
    Geo g, SegTable st, const T* __restrict__ q_idx, const float* __restrict__ w,
    const T* __restrict__ khat, float* __restrict__ scores, int64_t ld) {
  pdl_wait();
  pdl_trigger();
  using namespace simt_index;
  extern __shared__ float smem[];
  const int HI = g.HI, DI = g.DI;
  float* qr = smem;                       // [QT][HI][DI]
  float* ws = smem + QT * HI * DI;        // [QT][HI]

  const int item = blockIdx.x;
  const int si = find_segment(st, item);
  const int local = item - st.item0[si];
  const int q_len = st.q_len[si];
  const int64_t pos0 = st.pos0[si];
  const int64_t nblk_max = (pos0 + q_len - 1) / g.r;
  const int n_bt = (int)cdiv(nblk_max, BT);
  const int qt = local / n_bt, bt = local - qt * n_bt;
  const int q0 = qt * QT;
  const int nq = min(QT, q_len - q0);
  const int64_t b0 = (int64_t)bt * BT;
  const int64_t last_bt = (pos0 + q0 + nq - 1) / g.r;   // blocks in reach of the last query
  if (b0 >= last_bt) return;

  const int64_t tok0 = st.q_offset[si] + q0;
  rotate_queries_to_smem<T>(g, q_idx, tok0, nq, pos0 + q0, qr, QT);
  for (int e = threadIdx.x; e < QT * HI; e += blockDim.x)
    ws[e] = (e / HI < nq) ? w[tok0 * HI + e] : 0.f;
  __syncthreads();

  const int64_t b = b0 + threadIdx.x;
  if (b >= last_bt) return;
  const T* kb = khat + ((int64_t)st.slot[si] * (g.n_cap / g.r) + b) * DI;
  float acc[QT][4];
#pragma unroll
  for (int i = 0; i < QT; ++i)
#pragma unroll
    for (int h = 0; h < 4; ++h) acc[i][h] = 0.f;
  for (int d = 0; d < DI; ++d) {
    const float kv = IO<T>::to_f(kb[d]);
#pragma unroll
    for (int i = 0; i < QT; ++i)
#pragma unroll
      for (int h = 0; h < 4; ++h) acc[i][h] = fmaf(qr[(i * HI + h) * DI + d], kv, acc[i][h]);
  }
  for (int i = 0; i < nq; ++i) {
    const int64_t t = pos0 + q0 + i;
    if (b >= t / g.r) continue;
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < 4; ++h) s += ws[i * HI + h] * fmaxf(acc[i][h], 0.f);
    scores[(tok0 + i) * ld + b] = s;
  }
}

inline int simt_index_items(int q_len, int pos0, int r) {
  if (q_len <= 0) return 0;
  int64_t nblk_max = ((int64_t)pos0 + q_len - 1) / r;
  return (int)(cdiv(q_len, simt_index::QT) * cdiv(nblk_max, simt_index::BT));
}

template <typename T>
cudaError_t launch_index_simt(const Geo& g, const SegTable& st, const void* q_idx, const float* w,
                              const void* khat, float* scores, int64_t ld, cudaStream_t s) {
  using namespace simt_index;
  const int items = st.item0[st.n];
  if (items == 0) return cudaSuccess;
  size_t smem = sizeof(float) * (QT * g.HI * g.DI + QT * g.HI);
  count_launch();
  return launch_chained(index_scores_simt_kernel<T>, dim3(items), dim3(BT), smem, s, g, st, (const T*)q_idx, w,
                        (const T*)khat,
                        scores, ld);
}

}  // namespace qsa
