// qsa_internal.cuh -- types and device helpers shared by the QSA kernels.
//
// The library is one translation unit (qsa_api.cu includes every kernel
// file), so file-scope device state such as the error word has one instance
// per device.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/qsa.h"

namespace qsa {

constexpr int kMaxSegs = 128;     // segments per launch: the table travels as a kernel parameter
constexpr int kHeadDim = 256;     // main attention head dim (Miles docs section 1: kv-channels 256)
constexpr int kMaxHpg = 16;       // query heads per KV group handled by one tile
constexpr int kMaxBudgetBlocks = 512;
constexpr int kMaxRopeHalf = 64;

// Layer geometry, passed by value to every kernel.
struct Geo {
  int32_t r;          // tokens per micro-block
  int32_t S;          // budget in blocks
  int32_t H;          // query heads
  int32_t G;          // KV groups
  int32_t hpg;        // heads per group
  int32_t HI;         // indexer heads
  int32_t DI;         // indexer dim
  int32_t rope_half;  // rotated dims / 2
  float scale;        // softmax scale
  int32_t n_slots;
  int64_t n_cap;      // tokens per cache slot
  double theta[kMaxRopeHalf];  // rope_base^(-2i/rope_dims), formed on the host in fp64
};

// Segment table of one launch, with a prefix sum of the work items each
// segment contributes (the kernel maps blockIdx to a segment by bisection).
// blk_lo / blk_cap restrict the blocks the indexer scores for the segment's
// queries to [blk_lo, limit), limit = blk_cap when > 0, else the causal
// limit floor(t/r); pslot / pblk: the segment's blocks below pblk live in
// cache slot pslot (a prefix shared with other sequences), the rest in slot.
struct SegTable {
  int32_t n;
  int32_t q_offset[kMaxSegs];
  int32_t q_len[kMaxSegs];
  int32_t pos0[kMaxSegs];
  int32_t slot[kMaxSegs];
  int32_t item0[kMaxSegs + 1];
  int32_t blk_lo[kMaxSegs];
  int32_t blk_cap[kMaxSegs];
  int32_t pslot[kMaxSegs];
  int32_t pblk[kMaxSegs];
};

// Per-segment fields of SegTable beyond qsa_segment_t (all zero by default).
struct SegExtra {
  int32_t blk_lo, blk_cap, pslot, pblk;
};

__device__ __forceinline__ int find_segment(const SegTable& st, int item) {
  int lo = 0, hi = st.n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (st.item0[mid] <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------- dtype traits
template <typename T> struct IO;
template <> struct IO<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct IO<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// ---------------------------------------------------------------- rotary encoding
// cos/sin of the angle pos*theta_i: the angle is formed in fp64 and the result
// rounded to fp32, so positions up to 2^20 keep full fp32 accuracy.
__device__ __forceinline__ void rope_cs(const Geo& g, int64_t pos, int i, float& c, float& s) {
  double a = (double)pos * g.theta[i];
  double sd, cd;
  sincos(a, &sd, &cd);
  c = (float)cd;
  s = (float)sd;
}

// One rotate-half pair (x_i, x_{i+half}) at angle (c, s), fp32 with every
// product rounded separately (no contraction into FMA).
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float& oa, float& ob) {
  oa = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
  ob = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

// ---------------------------------------------------------------- status word
// Written by bounded device-side waits that gave up; read by qsa_device_status().
static __device__ unsigned int g_qsa_device_error;

enum : unsigned int { kErrNone = 0, kErrWaitTimeout = 1, kErrBadIndex = 2 };

__device__ __forceinline__ void report_error(unsigned int code) {
  atomicCAS(&g_qsa_device_error, 0u, code);
}

// Rows whose selection took an exact fallback (the sampled threshold admitted
// too few or too many candidates); read and reset by qsa_select_fallbacks().
static __device__ unsigned long long g_qsa_select_fallbacks;

__device__ __forceinline__ void count_fallback() {
  if (threadIdx.x == 0) atomicAdd(&g_qsa_select_fallbacks, 1ull);
}

// Cache row of token `j_in_block` of kept block `b`, or -1 when b is not a
// block of the cache (a caller-supplied selection out of range: reported and
// skipped, never dereferenced).
__device__ __forceinline__ int64_t block_row(int32_t b, int j_in_block, const Geo& g) {
  if (b < 0 || (int64_t)b >= g.n_cap / g.r) {
    if (b != -1) report_error(kErrBadIndex);
    return -1;
  }
  return (int64_t)b * g.r + j_in_block;
}

// Host-side count of kernels this library has launched (qsa_launch_count).
inline std::atomic<long long>& launch_counter() {
  static std::atomic<long long> n{0};
  return n;
}
inline void count_launch() { launch_counter().fetch_add(1, std::memory_order_relaxed); }

// ---------------------------------------------------------------- launch chaining
// Every kernel is launched with programmatic stream serialization: it may be
// scheduled while the previous kernel of the stream is still finishing, does
// its local set-up, then waits (pdl_wait) for that kernel's completion and
// memory before touching global memory, and immediately lets the next kernel
// of the stream start scheduling (pdl_trigger).  Without the launch
// attribute both instructions are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- misc
__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// fp32 score -> uint32 key whose unsigned order is the float order (-0 -> +0).
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace qsa
