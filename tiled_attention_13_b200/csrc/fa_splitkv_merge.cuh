// fa_splitkv_merge.cuh -- the merge step of split-KV attention.
//
// The split kernel leaves, for every query row and every slice s of the key
// tiles, the attention of that row over the slice alone: O_s (normalised,
// fp32) and LSE_s.  Attention over all keys follows from those by the online
// softmax's combination rule applied to whole slices (page 1, section
// 在线 Softmax 的数学原理拆解: a running result is rescaled by the exponent of
// its max's change and summed):
//
//   LSE = m + ln sum_s exp(LSE_s - m),   m = max_s LSE_s
//   O   = sum_s exp(LSE_s - LSE) O_s
//
// The kernel is HBM-bound and tiny next to the split kernel: it reads
// n_splits * (D + 1) fp32 values per row and writes one row of O.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "pdl.cuh"
#include "ptx.cuh"  // FA_INDEX_OK

namespace fa {

constexpr int MERGE_ROWS_PER_CTA = 8;  // one warp per query row
constexpr int MERGE_THREADS = 32 * MERGE_ROWS_PER_CTA;

template <typename T>
__device__ __forceinline__ void merge_store(T* dst, const float* x, int n);

template <>
__device__ __forceinline__ void merge_store<__nv_bfloat16>(__nv_bfloat16* dst, const float* x, int n) {
  if (n == 4) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]), b = __floats2bfloat162_rn(x[2], x[3]);
    *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  } else {
    __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<uint32_t*>(&a);
  }
}

template <>
__device__ __forceinline__ void merge_store<__half>(__half* dst, const float* x, int n) {
  if (n == 4) {
    __half2 a = __floats2half2_rn(x[0], x[1]), b = __floats2half2_rn(x[2], x[3]);
    *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  } else {
    __half2 a = __floats2half2_rn(x[0], x[1]);
    *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<uint32_t*>(&a);
  }
}

// Rows are numbered r = (b * H + h) * Nq + n, the order of o_part / lse_part
// within a slice ([n_splits, B, H, Nq, D] and [n_splits, B, H, Nq]).  Lane l
// of a row's warp owns columns [l * D/32, (l + 1) * D/32).
template <int D, typename T>
__global__ void __launch_bounds__(MERGE_THREADS)
    fa_splitkv_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, T* __restrict__ o,
                            float* __restrict__ lse, int B, int H, int Nq, int n_splits, int bsnd) {
  constexpr int E = D / 32;  // 4 (d = 128) or 2 (d = 64)
  // a dependent launch: the partial results are read once the split kernel has completed
  pdl_launch_dependents();
  pdl_wait();
  const long long rows = (long long)B * H * Nq;
  const long long r = (long long)blockIdx.x * MERGE_ROWS_PER_CTA + (threadIdx.x >> 5);
  if (r >= rows) return;
  if (!FA_INDEX_OK(&g_status_word, r >= 0 && n_splits >= 1)) return;
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  for (int s = 0; s < n_splits; ++s) m = fmaxf(m, lse_part[(long long)s * rows + r]);
  const float ms = (m == -INFINITY) ? 0.f : m;  // no slice saw a key: weights 0, not NaN
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float tot = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const long long sr = (long long)s * rows + r;
    const float wgt = expf(lse_part[sr] - ms);
    tot += wgt;
    const float* src = o_part + sr * D + lane * E;
    if constexpr (E == 4) {
      const float4 x = *reinterpret_cast<const float4*>(src);
      acc[0] += wgt * x.x; acc[1] += wgt * x.y; acc[2] += wgt * x.z; acc[3] += wgt * x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(src);
      acc[0] += wgt * x.x; acc[1] += wgt * x.y;
    }
  }
  const float inv = 1.f / tot;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] *= inv;
  const int n = (int)(r % Nq);
  const long long bh = r / Nq;
  const int h = (int)(bh % H), b = (int)(bh / H);
  const long long orow = bsnd ? ((long long)b * Nq + n) * H + h : r;
  merge_store<T>(o + orow * D + lane * E, acc, E);
  if (lane == 0 && lse != nullptr) lse[r] = ms + logf(tot);
}

}  // namespace fa
