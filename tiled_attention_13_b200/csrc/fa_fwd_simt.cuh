// fa_fwd_simt.cuh -- exact-fp32 CUDA-core attention forward (fp32 inputs).
//
// Same method as the tensor-core kernel (page 1, "CANN ops-transformer
// FlashAttentionScore", section 分块 Tiling 的计算骨架, with page 3's
// unnormalised accumulator, "ops-nn efficient attention for AIGC", section
// 2.2), on fp32 FMAs: tf32 tensor cores would round the inputs to 10 mantissa
// bits, too coarse for the 1e-3 LSE bound at d = 64.
//
// CTA = 4 warps = 32 query rows of one (batch, head); each warp owns 8 rows.
// K/V tiles of 32 keys are staged in shared memory (K rows padded by one
// float so that lane l reading key l is bank-conflict free).  Lane l scores
// key l of the tile; row max / row sum are warp shuffles; for P V lane l owns
// output columns l, l+32, ... and receives p_key by shuffle.
#pragma once

#include "ptx.cuh"  // FA_INDEX_OK

namespace fa {

constexpr int SIMT_ROWS = 32;   // query rows per CTA
constexpr int SIMT_KEYS = 32;   // keys per KV tile
constexpr int SIMT_THREADS = 128;

struct SimtParams {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  float* lse;
  int B, H, Nq, Nkv;
  int Hkv;           // K/V heads (divides H); query head h reads K/V head h / (H / Hkv)
  int bsnd, causal;
  float scale_log2;  // scale * log2(e)
  int n_qblocks;     // ceil(Nq / SIMT_ROWS)
};

__device__ __forceinline__ long long simt_row(const SimtParams& p, int b, int h, int n, int N) {
  return p.bsnd ? ((long long)b * N + n) * p.H + h : ((long long)b * p.H + h) * N + n;
}
// Row (b, K/V head hk, key n) of k or v.
__device__ __forceinline__ long long simt_kv_row(const SimtParams& p, int b, int hk, int n) {
  return p.bsnd ? ((long long)b * p.Nkv + n) * p.Hkv + hk : ((long long)b * p.Hkv + hk) * p.Nkv + n;
}

template <int D>
constexpr int simt_smem_bytes() {
  return (SIMT_ROWS * D + SIMT_KEYS * (D + 1) + SIMT_KEYS * D) * 4;
}

template <int D>
__global__ void __launch_bounds__(SIMT_THREADS) fa_fwd_simt_kernel(SimtParams p) {
  constexpr int CPL = D / 32;  // output columns per lane
  extern __shared__ float simt_smem[];
  float(*Qs)[D] = reinterpret_cast<float(*)[D]>(simt_smem);
  float(*Ks)[D + 1] = reinterpret_cast<float(*)[D + 1]>(simt_smem + SIMT_ROWS * D);
  float(*Vs)[D] = reinterpret_cast<float(*)[D]>(simt_smem + SIMT_ROWS * D + SIMT_KEYS * (D + 1));

  const int qb = blockIdx.x % p.n_qblocks;
  const int bh = blockIdx.x / p.n_qblocks;
  const int b = bh / p.H, h = bh % p.H;
  const int hk = h / (p.H / p.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = qb * SIMT_ROWS;

  for (int idx = threadIdx.x; idx < SIMT_ROWS * D; idx += SIMT_THREADS) {
    const int r = idx / D, c = idx % D;
    const int n = row0 + r;
    const long long qi = simt_row(p, b, h, n, p.Nq) * D + c;
    Qs[r][c] = (n < p.Nq && FA_INDEX_OK(&g_status_word, qi >= 0 && qi < (long long)p.B * p.H * p.Nq * D)) ? p.q[qi]
                                                                                                        : 0.f;
  }

  float m[8], l[8], acc[8][CPL];
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int t = 0; t < CPL; ++t) acc[rr][t] = 0.f;
  }

  int kv_end = p.Nkv;
  if (p.causal) {
    const int last_row = row0 + SIMT_ROWS - 1;
    if (last_row + 1 < kv_end) kv_end = last_row + 1;
  }

  for (int kb = 0; kb < kv_end; kb += SIMT_KEYS) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < SIMT_KEYS * D; idx += SIMT_THREADS) {
      const int r = idx / D, c = idx % D;
      const int n = kb + r;
      const long long off = n < p.Nkv ? simt_kv_row(p, b, hk, n) * D + c : 0;
      const bool in = n < p.Nkv && FA_INDEX_OK(&g_status_word, off >= 0 && off < (long long)p.B * p.Hkv * p.Nkv * D);
      Ks[r][c] = in ? p.k[off] : 0.f;
      Vs[r][c] = in ? p.v[off] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int lr = warp * 8 + rr;
      const int grow = row0 + lr;
      float s = 0.f;
#pragma unroll 16
      for (int c = 0; c < D; ++c) s = fmaf(Qs[lr][c], Ks[lane][c], s);
      const int key = kb + lane;
      const bool vis = key < p.Nkv && (!p.causal || key <= grow);
      const float x = vis ? s * p.scale_log2 : -INFINITY;
      float mt = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
      const float m_new = fmaxf(m[rr], mt);
      const float ref = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = exp2f(m[rr] - ref);
      const float pv = vis ? exp2f(x - ref) : 0.f;
      float ps = pv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[rr] = l[rr] * corr + ps;
      m[rr] = m_new;
#pragma unroll
      for (int t = 0; t < CPL; ++t) acc[rr][t] *= corr;
#pragma unroll 8
      for (int kk = 0; kk < SIMT_KEYS; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, pv, kk);
#pragma unroll
        for (int t = 0; t < CPL; ++t) acc[rr][t] = fmaf(pk, Vs[kk][lane + 32 * t], acc[rr][t]);
      }
    }
  }

#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int grow = row0 + warp * 8 + rr;
    if (grow >= p.Nq) continue;
    const float inv = 1.f / l[rr];
    const long long oi = simt_row(p, b, h, grow, p.Nq) * D;
    if (!FA_INDEX_OK(&g_status_word, oi >= 0 && oi + D <= (long long)p.B * p.H * p.Nq * D)) continue;
    float* orow = p.o + oi;
#pragma unroll
    for (int t = 0; t < CPL; ++t) orow[lane + 32 * t] = acc[rr][t] * inv;
    if (p.lse != nullptr && lane == 0)
      p.lse[((long long)b * p.H + h) * p.Nq + grow] = (m[rr] + log2f(l[rr])) * 0.69314718055994530942f;
  }
}

}  // namespace fa
