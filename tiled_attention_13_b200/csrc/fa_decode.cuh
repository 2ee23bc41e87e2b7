// fa_decode.cuh -- split-KV attention for decoding-shaped calls on CUDA
// cores: at most 8 query rows per (batch, K/V head), contiguous K/V, bf16 or
// fp16, head dim D in {64, 128}.
//
// A decoding step adds one token per sequence and attends from its query
// rows to the whole cache (page 1, "CANN ops-transformer FlashAttentionScore",
// section GatherPAKVCache 的显存管理逻辑: the step's latency is the forward
// operator's job).  With one row per head the work is one FLOP per K/V byte:
// the step is an HBM stream of K and V, and a 128-row tensor-core tile would
// compute 127 empty rows.  This kernel reads K and V once, through TMA, and
// does the arithmetic on CUDA cores.
//
// Work: the split-KV plan cuts the keys of every (batch, K/V head) into
// n_splits slices of whole 128-key tiles.  One CTA per (slice, batch, K/V
// head) takes every query row that reads this K/V head (the query heads of
// the group times Nq, R <= 8 rows).  Its four warps split the slice into
// 32-key chunks, round robin; each warp streams its chunks through a
// three-stage ring of its own (lane 0 issues the TMA loads, K and V of a
// chunk on one barrier) and keeps, per row, the online-softmax state of its
// chunks (page 1, section 在线 Softmax 的数学原理拆解): running max m, sum l and
// the unnormalised O.
//   scores  lane = key: its 32 scores (one per key) from its K row in shared
//           memory (128-byte swizzle: conflict-free across the warp) and the
//           rows' q from shared memory (broadcast);
//   softmax warp max of the scores (shuffles), p = 2^(s - m) per lane;
//   P V     lane = D/32 columns: for each of the 32 keys, p broadcast by a
//           shuffle and that key's V columns from shared memory.
// At the end the four warps' states are combined through shared memory (the
// same rule, across warps) and written as the slice's fp32 O and LSE for the
// merge kernel, or, when the plan has one slice, as the final O and LSE.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "tc_common.cuh"
#include "ptx.cuh"

namespace fa {

constexpr int DEC_WARPS = 4;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_ROWS = 8;  // query rows per (batch, K/V head) at most
constexpr int DEC_CHUNK = 32;  // keys per chunk
constexpr int DEC_ST = 3;      // ring stages per warp

template <int D>
struct DecCfg {
  static constexpr int SUB = D / 64;                    // 64-column sub-tiles of a chunk
  static constexpr int SUB_BYTES = DEC_CHUNK * 128;     // 32 rows x 128 bytes
  static constexpr int KV_BYTES = SUB * SUB_BYTES;      // one chunk of K (or V)
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;      // K then V
  static constexpr int OFF_RING = 0;                    // [warp][stage]
  static constexpr int OFF_Q = DEC_WARPS * DEC_ST * STAGE_BYTES;          // q, fp32 [R][D]
  static constexpr int OFF_RED = OFF_Q + DEC_ROWS * D * 4;                 // per warp: m, l [R], O [R][D]
  static constexpr int RED_FLOATS = DEC_ROWS * (2 + D);
  static constexpr int OFF_BAR = OFF_RED + DEC_WARPS * RED_FLOATS * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + DEC_WARPS * DEC_ST * 8 + 1024;
  static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory of sm_100");
};

struct DecParams {
  const void* q;
  void* o;           // final O when n_splits == 1, else fp32 o_part [n_splits, B, H, Nq, D]
  float* lse;        // final LSE (may be nullptr) when n_splits == 1, else lse_part [n_splits, B, H, Nq]
  int B, H, Hkv, Nq, Nkv;
  int bsnd;
  float scale_log2;
  int n_splits, split_keys;  // slice s holds keys [s * split_keys, min(Nkv, (s + 1) * split_keys))
  uint64_t timeout_ns;
};

template <typename T>
__device__ __forceinline__ void dec_unpack8(uint4 w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    } else {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
}

// RR: the rows a CTA computes, R rounded up to a power of two (1, 2, 4 or 8),
// a compile-time count so that no per-row work is predicated off; rows past R
// have q = 0 and are not stored.
template <int D, typename T, int RR>
__global__ void __launch_bounds__(DEC_THREADS, 1)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     DecParams p, unsigned int* status_word) {
  using C = DecCfg<D>;
  constexpr int E = D / 32;  // columns per lane in P V
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* qs = reinterpret_cast<float*>(smem + C::OFF_Q);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BHk = p.B * p.Hkv;
  const int sp = blockIdx.x / BHk;
  const int bhk = blockIdx.x - sp * BHk;
  const int b = bhk / p.Hkv, hk = bhk - b * p.Hkv;
  const int group = p.H / p.Hkv;
  const int R = group * p.Nq;  // rows: (query head hk * group + g, position n), row = g * Nq + n
  const int k0 = sp * p.split_keys;
  const int k1 = (k0 + p.split_keys < p.Nkv) ? k0 + p.split_keys : p.Nkv;
  const int nchunks = (k1 - k0 + DEC_CHUNK - 1) / DEC_CHUNK;

  // q of the R rows, as fp32 (zeros past R)
  for (int i = threadIdx.x; i < DEC_ROWS * D; i += DEC_THREADS) {
    const int rr = i / D, c = i - rr * D;
    float x = 0.f;
    if (rr < R) {
      const int h = hk * group + rr / p.Nq, n = rr % p.Nq;
      const long long off = p.bsnd ? (((long long)b * p.Nq + n) * p.H + h) * D : (((long long)b * p.H + h) * p.Nq + n) * D;
      const T v = static_cast<const T*>(p.q)[off + c];
      if constexpr (std::is_same<T, __nv_bfloat16>::value) x = __bfloat162float(v); else x = __half2float(v);
    }
    qs[i] = x;
  }
  if (lane == 0)
    for (int s = 0; s < DEC_ST; ++s) mbar_init(smem_u32(&bars[warp * DEC_ST + s]), 1);
  fence_barrier_init();
  __syncthreads();

  volatile int abort_local = 0;  // per-thread: the warps do not wait on one another
  WaitCtx wctx{&abort_local, status_word, p.timeout_ns, 1u};
  const uint32_t ring = sbase + C::OFF_RING + warp * DEC_ST * C::STAGE_BYTES;
  auto bar = [&](int s) { return smem_u32(&bars[warp * DEC_ST + s]); };
  const uint64_t pol = l2_policy_evict_first();
  // this warp's chunks: warp, warp + 4, ...
  const int mine = nchunks > warp ? (nchunks - warp + DEC_WARPS - 1) / DEC_WARPS : 0;
  auto issue = [&](int j) {  // load this warp's j-th chunk into stage j % DEC_ST
    const int key = k0 + (warp + j * DEC_WARPS) * DEC_CHUNK;
    const uint32_t dst = ring + (j % DEC_ST) * C::STAGE_BYTES;
    mbar_arrive_expect_tx(bar(j % DEC_ST), C::STAGE_BYTES);
    for (int c = 0; c < C::SUB; ++c) {
      if (p.bsnd) {
        tma_load_4d(dst + c * C::SUB_BYTES, &tm_k, bar(j % DEC_ST), c * 64, hk, key, b, pol);
        tma_load_4d(dst + C::KV_BYTES + c * C::SUB_BYTES, &tm_v, bar(j % DEC_ST), c * 64, hk, key, b, pol);
      } else {
        tma_load_4d(dst + c * C::SUB_BYTES, &tm_k, bar(j % DEC_ST), c * 64, key, hk, b, pol);
        tma_load_4d(dst + C::KV_BYTES + c * C::SUB_BYTES, &tm_v, bar(j % DEC_ST), c * 64, key, hk, b, pol);
      }
    }
  };
  if (lane == 0)
    for (int j = 0; j < DEC_ST && j < mine; ++j) issue(j);
  __syncwarp();

  float m[RR], l[RR], acc[RR][E];
#pragma unroll
  for (int r = 0; r < RR; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[r][e] = 0.f;
  }
  const float sl2 = p.scale_log2;
  int done = 0;  // chunks consumed (their stage may be refilled)
  for (int j = 0; j < mine; ++j) {
    const int st = j % DEC_ST;
    if (!__all_sync(0xffffffffu, mbar_wait(bar(st), (j / DEC_ST) & 1, wctx))) break;
    const uint32_t kb = ring + st * C::STAGE_BYTES, vb = kb + C::KV_BYTES;
    const int key = k0 + (warp + j * DEC_WARPS) * DEC_CHUNK + lane;  // this lane's key
    // scores: lane = key
    float s[RR], s2[RR];  // two partial sums per row: shorter FMA chains
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] = s2[r] = 0.f;
#pragma unroll
    for (int c = 0; c < C::SUB; ++c) {
#pragma unroll
      for (int pc = 0; pc < 8; ++pc) {
        uint4 w;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                     : "r"(kb + c * C::SUB_BYTES + lane * 128 + ((pc ^ (lane & 7)) << 4)));
        float kf[8];
        dec_unpack8<T>(w, kf);
#pragma unroll
        for (int r = 0; r < RR; ++r) {
          {
            const float4 qa = *reinterpret_cast<const float4*>(qs + r * D + c * 64 + pc * 8);
            const float4 qb = *reinterpret_cast<const float4*>(qs + r * D + c * 64 + pc * 8 + 4);
            s[r] = fmaf(qa.x, kf[0], s[r]); s2[r] = fmaf(qa.y, kf[1], s2[r]);
            s[r] = fmaf(qa.z, kf[2], s[r]); s2[r] = fmaf(qa.w, kf[3], s2[r]);
            s[r] = fmaf(qb.x, kf[4], s[r]); s2[r] = fmaf(qb.y, kf[5], s2[r]);
            s[r] = fmaf(qb.z, kf[6], s[r]); s2[r] = fmaf(qb.w, kf[7], s2[r]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] += s2[r];
    const bool live = key < k1;
    float pr[RR];
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      const float x = live ? s[r] * sl2 : -INFINITY;
      float mx = x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m[r], mx);  // finite: every chunk has a live key 0
      const float corr = ex2(m[r] - m_new);  // 0 when m[r] = -inf
      m[r] = m_new;
      pr[r] = ex2(x - m_new);
      l[r] = l[r] * corr + pr[r];  // this lane's share; summed over lanes at the end
#pragma unroll
      for (int e = 0; e < E; ++e) acc[r][e] *= corr;
    }
    // P V: lane = columns [lane * E, lane * E + E)
    const int cb = lane * E * 2;  // byte offset of this lane's columns in a key row
#pragma unroll 4
    for (int kk = 0; kk < DEC_CHUNK; ++kk) {
      const uint32_t vrow = vb + (cb >> 7) * C::SUB_BYTES + kk * 128;
      const uint32_t piece = ((cb & 127) >> 4) ^ (kk & 7);
      float vf[8];  // the first E are this lane's columns
      if constexpr (E == 4) {
        uint32_t w0, w1;
        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(vrow + (piece << 4) + (cb & 15)));
        dec_unpack8<T>(make_uint4(w0, w1, 0u, 0u), vf);
      } else {
        uint32_t w0;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(vrow + (piece << 4) + (cb & 15)));
        dec_unpack8<T>(make_uint4(w0, 0u, 0u, 0u), vf);
      }
#pragma unroll
      for (int r = 0; r < RR; ++r) {
        const float pk = __shfl_sync(0xffffffffu, pr[r], kk);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[r][e] = fmaf(pk, vf[e], acc[r][e]);
      }
    }
    __syncwarp();
    ++done;
    // the stage is read: refill it with this warp's chunk j + DEC_ST
    if (lane == 0 && j + DEC_ST < mine) issue(j + DEC_ST);
    __syncwarp();
  }
  // Every copy this warp started lands before the CTA may exit.
  if (lane == 0) {
    WaitCtx drain{&abort_local, status_word, p.timeout_ns, 1u};
    for (int j = done; j < mine && j < done + DEC_ST; ++j) mbar_wait(bar(j % DEC_ST), (j / DEC_ST) & 1, drain);
  }
  // this warp's state into shared memory: m, l (summed over lanes), O
  float* rw = red + warp * C::RED_FLOATS;
#pragma unroll
  for (int r = 0; r < RR; ++r) {
    float lt = l[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
    if (lane == 0) {
      rw[r] = (done == mine && mine > 0) ? m[r] : -INFINITY;
      rw[DEC_ROWS + r] = lt;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) rw[2 * DEC_ROWS + r * D + lane * E + e] = acc[r][e];
  }
  __syncthreads();
  // combine the four warps' states, row by row, in warp 0 (lane = columns)
  if (warp == 0) {
    for (int r = 0; r < R; ++r) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < DEC_WARPS; ++w) mm = fmaxf(mm, red[w * C::RED_FLOATS + r]);
      const float ms = (mm == -INFINITY) ? 0.f : mm;
      float lt = 0.f, o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = 0.f;
#pragma unroll
      for (int w = 0; w < DEC_WARPS; ++w) {
        const float* rv = red + w * C::RED_FLOATS;
        const float f = ex2(rv[r] - ms);  // 0 for a warp without keys
        lt += f * rv[DEC_ROWS + r];
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(f, rv[2 * DEC_ROWS + r * D + lane * E + e], o[e]);
      }
      const float inv = 1.f / lt;
      const int h = hk * group + r / p.Nq, n = r % p.Nq;
      const float lse_r = (ms + __log2f(lt)) * 0.69314718055994530942f;
      if (p.n_splits > 1) {
        const long long prow = (((long long)sp * p.B + b) * p.H + h) * p.Nq + n;
        float* op = static_cast<float*>(p.o) + prow * D + lane * E;
        if (FA_INDEX_OK(status_word, prow < (long long)p.n_splits * p.B * p.H * p.Nq)) {
#pragma unroll
          for (int e = 0; e < E; ++e) op[e] = o[e] * inv;
          if (lane == 0) p.lse[prow] = lse_r;
        }
      } else {
        const long long orow = p.bsnd ? ((long long)b * p.Nq + n) * p.H + h : ((long long)b * p.H + h) * p.Nq + n;
        T* op = static_cast<T*>(p.o) + orow * D + lane * E;
        if (FA_INDEX_OK(status_word, orow < (long long)p.B * p.H * p.Nq)) {
#pragma unroll
          for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(op + e) = sh_pack2<T>(o[e] * inv, o[e + 1] * inv);
          if (lane == 0 && p.lse != nullptr) p.lse[((long long)b * p.H + h) * p.Nq + n] = lse_r;
        }
      }
    }
  }
}

}  // namespace fa
