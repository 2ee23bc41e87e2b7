// fa_decode.cuh -- split-KV attention for decoding-shaped calls on CUDA
// cores: at most 8 query rows per (batch, K/V head), K/V contiguous or in a
// paged cache (blocks of 16 or more keys), bf16 or fp16, head dim D in
// {64, 128}.
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
// the group times Nq, R <= 8 rows).  Its six warps split the slice into
// 16-key chunks, round robin; each warp streams its chunks through a
// two-stage ring of its own (lane 0 issues the TMA loads, K and V of a
// chunk on one barrier) and keeps, per row, the online-softmax state of its
// chunks (page 1, section 在线 Softmax 的数学原理拆解): running max m, sum l and
// the unnormalised O.  A CTA takes about 100 KB of shared memory, so two
// share an SM: twelve warps keep loads in flight and hide one another's
// latency (against eight warps with three-stage rings, the paged step ran
// 7 % faster and the contiguous one 1 %).
//   scores  lanes l and l + 16 = key l: each takes half of its K row in
//           shared memory (128-byte swizzle: conflict-free across the warp)
//           against the rows' q (shared memory, broadcast), and one shuffle
//           adds the halves;
//   softmax max over the 16 keys (shuffles), p = 2^(s - m) per lane;
//   P V     lane = D/32 columns: for each of the 16 keys, p broadcast by a
//           shuffle and that key's V columns from shared memory.
// At the end the six warps' states are combined through shared memory (the
// same rule, across warps) and written as the slice's fp32 O and LSE for the
// merge kernel, or, when the plan has one slice, as the final O and LSE.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "tc_common.cuh"
#include "pdl.cuh"
#include "ptx.cuh"

namespace fa {

constexpr int DEC_WARPS = 6;
constexpr int DEC_THREADS = 32 * DEC_WARPS;
constexpr int DEC_ROWS = 8;  // query rows per (batch, K/V head) at most
constexpr int DEC_CHUNK = 16;  // keys per chunk
constexpr int DEC_ST = 2;      // ring stages per warp
constexpr int DEC_CTAS_PER_SM = 2;

template <int D>
struct DecCfg {
  static constexpr int SUB = D / 64;                    // 64-column sub-tiles of a chunk
  static constexpr int SUB_BYTES = DEC_CHUNK * 128;     // 16 rows x 128 bytes
  static constexpr int KV_BYTES = SUB * SUB_BYTES;      // one chunk of K (or V)
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;      // K then V
  static constexpr int RING_BYTES = DEC_ST * STAGE_BYTES;  // one warp's ring
  static constexpr int OFF_RING = 0;                    // [warp][stage]
  static constexpr int OFF_Q = DEC_WARPS * RING_BYTES;  // q, fp32 [R][D]
  // per warp, after its ring has drained: m, l [R], O [R][D] in its own ring
  static constexpr int RED_FLOATS = DEC_ROWS * (2 + D);
  static_assert(RED_FLOATS * 4 <= RING_BYTES, "a warp's state must fit in its ring");
  static constexpr int OFF_BAR = OFF_Q + DEC_ROWS * D * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + DEC_WARPS * DEC_ST * 8 + 1024;
  // two CTAs per SM (228 KB, 1 KB of it reserved per CTA)
  static_assert(DEC_CTAS_PER_SM * (SMEM_BYTES + 1024) <= 233472, "two CTAs must share an SM");
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
  // paged K / V (block_table != nullptr): caches [num_blocks, bs, Hkv, D],
  // key j of sequence b in block block_table[b * max_blocks + j / bs] at row
  // j % bs; bs = 2^bs_log2 >= 16, so a 16-key chunk lies in one block
  const int* block_table;
  int max_blocks, bs_log2;
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
// have q = 0 and are not stored.  PAGED: K / V through the block table (a
// separate instantiation: the table logic costs the contiguous case about
// 10 % when it is a runtime branch).
template <int D, typename T, int RR, bool PAGED>
__global__ void __launch_bounds__(DEC_THREADS, DEC_CTAS_PER_SM)
    fa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     DecParams p, unsigned int* status_word) {
  using C = DecCfg<D>;
  constexpr int E = D / 32;  // columns per lane in P V
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* qs = reinterpret_cast<float*>(smem + C::OFF_Q);
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

  // Launched as a dependent launch: the next kernel may start its prologue as
  // this grid's CTAs exit; this one reads q, K and V only once the previous
  // kernel of the stream has completed.
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  pdl_wait();
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
  // Paged caches: the physical block of each of this warp's chunks, read 32
  // chunks at a time (lane i holds chunk base + i) one batch ahead, so the
  // table read is not on the load issue's path.
  constexpr bool paged = PAGED;  // p.block_table != nullptr
  auto table_entry = [&](int jj) -> int {
    if (jj >= mine) return 0;
    const int lb = (k0 + (warp + jj * DEC_WARPS) * DEC_CHUNK) >> p.bs_log2;
    const long long ti = (long long)b * p.max_blocks + lb;
    return FA_INDEX_OK(status_word, lb < p.max_blocks) ? p.block_table[ti] : 0;
  };
  int tb_base = 0, tb_cur = 0, tb_nxt = 0;
  if (paged) {
    tb_cur = table_entry(lane);
    tb_nxt = table_entry(32 + lane);
  }
  auto chunk_block = [&](int jj) -> int {  // whole warp: the physical block of chunk jj (jj ascending)
    if (!paged) return 0;
    if (jj - tb_base >= 32) {
      tb_base += 32;
      tb_cur = tb_nxt;
      tb_nxt = table_entry(tb_base + 32 + lane);
    }
    return __shfl_sync(0xffffffffu, tb_cur, jj - tb_base);
  };
  auto issue = [&](int j, int blk) {  // load this warp's j-th chunk into stage j % DEC_ST
    const int key = k0 + (warp + j * DEC_WARPS) * DEC_CHUNK;
    const uint32_t dst = ring + (j % DEC_ST) * C::STAGE_BYTES;
    mbar_arrive_expect_tx(bar(j % DEC_ST), C::STAGE_BYTES);
    for (int c = 0; c < C::SUB; ++c) {
      if (paged) {
        const int row = key & ((1 << p.bs_log2) - 1);
        tma_load_4d(dst + c * C::SUB_BYTES, &tm_k, bar(j % DEC_ST), c * 64, hk, row, blk, pol);
        tma_load_4d(dst + C::KV_BYTES + c * C::SUB_BYTES, &tm_v, bar(j % DEC_ST), c * 64, hk, row, blk, pol);
      } else if (p.bsnd) {
        tma_load_4d(dst + c * C::SUB_BYTES, &tm_k, bar(j % DEC_ST), c * 64, hk, key, b, pol);
        tma_load_4d(dst + C::KV_BYTES + c * C::SUB_BYTES, &tm_v, bar(j % DEC_ST), c * 64, hk, key, b, pol);
      } else {
        tma_load_4d(dst + c * C::SUB_BYTES, &tm_k, bar(j % DEC_ST), c * 64, key, hk, b, pol);
        tma_load_4d(dst + C::KV_BYTES + c * C::SUB_BYTES, &tm_v, bar(j % DEC_ST), c * 64, key, hk, b, pol);
      }
    }
  };
  for (int j = 0; j < DEC_ST && j < mine; ++j) {
    const int blk = chunk_block(j);
    if (lane == 0) issue(j, blk);
  }
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
    if (paged) {
      // The last chunk of a paged sequence: its rows past k1 are the block's
      // other contents, not zeros; clear those V rows so that p = 0 meets 0
      // (0 * NaN would be NaN).  The refill of this stage comes after a fence.
      const int live = k1 - (k0 + (warp + j * DEC_WARPS) * DEC_CHUNK);
      if (live < DEC_CHUNK) {
        for (int i = lane; i < (DEC_CHUNK - live) * 8 * C::SUB; i += 32) {
          const int rr = live + i / (8 * C::SUB), c = (i / 8) % C::SUB, q16 = i % 8;
          st_shared_v4(vb + c * C::SUB_BYTES + rr * 128 + q16 * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
    }
    const int kl = lane & 15, half = lane >> 4;  // key of the chunk, half of the row
    const int key = k0 + (warp + j * DEC_WARPS) * DEC_CHUNK + kl;  // this lane's key
    // scores: lanes kl and kl + 16 = key kl, each over D / 2 columns
    float s[RR], s2[RR];  // two partial sums per row: shorter FMA chains
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] = s2[r] = 0.f;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
      const int col = half * (D / 2) + i * 8;  // first of the 8 columns of this piece
      const int c = col >> 6, pc = (col & 63) >> 3;
      uint4 w;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                   : "r"(kb + c * C::SUB_BYTES + kl * 128 + ((pc ^ (kl & 7)) << 4)));
      float kf[8];
      dec_unpack8<T>(w, kf);
#pragma unroll
      for (int r = 0; r < RR; ++r) {
        const float4 qa = *reinterpret_cast<const float4*>(qs + r * D + col);
        const float4 qb = *reinterpret_cast<const float4*>(qs + r * D + col + 4);
        s[r] = fmaf(qa.x, kf[0], s[r]); s2[r] = fmaf(qa.y, kf[1], s2[r]);
        s[r] = fmaf(qa.z, kf[2], s[r]); s2[r] = fmaf(qa.w, kf[3], s2[r]);
        s[r] = fmaf(qb.x, kf[4], s[r]); s2[r] = fmaf(qb.y, kf[5], s2[r]);
        s[r] = fmaf(qb.z, kf[6], s[r]); s2[r] = fmaf(qb.w, kf[7], s2[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      s[r] += s2[r];
      s[r] += __shfl_xor_sync(0xffffffffu, s[r], 16);  // both halves of the row
    }
    const bool live = key < k1;
    float pr[RR];
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      const float x = live ? s[r] * sl2 : -INFINITY;
      float mx = x;  // over the 16 keys (lanes 16-31 repeat lanes 0-15)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m[r], mx);  // finite: every chunk has a live key 0
      const float corr = ex2(m[r] - m_new);  // 0 when m[r] = -inf
      m[r] = m_new;
      pr[r] = ex2(x - m_new);
      l[r] = l[r] * corr + (half == 0 ? pr[r] : 0.f);  // this key's share, once; summed over lanes at the end
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
    if (j + DEC_ST < mine) {
      const int blk = chunk_block(j + DEC_ST);
      if (lane == 0) issue(j + DEC_ST, blk);
    }
    __syncwarp();
  }
  // Every copy this warp started lands before the CTA may exit.
  if (lane == 0) {
    WaitCtx drain{&abort_local, status_word, p.timeout_ns, 1u};
    for (int j = done; j < mine && j < done + DEC_ST; ++j) mbar_wait(bar(j % DEC_ST), (j / DEC_ST) & 1, drain);
  }
  // this warp's state into shared memory, in its own (drained) ring: m, l
  // (summed over lanes), O
  __syncwarp();
  float* rw = reinterpret_cast<float*>(smem + C::OFF_RING + warp * C::RING_BYTES);
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
  // combine the warps' states, row by row, in warp 0 (lane = columns)
  if (warp == 0) {
    for (int r = 0; r < R; ++r) {
      float mm = -INFINITY;
#pragma unroll
      for (int w = 0; w < DEC_WARPS; ++w)
        mm = fmaxf(mm, reinterpret_cast<const float*>(smem + C::OFF_RING + w * C::RING_BYTES)[r]);
      const float ms = (mm == -INFINITY) ? 0.f : mm;
      float lt = 0.f, o[E];
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = 0.f;
#pragma unroll
      for (int w = 0; w < DEC_WARPS; ++w) {
        const float* rv = reinterpret_cast<const float*>(smem + C::OFF_RING + w * C::RING_BYTES);
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
