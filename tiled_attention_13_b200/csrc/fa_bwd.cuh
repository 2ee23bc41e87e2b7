// fa_bwd.cuh -- the backward pass of the attention forward on tcgen05 tensor
// cores, bf16 or fp16 inputs, fp32 accumulation, head dim D in {64, 128}.
//
// Method (page 1, "CANN ops-transformer FlashAttentionScore", section
// 反向传播的重算策略及其合理性: the forward keeps only its row statistics, and
// the backward rebuilds each tile of P from Q, K and them instead of reading a
// stored N x N matrix).  With S = scale Q K^T, P = exp(S - LSE) (LSE the
// forward's per-row log-sum-exp), and D_i = sum_c dO_ic O_ic:
//
//   dV = P^T dO,   dP = dO V^T,   dS = P o (dP - D),
//   dQ = scale dS K,   dK = scale dS^T Q.
//
// Three kernels go out on the stream:
//   fa_bwd_pre_kernel    D and LSE * log2(e) per query row, into the caller's
//                        workspace, padded to whole 128-row tiles (padding:
//                        LSE = +inf, so P = 0 there, and D = 0).
//   fa_bwd_kernel        one CTA per (batch, K/V head, 128-key tile), head-major, keeping
//                        that tile's K and V in shared memory and its dK and
//                        dV in tensor memory while it walks every query tile
//                        of every query head that reads this K/V head (under
//                        a causal mask only the query tiles at or after the
//                        key tile).  dQ of each step is added to an fp32
//                        accumulator in the workspace (vector reductions).
//   fa_bwd_post_kernel   dQ = scale * accumulator, rounded to the input dtype.
//
// fa_bwd_kernel, per query tile (step s):
//   warp 5      TMA: K, V once; Q(s) and dO(s) into a two-stage ring.
//   warp 4      MMA issuer (whole warp, elect.sync):
//                 S^T = K Q^T -> R_S;  dP^T = V dO^T -> R_DP;
//                 then, once P^T and dS^T are written:
//                 dV += P^T dO (A = P^T from TMEM), dK += dS^T Q (A = dS^T
//                 from TMEM), dQ = dS K (A = dS from shared memory, read
//                 M-major from the transposed tile) -> R_DQ.
//   warps 0-3   one key row (one TMEM lane) per thread: P^T = 2^(S^T scale
//               log2 e - LSE log2 e) for its 128 query columns (the column
//               statistics come from the workspace by uniform vector loads),
//               then dS^T = P^T o (dP^T - D); P^T and dS^T go back to tensor
//               memory as 16-bit pairs, dS^T also to shared memory in the
//               128-byte-swizzled layout; then the thread reads one query row
//               of dQ and adds it to the accumulator (vector reductions).
//               After the last step it
//               writes its key row of dV and scale * dK.
//
// TMEM (512 columns): R_S [0, 128), R_DP [128, 256), dV [256, 256 + D),
// dK [256 + D, 256 + 2D); R_DQ is [256 + 2D, 256 + 3D) when D = 64, and R_DP
// when D = 128 (the next dP^T then waits until this dQ has been read out,
// while the next S^T, in R_S, need not).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "tc_common.cuh"
#include "ptx.cuh"

namespace fa {

#ifndef FA_BWD_BULK_DQ
#define FA_BWD_BULK_DQ 0
#endif
// 0 (default): dQ rows reach the accumulator as per-thread 16-byte vector
// reductions; 1: as bulk reductions from shared memory (one per thread and 32
// columns), measured slower on the LLaMA-13B 8K backward (310 against 383
// TFLOP/s).
constexpr int BWD_BULK_DQ = FA_BWD_BULK_DQ;
constexpr int BWD_WARP_MMA = 4;
constexpr int BWD_WARP_TMA = 5;
constexpr int BWD_THREADS = 32 * 6;

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int QST = 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = TILE_BYTES;
  static constexpr int OFF_Q = 2 * TILE_BYTES;
  static constexpr int OFF_DO = OFF_Q + QST * TILE_BYTES;
  static constexpr int OFF_DS = OFF_DO + QST * TILE_BYTES;  // dS^T, 128 keys x 128 queries, 16-bit
  static constexpr int OFF_BAR = OFF_DS + 128 * 128 * 2;
  // kv_full qd_full[QST] qd_empty[QST] s_full dp_full p_ready dq_full dq_free ds_free dkdv_full drain
  static constexpr int NBAR = 1 + 2 * QST + 8;
  static constexpr int USED = OFF_BAR + NBAR * 8 + 16 + 1024;
  // At least 120 KB, so that one CTA (and its 512 TMEM columns) fits an SM.
  static constexpr int SMEM_BYTES = USED > 120 * 1024 ? USED : 120 * 1024;
  static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory of sm_100");
  static constexpr uint32_t R_S = 0, R_DP = 128, R_DV = 256, R_DK = 256 + D;
  static constexpr uint32_t R_DQ = (D == 64) ? 256 + 2 * D : R_DP;
};

struct BwdParams {
  const void* o;       // forward output, for D (pre kernel)
  const void* dout;    // dO (pre kernel)
  const float* lse;    // forward LSE [B, H, Nq] (pre kernel)
  float* lse2;         // workspace: LSE * log2(e) [B, H, nq_pad], +inf on padding rows
  float* delta;        // workspace: D [B, H, nq_pad], 0 on padding rows
  float* dq_acc;       // workspace: fp32 [B, H, Nq, D]
  void* dq;            // outputs, q's / k's layout and dtype
  void* dk;
  void* dv;
  int B, H, Hkv, Nq, Nkv;
  int bsnd, causal;
  float scale, scale_log2;
  int qtiles, kvtiles, nq_pad;
  uint64_t timeout_ns;
};

// Instruction descriptor, kind::f16 with fp32 accumulation, either operand
// K-major (false) or MN-major (true): bits [4,6) D format 1 (f32), [7,10) A
// and [10,13) B format (0 f16, 1 bf16), bit 15 A major, bit 16 B major,
// [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t bwd_idesc(bool bf16, bool a_mn, bool b_mn, uint32_t M, uint32_t N) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

template <typename T>
__device__ __forceinline__ float bwd_to_f(T x);
template <>
__device__ __forceinline__ float bwd_to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float bwd_to_f<__half>(__half x) { return __half2float(x); }

// Element offset of row n of (b, h) in a [B,H,N,D] (BHND) or [B,N,H,D] tensor.
__host__ __device__ __forceinline__ long long bwd_row(int bsnd, int b, int h, int n, int H, int N, int D) {
  return bsnd ? (((long long)b * N + n) * H + h) * D : (((long long)b * H + h) * N + n) * D;
}

// One thread per padded query row: D = sum dO o O (fp32), LSE * log2 e.
template <int D, typename T>
__global__ void fa_bwd_pre_kernel(BwdParams p) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long rows = (long long)p.B * p.H * p.nq_pad;
  if (idx >= rows) return;
  const int n = (int)(idx % p.nq_pad);
  const long long bh = idx / p.nq_pad;
  const int h = (int)(bh % p.H), b = (int)(bh / p.H);
  if (n >= p.Nq) {
    p.lse2[idx] = INFINITY;
    p.delta[idx] = 0.f;
    return;
  }
  const long long off = bwd_row(p.bsnd, b, h, n, p.H, p.Nq, D);
  const uint4* o4 = reinterpret_cast<const uint4*>(static_cast<const T*>(p.o) + off);
  const uint4* d4 = reinterpret_cast<const uint4*>(static_cast<const T*>(p.dout) + off);
  float acc = 0.f;
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    const uint4 a = o4[c], g = d4[c];
    const T* ae = reinterpret_cast<const T*>(&a);
    const T* ge = reinterpret_cast<const T*>(&g);
#pragma unroll
    for (int t = 0; t < 8; ++t) acc = fmaf(bwd_to_f<T>(ae[t]), bwd_to_f<T>(ge[t]), acc);
  }
  p.delta[idx] = acc;
  p.lse2[idx] = p.lse[bh * p.Nq + n] * 1.4426950408889634f;
}

// dQ = scale * accumulator in q's layout and dtype: one thread per 8 values.
template <int D, typename T>
__global__ void fa_bwd_post_kernel(BwdParams p) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.B * p.H * p.Nq * (D / 8);
  if (idx >= total) return;
  const int c8 = (int)(idx % (D / 8));
  const long long r = idx / (D / 8);  // (b, h, n) in [B, H, Nq] order
  const int n = (int)(r % p.Nq);
  const long long bh = r / p.Nq;
  const int h = (int)(bh % p.H), b = (int)(bh / p.H);
  const float4* a = reinterpret_cast<const float4*>(p.dq_acc + r * D + 8 * c8);
  const float4 x = a[0], y = a[1];
  uint4 out;
  out.x = sh_pack2<T>(x.x * p.scale, x.y * p.scale);
  out.y = sh_pack2<T>(x.z * p.scale, x.w * p.scale);
  out.z = sh_pack2<T>(y.x * p.scale, y.y * p.scale);
  out.w = sh_pack2<T>(y.z * p.scale, y.w * p.scale);
  *reinterpret_cast<uint4*>(static_cast<T*>(p.dq) + bwd_row(p.bsnd, b, h, n, p.H, p.Nq, D) + 8 * c8) = out;
}

template <int D, typename T>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, BwdParams p,
                  unsigned int* status_word) {
  using C = BwdCfg<D>;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int QST = C::QST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const int B_KV = 0, B_QFULL = 1, B_QEMPTY = 1 + QST, B_SFULL = 1 + 2 * QST, B_DPFULL = B_SFULL + 1,
            B_PREADY = B_SFULL + 2, B_DQFULL = B_SFULL + 3, B_DQFREE = B_SFULL + 4, B_DSFREE = B_SFULL + 5,
            B_DKDV = B_SFULL + 6, B_DRAIN = B_SFULL + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // This CTA's (batch, K/V head) and key tile: head-major, so that the CTAs
  // in flight share a few heads' Q, dO and dQ accumulator in L2; within a
  // head the heaviest key tiles (the first, under a causal mask) go first.
  const int bhk = blockIdx.x / p.kvtiles;
  const int kt = blockIdx.x - bhk * p.kvtiles;
  const int b = bhk / p.Hkv, hk = bhk - b * p.Hkv;
  const int group = p.H / p.Hkv;
  const int qt0 = p.causal ? kt : 0;  // query i sees key j iff j <= i: tiles before kt see none of these keys
  const int nqt = p.qtiles > qt0 ? p.qtiles - qt0 : 0;
  const int n = group * nqt;  // steps: (query head of the group, query tile)

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_DPFULL), 1);
    mbar_init(bar(B_PREADY), 4);
    mbar_init(bar(B_DQFULL), 1);
    mbar_init(bar(B_DQFREE), 4);
    mbar_init(bar(B_DSFREE), 1);
    mbar_init(bar(B_DKDV), 1);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == BWD_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == BWD_WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wctx{abort_flag, status_word, p.timeout_ns, 1u};

  if (warp == BWD_WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      const uint64_t pol_kv = l2_policy_evict_first();
      const uint64_t pol_q = l2_policy_evict_last();  // Q and dO are read by every key tile of the head
      mbar_arrive_expect_tx(bar(B_KV), 2 * C::TILE_BYTES);
      for (int c = 0; c < C::CHUNKS; ++c) {
        if (p.bsnd) {
          tma_load_4d(sbase + C::OFF_K + c * C::CHUNK_BYTES, &tm_k, bar(B_KV), c * 64, hk, kt * 128, b, pol_kv);
          tma_load_4d(sbase + C::OFF_V + c * C::CHUNK_BYTES, &tm_v, bar(B_KV), c * 64, hk, kt * 128, b, pol_kv);
        } else {
          tma_load_4d(sbase + C::OFF_K + c * C::CHUNK_BYTES, &tm_k, bar(B_KV), c * 64, kt * 128, hk, b, pol_kv);
          tma_load_4d(sbase + C::OFF_V + c * C::CHUNK_BYTES, &tm_v, bar(B_KV), c * 64, kt * 128, hk, b, pol_kv);
        }
      }
      int s = 0;
      for (; s < n; ++s) {
        const int h = hk * group + s / nqt, qt = qt0 + s % nqt;
        const int st = s % QST;
        if (!mbar_wait(bar(B_QEMPTY + st), ((s / QST) & 1) ^ 1, wctx)) break;
        mbar_arrive_expect_tx(bar(B_QFULL + st), 2 * C::TILE_BYTES);
        const uint32_t qd = sbase + C::OFF_Q + st * C::TILE_BYTES, dd = sbase + C::OFF_DO + st * C::TILE_BYTES;
        for (int c = 0; c < C::CHUNKS; ++c) {
          if (p.bsnd) {
            tma_load_4d(qd + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + st), c * 64, h, qt * 128, b, pol_q);
            tma_load_4d(dd + c * C::CHUNK_BYTES, &tm_do, bar(B_QFULL + st), c * 64, h, qt * 128, b, pol_q);
          } else {
            tma_load_4d(qd + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + st), c * 64, qt * 128, h, b, pol_q);
            tma_load_4d(dd + c * C::CHUNK_BYTES, &tm_do, bar(B_QFULL + st), c * 64, qt * 128, h, b, pol_q);
          }
        }
      }
      // Every copy this thread started lands before the CTA may exit.
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_KV), 0, drain);
      for (int i = 1; i <= QST && s - i >= 0; ++i) {
        const int g = s - i;
        mbar_wait(bar(B_QFULL + g % QST), (g / QST) & 1, drain);
      }
    }
    __syncwarp();
  } else if (warp == BWD_WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t ID_KK = bwd_idesc(IS_BF16, false, false, 128, 128);  // S^T, dP^T
    constexpr uint32_t ID_TB = bwd_idesc(IS_BF16, false, true, 128, D);     // dV, dK: A from TMEM, B MN-major
    constexpr uint32_t ID_DQ = bwd_idesc(IS_BF16, true, true, 128, D);      // dQ: A and B MN-major
    const uint64_t dK_k = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);             // K, K-major (S^T's A)
    const uint64_t dV_k = smem_desc_sw128(sbase + C::OFF_V, 16, 1024);             // V, K-major (dP^T's A)
    const uint64_t dK_mn = smem_desc_sw128(sbase + C::OFF_K, C::CHUNK_BYTES, 1024);  // K, N-major (dQ's B)
    const uint64_t dQ_k0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dQ_mn0 = smem_desc_sw128(sbase + C::OFF_Q, C::CHUNK_BYTES, 1024);
    const uint64_t dO_k0 = smem_desc_sw128(sbase + C::OFF_DO, 16, 1024);
    const uint64_t dO_mn0 = smem_desc_sw128(sbase + C::OFF_DO, C::CHUNK_BYTES, 1024);
    const uint64_t dS_mn = smem_desc_sw128(sbase + C::OFF_DS, C::CHUNK_BYTES, 1024);  // dS^T tile read M-major
    auto wait_all = [&](int bi, uint32_t ph) { return __all_sync(0xffffffffu, mbar_wait(bar(bi), ph, wctx)); };
    bool ok = n > 0 && wait_all(B_KV, 0);
    if (ok) tc_fence_after();
    // S^T(s) = K Q(s)^T into R_S (free once P^T(s-1) was read by dV(s-1): issue order)
    auto issue_s = [&](int s) -> bool {
      const int st = s % QST;
      if (!wait_all(B_QFULL + st, (s / QST) & 1)) return false;
      tc_fence_after();
      const uint64_t dq = dQ_k0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t o = (uint64_t)(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4);
        sh_mma_ss(tmem + C::R_S, dK_k + o, dq + o, ID_KK, kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(bar(B_SFULL));
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int s = 0; s < n && ok; ++s) {
      const int st = s % QST;
      // dP^T(s) = V dO(s)^T into R_DP; with D = 128 R_DP also holds dQ(s-1)
      // until the softmax warps have read it out.
      if (D == 128 && s > 0) {
        if (!wait_all(B_DQFREE, (s - 1) & 1)) { ok = false; break; }
        tc_fence_after();
      }
      const uint64_t ddo = dO_k0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t o = (uint64_t)(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4);
        sh_mma_ss(tmem + C::R_DP, dV_k + o, ddo + o, ID_KK, kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(bar(B_DPFULL));
      if (!wait_all(B_PREADY, s & 1)) { ok = false; break; }
      tc_fence_after();
      const uint64_t dom = dO_mn0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
      const uint64_t dqm = dQ_mn0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
      // dV += P^T dO(s), dK += dS^T Q(s): 8 steps of 16 query columns each
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ts(tmem + C::R_DV, tmem + C::R_S + 8 * kk, dom + (uint64_t)((kk * 2048) >> 4), ID_TB,
                  (s > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ts(tmem + C::R_DK, tmem + C::R_DP + 8 * kk, dqm + (uint64_t)((kk * 2048) >> 4), ID_TB,
                  (s > 0 || kk > 0) ? 1u : 0u);
      // dQ(s) = dS K: 8 steps of 16 keys
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ss(tmem + C::R_DQ, dS_mn + (uint64_t)((kk * 2048) >> 4), dK_mn + (uint64_t)((kk * 2048) >> 4), ID_DQ,
                  kk > 0 ? 1u : 0u);
      mma_commit_elect(bar(B_DQFULL));
      mma_commit_elect(bar(B_DSFREE));
      mma_commit_elect(bar(B_QEMPTY + st));
      if (s + 1 < n && !issue_s(s + 1)) { ok = false; break; }
    }
    if (n > 0) mma_commit_elect(bar(B_DKDV));
    mma_commit_elect(bar(B_DRAIN));
    {
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_DRAIN), 0, drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise + dQ + epilogue (warps 0-3)
    const int r = warp * 32 + lane;  // TMEM lane: key row (S^T, dP^T, dV, dK) or query row (dQ)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tl = tmem + lane_base;
    const int key = kt * 128 + r;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int s = 0; s < n && ok; ++s) {
      const int h = hk * group + s / nqt, qt = qt0 + s % nqt;
      const long long bh = (long long)b * p.H + h;
      const float* lse2 = p.lse2 + bh * p.nq_pad + qt * 128;  // 128 query columns (padded)
      const float* dlt = p.delta + bh * p.nq_pad + qt * 128;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL), s & 1, wctx));
      if (!ok) break;
      tc_fence_after();
      // visible iff key < Nkv and (causal) key <= query
      const bool need_mask = (kt * 128 + 128 > p.Nkv) || (p.causal && kt == qt);
      float pr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float sc[32];
        tmem_ld32(tl + C::R_S + 32 * c, sc);
        float4 l4[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) l4[t] = reinterpret_cast<const float4*>(lse2 + 32 * c)[t];
        const float* lv = reinterpret_cast<const float*>(l4);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          float x = fmaf(sc[t], sl2, -lv[t]);
          if (need_mask) {
            const int qi = qt * 128 + 32 * c + t;
            if (key >= p.Nkv || (p.causal && key > qi)) x = -INFINITY;
          }
          pr[32 * c + t] = ex2(x);
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = sh_pack2<T>(pr[32 * c + 2 * t], pr[32 * c + 2 * t + 1]);
        sh_tmem_st16(tl + C::R_S + 16 * c, pk);  // P^T over columns already read
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DPFULL), s & 1, wctx));
      if (ok && s > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DSFREE), (s - 1) & 1, wctx));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float dp[32];
        tmem_ld32(tl + C::R_DP + 32 * c, dp);
        float4 d4[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) d4[t] = reinterpret_cast<const float4*>(dlt + 32 * c)[t];
        const float* dv = reinterpret_cast<const float*>(d4);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          pk[t] = sh_pack2<T>(pr[32 * c + 2 * t] * (dp[2 * t] - dv[2 * t]),
                              pr[32 * c + 2 * t + 1] * (dp[2 * t + 1] - dv[2 * t + 1]));
        sh_tmem_st16(tl + C::R_DP + 16 * c, pk);  // dS^T over columns already read
        // the same 32 query columns of this key row into the shared dS^T tile:
        // 64-column chunk c / 2, 16-byte pieces 4 (c % 2) .. + 3, 128-byte swizzle
        const uint32_t rowb = sbase + C::OFF_DS + (c >> 1) * C::CHUNK_BYTES + r * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int piece = 4 * (c & 1) + j;
          st_shared_v4(rowb + ((piece ^ (r & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar(B_PREADY));
      // dQ(s): this thread's query row qt * 128 + r, added to the accumulator
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DQFULL), s & 1, wctx));
      if (!ok) break;
      tc_fence_after();
      const int qrow = qt * 128 + r;
      float* acc = p.dq_acc + (bh * p.Nq + qrow) * D;
      const bool qvalid = qrow < p.Nq && FA_INDEX_OK(status_word, (bh * p.Nq + qrow) < (long long)p.B * p.H * p.Nq);
      if constexpr (BWD_BULK_DQ) {
        // 32 columns at a time through the dS tile (free: dQ's MMA has read
        // it): this thread's 128 bytes at a row stride of 144 bytes (eight
        // consecutive rows then fall on different banks), then one bulk add
        // of them into the accumulator row.
        const uint32_t rowb = sbase + C::OFF_DS + r * 144;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          float v[32];
          tmem_ld32(tl + C::R_DQ + c0, v);
          if (c0 > 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(rowb + j * 16, __float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                         __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
          fence_proxy_async_smem();
          if (qvalid)
            asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], 128;" ::"l"(acc + c0),
                         "r"(rowb)
                         : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // the dS tile is written again next step
      } else {
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float v[32];
          tmem_ld32(tl + C::R_DQ + c, v);
          if (qvalid) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(acc + c + 4 * t), "f"(v[4 * t]),
                           "f"(v[4 * t + 1]), "f"(v[4 * t + 2]), "f"(v[4 * t + 3])
                           : "memory");
          }
        }
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_DQFREE));
    }
    if constexpr (BWD_BULK_DQ) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // dQ adds complete
    // ---------------------------------------------------------- dK, dV of this key row
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DKDV), 0, wctx));
    if (ok) {
      tc_fence_after();
      const long long off = bwd_row(p.bsnd, b, hk, key < p.Nkv ? key : 0, p.Hkv, p.Nkv, D);
      const bool store =
          key < p.Nkv && FA_INDEX_OK(status_word, off >= 0 && off + D <= (long long)p.B * p.Hkv * p.Nkv * D);
      T* dvp = static_cast<T*>(p.dv) + off;
      T* dkp = static_cast<T*>(p.dk) + off;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float v[32], k2[32];
        if (n > 0) {
          tmem_ld32(tl + C::R_DV + c, v);
          tmem_ld32(tl + C::R_DK + c, k2);
        } else {  // no query sees these keys
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = k2[t] = 0.f;
        }
        if (store) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            *reinterpret_cast<uint4*>(dvp + c + 8 * t) =
                make_uint4(sh_pack2<T>(v[8 * t], v[8 * t + 1]), sh_pack2<T>(v[8 * t + 2], v[8 * t + 3]),
                           sh_pack2<T>(v[8 * t + 4], v[8 * t + 5]), sh_pack2<T>(v[8 * t + 6], v[8 * t + 7]));
            *reinterpret_cast<uint4*>(dkp + c + 8 * t) = make_uint4(
                sh_pack2<T>(k2[8 * t] * p.scale, k2[8 * t + 1] * p.scale),
                sh_pack2<T>(k2[8 * t + 2] * p.scale, k2[8 * t + 3] * p.scale),
                sh_pack2<T>(k2[8 * t + 4] * p.scale, k2[8 * t + 5] * p.scale),
                sh_pack2<T>(k2[8 * t + 6] * p.scale, k2[8 * t + 7] * p.scale));
          }
        }
      }
    }
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == BWD_WARP_MMA) tmem_dealloc(tmem, 512);
}

}  // namespace fa
