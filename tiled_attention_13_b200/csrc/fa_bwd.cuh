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
//                        LSE = +inf, so P = 0 there, and D = 0); it also
//                        clears the fp32 dQ accumulator.
//   fa_bwd_kernel        one CTA per (batch, K/V head, 128-key tile), head-major, keeping
//                        that tile's K and V in shared memory and its dK and
//                        dV in tensor memory while it walks every query tile
//                        of every query head that reads this K/V head (under
//                        a causal mask only the query tiles at or after the
//                        key tile).  dQ of each step is added to an fp32
//                        accumulator in the workspace (TMA reduce-adds).
//   fa_bwd_post_kernel   dQ = scale * accumulator, rounded to the input dtype.
//
// fa_bwd_kernel, per query tile (step s), 320 threads:
//   warp 9      TMA: K, V once; Q(s) and dO(s) into a two-stage ring; the
//               step's column statistics (LSE * log2 e and D, 512 bytes
//               each) into single-stage shared buffers, each reloaded as
//               soon as the phase that reads it has handed over.  Once
//               the elementwise warps have staged dQ(s) in that stage, the
//               same thread adds it to the accumulator (TMA reduce-adds of
//               32 x 32 fp32 boxes) and reloads the stage for step s + 2
//               when the adds have read it.
//   warp 8      MMA issuer (whole warp, elect.sync):
//                 S^T = K Q^T -> R_S;  dP^T = V dO^T -> R_DP;
//                 dV += P^T dO (A = P^T from TMEM) as soon as P^T is written;
//                 once dS^T is: dK += dS^T Q (A = dS^T from TMEM), dQ = dS K
//                 (A = dS from shared memory, read M-major from the
//                 transposed tile) -> R_DQ; then S^T of the next step.
//   warps 0-7   two warpgroups; group g takes query columns [64 g, 64 g +
//               64) of each step, warp w % 4 of a group TMEM lanes 32 w ..
//               32 w + 31, one key row per thread: P^T = 2^(S^T scale log2 e
//               - LSE log2 e) (the column statistics read from shared
//               memory), then dS^T = P^T o (dP^T -
//               D); P^T and dS^T go back to tensor memory as 16-bit pairs
//               over columns the group has read, dS^T also to shared memory
//               (128-byte swizzle); then each thread reads its query row of
//               dQ (columns [g D/2, g D/2 + D/2)) and stages it in the step's
//               Q (group 0) or dO (group 1) tile, whose MMAs are done.  After
//               the last step: dV and scale * dK of its key row, the group's
//               columns.
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

#ifndef FA_BWD_VEC_DQ
#define FA_BWD_VEC_DQ 0
#endif
// How dQ(s) reaches the fp32 accumulator.  0 (default): each warp stages its
// 32 query rows in shared memory (128-byte swizzle) and one lane adds them
// with TMA tensor reduce-adds, 32 x 32 fp32 per instruction; 1: per-thread
// 16-byte vector reductions (red.global.add.v4.f32), one row per thread: 32
// separate 16-byte atomics per warp instruction, which the step trace showed
// taking 2.9 us of a 7.3 us step.
constexpr int BWD_VEC_DQ = FA_BWD_VEC_DQ;

// TMA tensor reduce-add shared -> global (4-D tile, fp32 add; rows outside the
// tensor are skipped by the tensor map).
__device__ __forceinline__ void bwd_tma_reduce_add_4d(const void* tmap, uint32_t src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   tmap),
               "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (a multiple of 16; both
// addresses 16-byte aligned), completing on the mbarrier's transaction count.
__device__ __forceinline__ void bwd_bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Optional timeline (compile with -DFA_TRACE_BWD): %globaltimer stamps of the
// first steps of a few CTAs, readable through fa_debug_bwd_trace_read().
#ifdef FA_TRACE_BWD
constexpr int BWT_CTAS = 8, BWT_STEPS = 8, BWT_EV = 8;
__device__ unsigned long long g_trace_bwd[BWT_CTAS * BWT_STEPS * BWT_EV];
#define FA_BWT(cond, s, ev)                                                                             \
  do {                                                                                                 \
    if ((cond) && blockIdx.x < BWT_CTAS && (s) < BWT_STEPS)                                            \
      g_trace_bwd[(blockIdx.x * BWT_STEPS + (s)) * BWT_EV + (ev)] = globaltimer_ns();                  \
  } while (0)
#else
#define FA_BWT(cond, s, ev) \
  do {                      \
  } while (0)
#endif
constexpr int BWD_EW_WARPS = 8;  // elementwise warps: two warpgroups, one per half of a step's query columns
constexpr int BWD_WARP_MMA = 8;
constexpr int BWD_WARP_TMA = 9;
constexpr int BWD_THREADS = 32 * 10;

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
  static constexpr int OFF_STATS = OFF_DS + 128 * 128 * 2;  // LSE * log2 e [128], then D [128], fp32
  static constexpr int OFF_BAR = OFF_STATS + 2 * 128 * 4;
  // kv_full qd_full[QST] qd_empty[QST] s_full dp_full p_ready dq_full dq_free ds_free dkdv_full drain pt_ready
  // lse_full delta_full
  static constexpr int NBAR = 1 + 2 * QST + 11;
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

// D = sum dO o O (fp32) and LSE * log2 e per padded query row, and the
// row's fp32 dQ accumulator cleared: D / 8 lanes per row, each reading 16
// bytes of O and of dO (a row's reads are one contiguous segment per
// tensor) and clearing 32 bytes of the accumulator; a shuffle reduction
// within the row's lanes forms D.
template <int D, typename T>
__global__ void fa_bwd_pre_kernel(BwdParams p) {
  constexpr int LPR = D / 8;  // lanes per row; divides 32, so a row's lanes share a warp
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long idx = gid / LPR;  // padded row (b, h, n) in [B, H, nq_pad] order
  const int part = (int)(gid % LPR);
  const long long rows = (long long)p.B * p.H * p.nq_pad;
  if (idx >= rows) return;  // whole rows leave together
  const int n = (int)(idx % p.nq_pad);
  const long long bh = idx / p.nq_pad;
  if (n >= p.Nq) {
    if (part == 0) {
      p.lse2[idx] = INFINITY;
      p.delta[idx] = 0.f;
    }
    return;
  }
  const int h = (int)(bh % p.H), b = (int)(bh / p.H);
  const long long off = bwd_row(p.bsnd, b, h, n, p.H, p.Nq, D) + 8 * part;
  const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.o) + off);
  const uint4 g = *reinterpret_cast<const uint4*>(static_cast<const T*>(p.dout) + off);
  float4* acc_row = reinterpret_cast<float4*>(p.dq_acc + (bh * p.Nq + n) * D + 8 * part);
  acc_row[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  acc_row[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  const T* ae = reinterpret_cast<const T*>(&a);
  const T* ge = reinterpret_cast<const T*>(&g);
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) acc = fmaf(bwd_to_f<T>(ae[t]), bwd_to_f<T>(ge[t]), acc);
  const unsigned gmask = (LPR == 32) ? 0xffffffffu : (((1u << LPR) - 1u) << ((threadIdx.x & 31) & ~(LPR - 1)));
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(gmask, acc, o);
  if (part == 0) {
    p.delta[idx] = acc;
    p.lse2[idx] = p.lse[bh * p.Nq + n] * 1.4426950408889634f;
  }
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
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, BwdParams p, unsigned int* status_word) {
  using C = BwdCfg<D>;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int QST = C::QST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const int B_KV = 0, B_QFULL = 1, B_QEMPTY = 1 + QST, B_SFULL = 1 + 2 * QST, B_DPFULL = B_SFULL + 1,
            B_PREADY = B_SFULL + 2, B_DQFULL = B_SFULL + 3, B_DQFREE = B_SFULL + 4, B_DSFREE = B_SFULL + 5,
            B_DKDV = B_SFULL + 6, B_DRAIN = B_SFULL + 7, B_PTREADY = B_SFULL + 8, B_LSEF = B_SFULL + 9,
            B_DLTF = B_SFULL + 10;
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
      mbar_init(bar(B_QEMPTY + s), BWD_EW_WARPS);  // released by the warps once their dQ adds read it
    }
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_DPFULL), 1);
    mbar_init(bar(B_PREADY), BWD_EW_WARPS);
    mbar_init(bar(B_DQFULL), 1);
    mbar_init(bar(B_DQFREE), BWD_EW_WARPS);
    mbar_init(bar(B_DSFREE), 1);
    mbar_init(bar(B_DKDV), 1);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_PTREADY), BWD_EW_WARPS);
    mbar_init(bar(B_LSEF), 1);
    mbar_init(bar(B_DLTF), 1);
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
    prefetch_tmap(&tm_dq);
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
      // dQ of step sd, staged by the eight elementwise warps in the Q and dO
      // tiles of its stage, goes to the accumulator: one reduce-add per
      // 32 x 32 box, then wait until they have read the stage.
      constexpr int DH = D / 2;
      auto add_dq = [&](int sd) {
        const int hd = hk * group + sd / nqt, qtd = qt0 + sd % nqt, std_ = sd % QST;
        if (!BWD_VEC_DQ) {
          for (int gg = 0; gg < 2; ++gg) {
            const uint32_t base = sbase + (gg == 0 ? C::OFF_Q : C::OFF_DO) + std_ * C::TILE_BYTES;
            for (int w = 0; w < 4; ++w)
              for (int k2 = 0; k2 < DH / 32; ++k2)
                bwd_tma_reduce_add_4d(&tm_dq, base + (w * (DH / 32) + k2) * 4096, DH * gg + 32 * k2,
                                      qtd * 128 + 32 * w, hd, b);
          }
          sh_bulk_commit();
          sh_bulk_wait_read0();
        }
      };
      int s = 0;
      int qd_issued = 0, stats_lse = 0, stats_dlt = 0;  // Q/dO stages and statistics loads issued
      for (; s < n; ++s) {
        const int h = hk * group + s / nqt, qt = qt0 + s % nqt;
        const int st = s % QST;
        if (s >= QST) {  // the stage's previous step: its dQ staged (so its MMAs are done), then added
          if (!mbar_wait(bar(B_QEMPTY + st), ((s / QST) - 1) & 1, wctx)) break;
          add_dq(s - QST);
        }
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
        qd_issued = s + 1;
        // Column statistics of step s: the LSE row once P^T(s - 1) has read
        // the buffer (the warps' arrivals on pt_ready), the D row once
        // dS^T(s - 1) has (p_ready).  Both waits come in the order the steps
        // produce them, after this step's Q and dO are on their way.
        const long long srow = ((long long)b * p.H + h) * p.nq_pad + (long long)qt * 128;
        if (s > 0 && !mbar_wait(bar(B_PTREADY), (s - 1) & 1, wctx)) break;
        mbar_arrive_expect_tx(bar(B_LSEF), 512);
        bwd_bulk_load(sbase + C::OFF_STATS, p.lse2 + srow, 512, bar(B_LSEF));
        if (s > 0 && !mbar_wait(bar(B_PREADY), (s - 1) & 1, wctx)) { ++stats_lse; break; }
        mbar_arrive_expect_tx(bar(B_DLTF), 512);
        bwd_bulk_load(sbase + C::OFF_STATS + 512, p.delta + srow, 512, bar(B_DLTF));
        ++stats_lse;
        ++stats_dlt;
      }
      // the last steps' dQ
      if (s == n)
        for (int sd = (n > QST ? n - QST : 0); sd < n; ++sd) {
          if (!mbar_wait(bar(B_QEMPTY + sd % QST), (sd / QST) & 1, wctx)) break;
          add_dq(sd);
        }
      // Every copy this thread started lands (and every add completes) before the CTA may exit.
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_KV), 0, drain);
      for (int i = 1; i <= QST && qd_issued - i >= 0; ++i) {
        const int g = qd_issued - i;
        mbar_wait(bar(B_QFULL + g % QST), (g / QST) & 1, drain);
      }
      if (stats_lse > 0) mbar_wait(bar(B_LSEF), (stats_lse - 1) & 1, drain);
      if (stats_dlt > 0) mbar_wait(bar(B_DLTF), (stats_dlt - 1) & 1, drain);
      sh_bulk_wait0();
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
      // dV += P^T dO(s) as soon as P^T is written (the warps compute dS^T
      // meanwhile); dK and dQ once dS^T is
      if (!wait_all(B_PTREADY, s & 1)) { ok = false; break; }
      tc_fence_after();
      const uint64_t dom = dO_mn0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
      // 8 steps of 16 query columns; queries 64 g + 16 i (g the warpgroup)
      // sit packed at column 64 g + 8 i
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ts(tmem + C::R_DV, tmem + C::R_S + 64 * (kk >> 2) + 8 * (kk & 3), dom + (uint64_t)((kk * 2048) >> 4),
                  ID_TB, (s > 0 || kk > 0) ? 1u : 0u);
      if (!wait_all(B_PREADY, s & 1)) { ok = false; break; }
      FA_BWT(lane == 0, s, 7);
      tc_fence_after();
      const uint64_t dqm = dQ_mn0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
      // dK += dS^T Q(s), in the same packed layout
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ts(tmem + C::R_DK, tmem + C::R_DP + 64 * (kk >> 2) + 8 * (kk & 3), dqm + (uint64_t)((kk * 2048) >> 4),
                  ID_TB, (s > 0 || kk > 0) ? 1u : 0u);
      // dQ(s) = dS K: 8 steps of 16 keys
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        sh_mma_ss(tmem + C::R_DQ, dS_mn + (uint64_t)((kk * 2048) >> 4), dK_mn + (uint64_t)((kk * 2048) >> 4), ID_DQ,
                  kk > 0 ? 1u : 0u);
      mma_commit_elect(bar(B_DQFULL));
      mma_commit_elect(bar(B_DSFREE));
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
    // ------------------------------------------------------------ elementwise + dQ + epilogue (warps 0-7)
    // Warpgroup g takes query columns [64 g, 64 g + 64) of every step (and,
    // for dQ, dV and dK, columns [g D / 2, g D / 2 + D / 2) of d); warp
    // w = warp % 4 of either group owns TMEM lanes 32 w .. 32 w + 31.
    const int g = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // TMEM lane: key row (S^T, dP^T, dV, dK) or query row (dQ)
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t tl = tmem + lane_base;
    const int key = kt * 128 + r;
    const float sl2 = p.scale_log2;
    constexpr int DH = D / 2;  // columns of d per warpgroup
    // this group's 64 column statistics of the current step in shared memory
    const float4* lse_s = reinterpret_cast<const float4*>(smem + C::OFF_STATS) + 16 * g;
    const float4* dlt_s = reinterpret_cast<const float4*>(smem + C::OFF_STATS + 512) + 16 * g;
    bool ok = true;
    for (int s = 0; s < n && ok; ++s) {
      const int h = hk * group + s / nqt, qt = qt0 + s % nqt;
      const int st = s % QST;
      const long long bh = (long long)b * p.H + h;
      FA_BWT(threadIdx.x == 0, s, 0);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL), s & 1, wctx) && mbar_wait(bar(B_LSEF), s & 1, wctx));
      if (!ok) break;
      FA_BWT(threadIdx.x == 0, s, 1);
      tc_fence_after();
      // visible iff key < Nkv and (causal) key <= query
      const bool need_mask = (kt * 128 + 128 > p.Nkv) || (p.causal && kt == qt);
      // the group's 64 scores of this key row in one tensor-memory read,
      // then P^T in place (64 independent exps per thread)
      float pr[64];
      tmem_ld64(tl + C::R_S + 64 * g, pr);
#pragma unroll
      for (int t8 = 0; t8 < 8; ++t8) {
        const float4 la = lse_s[2 * t8];
        const float4 lb = lse_s[2 * t8 + 1];
        const float lv[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = 8 * t8 + u;
          float x = fmaf(pr[t], sl2, -lv[u]);
          if (need_mask) {
            const int qi = qt * 128 + 64 * g + t;
            if (key >= p.Nkv || (p.causal && key > qi)) x = -INFINITY;
          }
          pr[t] = ex2(x);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = sh_pack2<T>(pr[32 * c + 2 * t], pr[32 * c + 2 * t + 1]);
        sh_tmem_st16(tl + C::R_S + 64 * g + 16 * c, pk);  // P^T over this group's columns already read
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(bar(B_PTREADY));
      FA_BWT(threadIdx.x == 0, s, 2);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DPFULL), s & 1, wctx));
      FA_BWT(threadIdx.x == 0, s, 3);
      if (ok && s > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DSFREE), (s - 1) & 1, wctx));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DLTF), s & 1, wctx));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        // D of these 32 columns first: its shared-memory reads overlap the
        // tensor-memory read of dP^T
        float4 dv4[8];
#pragma unroll
        for (int t4 = 0; t4 < 8; ++t4) dv4[t4] = dlt_s[8 * c + t4];
        float dp[32];
        tmem_ld32(tl + C::R_DP + 64 * g + 32 * c, dp);
        uint32_t pk[16];
#pragma unroll
        for (int t4 = 0; t4 < 8; ++t4) {
          const float4 d4 = dv4[t4];
          const int t = 4 * t4;
          pk[2 * t4] = sh_pack2<T>(pr[32 * c + t] * (dp[t] - d4.x), pr[32 * c + t + 1] * (dp[t + 1] - d4.y));
          pk[2 * t4 + 1] =
              sh_pack2<T>(pr[32 * c + t + 2] * (dp[t + 2] - d4.z), pr[32 * c + t + 3] * (dp[t + 3] - d4.w));
        }
        sh_tmem_st16(tl + C::R_DP + 64 * g + 16 * c, pk);  // dS^T over columns already read
        // the same 32 query columns of this key row into the shared dS^T tile:
        // 64-column chunk g, 16-byte pieces 4 c .. 4 c + 3, 128-byte swizzle
        const uint32_t rowb = sbase + C::OFF_DS + g * C::CHUNK_BYTES + r * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int piece = 4 * c + j;
          st_shared_v4(rowb + ((piece ^ (r & 7)) << 4), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(bar(B_PREADY));
      FA_BWT(threadIdx.x == 0, s, 4);
      // dQ(s): query rows qt * 128 + r, this group's D / 2 columns
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DQFULL), s & 1, wctx));
      if (!ok) break;
      FA_BWT(threadIdx.x == 0, s, 5);
      tc_fence_after();
      const int qrow = qt * 128 + r;
      float v[DH];
      if constexpr (DH == 64) {
        tmem_ld64(tl + C::R_DQ + DH * g, v);
      } else {
        tmem_ld32(tl + C::R_DQ + DH * g, v);
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_DQFREE));  // dQ is read: R_DQ may be written again
      FA_BWT(threadIdx.x == 0, s, 6);
      if constexpr (!BWD_VEC_DQ) {
        // Stage this warp's 32 rows x D / 2 columns in the step's Q or dO
        // tile (group 0 / 1; every MMA that reads them is done), as 32 x 32
        // boxes at 128-byte swizzle; the TMA warp adds them to the
        // accumulator.
        const uint32_t stage = sbase + (g == 0 ? C::OFF_Q : C::OFF_DO) + st * C::TILE_BYTES + wq * (DH / 32) * 4096;
#pragma unroll
        for (int k2 = 0; k2 < DH / 32; ++k2) {
          const uint32_t rowb = stage + k2 * 4096 + lane * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(rowb + ((j ^ (lane & 7)) << 4), __float_as_uint(v[32 * k2 + 4 * j]),
                         __float_as_uint(v[32 * k2 + 4 * j + 1]), __float_as_uint(v[32 * k2 + 4 * j + 2]),
                         __float_as_uint(v[32 * k2 + 4 * j + 3]));
        }
        fence_proxy_async_smem();
      } else {
        if (qrow < p.Nq && FA_INDEX_OK(status_word, (bh * p.Nq + qrow) < (long long)p.B * p.H * p.Nq)) {
          float* acc = p.dq_acc + (bh * p.Nq + qrow) * D + DH * g;
#pragma unroll
          for (int t = 0; t < DH / 4; ++t)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(acc + 4 * t), "f"(v[4 * t]),
                         "f"(v[4 * t + 1]), "f"(v[4 * t + 2]), "f"(v[4 * t + 3])
                         : "memory");
        }
      }
      mbar_arrive_warp(bar(B_QEMPTY + st));  // staged (or added): the TMA warp takes the stage from here
    }
    // ---------------------------------------------------------- dK, dV of this key row, this group's columns
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DKDV), 0, wctx));
    if (ok) {
      tc_fence_after();
      const long long off = bwd_row(p.bsnd, b, hk, key < p.Nkv ? key : 0, p.Hkv, p.Nkv, D);
      const bool store =
          key < p.Nkv && FA_INDEX_OK(status_word, off >= 0 && off + D <= (long long)p.B * p.Hkv * p.Nkv * D);
      T* dvp = static_cast<T*>(p.dv) + off;
      T* dkp = static_cast<T*>(p.dk) + off;
#pragma unroll 1
      for (int c = DH * g; c < DH * g + DH; c += 32) {
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
