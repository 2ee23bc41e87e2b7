// fa_fwd_short_wg.cuh -- tensor-core attention forward for short key
// sequences at head dim 64: Nkv <= 128, bf16 or fp16 inputs, fp32
// accumulation.  Four independent query-tile pipelines per CTA.
//
// The workload is page 3's AIGC cross-attention ("ops-nn efficient attention
// for AIGC", section 四: 4096 latent tokens attend to 77 text tokens).  With
// one KV tile per query tile the softmax is exact in one step (page 1, "CANN
// ops-transformer FlashAttentionScore", section 在线 Softmax 的数学原理拆解,
// with a single block): S = Q K^T, the row max, p = exp(S - max), l = sum p,
// O = P V / l.  Q is read and O written once, so the kernel is an HBM stream;
// what limits it is how many query tiles an SM keeps in flight, and the
// special-function unit that evaluates the exps.
//
// B200 mapping (512 threads, one CTA per SM):
//   CTA c owns a contiguous range of query tiles (b, h, qt), qt fastest;
//   warpgroup w takes the range's tiles w, w + 4, ... .  Each warpgroup is a
//   pipeline of its own, with its own barriers, shared-memory region and 128
//   tensor-memory columns, so a CTA with up to four tiles runs all of them at
//   once (the 4096 x 77 shape: 512 tiles on 148 SMs, three or four per CTA).
//   Lane 0 of the warpgroup's first warp issues its TMA loads and stores;
//   the whole warp issues its MMAs (elect.sync).  No warp is set aside for
//   either job: the 16 warps all run softmax, which keeps the register cap
//   at 128 per thread.
//   Shared memory per warpgroup: NS Q stages of 128 x 64 (the stage a tile's
//   Q came from holds its O for the TMA store), K and V of n_s rows each
//   (n_s = Nkv rounded up to 16; rows past Nkv read as zeros).  NS = 2 when
//   that fits, so the next tile's Q loads during the current tile.
//   Tensor memory per warpgroup (128 columns): S in [0, n_s), P packed to 16
//   bits in [0, n_s / 2), O in [64, 128).  O overlaps S columns [64, n_s) only
//   after the softmax has read all of S; the next S is issued only after the
//   epilogue has read O.
//   The exps of 8-key groups that no row of a warp can see are skipped
//   (warp-uniform test), so 77 keys cost 80 exps a row, not 96.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "pdl.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace fa {

#ifdef FA_TRACE_SHORT
constexpr int SWT_CTAS = 160, SWT_EV = 32;
__device__ unsigned long long g_trace_short_wg[SWT_CTAS * SWT_EV];
#define FA_SWT(cond, ev)                                                            \
  do {                                                                              \
    if ((cond) && blockIdx.x < SWT_CTAS) g_trace_short_wg[blockIdx.x * SWT_EV + (ev)] = globaltimer_ns(); \
  } while (0)
#else
#define FA_SWT(cond, ev) \
  do {                   \
  } while (0)
#endif

constexpr int SW_WGS = 4;
constexpr int SW_THREADS = 128 * SW_WGS;
constexpr int SW_Q_BYTES = 128 * 64 * 2;  // one 128 x 64 tile of 16-bit values
constexpr int SW_NBAR = 8;                // barriers per warpgroup
constexpr int SW_SMEM_MAX = 232448;       // per-CTA shared memory of sm_100

// Shared memory of one warpgroup and of the CTA for n_s key rows and ns Q stages.
__host__ __device__ constexpr int sw_wg_bytes(int n_s, int ns) { return ns * SW_Q_BYTES + 2 * n_s * 128; }
__host__ __device__ constexpr int sw_smem_bytes(int n_s, int ns) {
  return SW_WGS * sw_wg_bytes(n_s, ns) + SW_WGS * SW_NBAR * 8 + 16 + 1024;
}

struct SwParams {
  float* lse;  // [B, H, Nq] or nullptr
  int B, H, Nq, Nkv;
  int bsnd;          // 1: [B, N, H, D] rows, 0: [B, H, N, D]
  int causal;        // key j visible to query i iff j <= i
  float scale_log2;  // softmax scale * log2(e)
  int qtiles;        // ceil(Nq / 128)
  int n_tiles;       // B * H * qtiles
  int kv_group;      // query heads per K/V head
  int n_s;           // Nkv rounded up to 16: S columns, K / V rows loaded
  int ns;            // Q stages per warpgroup (1 or 2)
  uint64_t timeout_ns;
  int fault_mode;
};

struct SwTile {
  int b, h, qt, kv;
};
__host__ __device__ __forceinline__ SwTile sw_decode(int t, const SwParams& p) {
  SwTile x;
  const int bh = t / p.qtiles;
  x.qt = t - bh * p.qtiles;
  x.b = bh / p.H;
  x.h = bh - x.b * p.H;
  x.kv = x.b * (p.H / p.kv_group) + x.h / p.kv_group;
  return x;
}

// Tiles [t0, t1) of CTA c out of G: contiguous, sizes differing by at most one.
__host__ __device__ __forceinline__ void sw_range(int c, int G, int n_tiles, int& t0, int& t1) {
  t0 = (int)(((long long)c * n_tiles) / G);
  t1 = (int)(((long long)(c + 1) * n_tiles) / G);
}


// 16 columns per thread, then wait.
__device__ __forceinline__ void sw_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// A packed pair of 16-bit values times f, repacked.
template <typename T>
__device__ __forceinline__ uint32_t sw_scale_pk(uint32_t v, float f);
template <>
__device__ __forceinline__ uint32_t sw_scale_pk<__nv_bfloat16>(uint32_t v, float f) {
  const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
  return sh_pack2<__nv_bfloat16>(x.x * f, x.y * f);
}
template <>
__device__ __forceinline__ uint32_t sw_scale_pk<__half>(uint32_t v, float f) {
  const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&v));
  return sh_pack2<__half>(x.x * f, x.y * f);
}

template <typename T>
__global__ void __launch_bounds__(SW_THREADS, 1)
    fa_fwd_short_wg_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                           SwParams p, unsigned int* status_word) {
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int wg_bytes = sw_wg_bytes(p.n_s, p.ns);
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(smem + SW_WGS * wg_bytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars_all + SW_WGS * SW_NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  const bool lead_warp = (warp & 3) == 0;
  const bool leader = lead_warp && lane == 0;
  // this warpgroup's region and barriers: q_full[2] kv_full s_full p_full o_full o_staged drain
  const uint32_t rq = sbase + wg * wg_bytes;                 // Q stages
  const uint32_t rk = rq + p.ns * SW_Q_BYTES, rv = rk + p.n_s * 128;
  const uint32_t bb = smem_u32(bars_all + wg * SW_NBAR);
  const uint32_t B_QFULL = bb, B_KVFULL = bb + 16, B_SFULL = bb + 24, B_PFULL = bb + 32, B_OFULL = bb + 40,
                 B_OSTAGED = bb + 48, B_DRAIN = bb + 56;

  int t0, t1;
  sw_range(blockIdx.x, gridDim.x, p.n_tiles, t0, t1);
  const int n = t1 - t0;
  const int mine = n > wg ? (n - wg + SW_WGS - 1) / SW_WGS : 0;  // this warpgroup's tiles
  FA_SWT(threadIdx.x == 0, 0);

  int q_issued = 0;                      // Q loads issued by this warpgroup's leader
  int kv_cur = -1, kv_loads = 0;         // K/V head in the slot, loads issued
  uint64_t pol_q = 0, pol_kv = 0;  // L2 policies of the leader's loads
  auto issue_q = [&](int j) {  // leader: Q of this warpgroup's tile j into stage j % ns
    const SwTile x = sw_decode(t0 + wg + SW_WGS * j, p);
    const int s = j % p.ns;
    const uint32_t bar = B_QFULL + 8 * s;
    mbar_arrive_expect_tx(bar, SW_Q_BYTES);
    if (p.bsnd)
      tma_load_4d(rq + s * SW_Q_BYTES, &tm_q, bar, 0, x.h, x.qt * 128, x.b, pol_q);
    else
      tma_load_4d(rq + s * SW_Q_BYTES, &tm_q, bar, 0, x.qt * 128, x.h, x.b, pol_q);
  };
  auto issue_kv = [&](const SwTile& x) {  // leader: K and V of x's (batch, K/V head)
    const int hk = x.h / p.kv_group;
    mbar_arrive_expect_tx(B_KVFULL, 2 * p.n_s * 128);
    if (p.bsnd) {
      tma_load_4d(rk, &tm_k, B_KVFULL, 0, hk, 0, x.b, pol_kv);
      tma_load_4d(rv, &tm_v, B_KVFULL, 0, hk, 0, x.b, pol_kv);
    } else {
      tma_load_4d(rk, &tm_k, B_KVFULL, 0, 0, hk, x.b, pol_kv);
      tma_load_4d(rv, &tm_v, B_KVFULL, 0, 0, hk, x.b, pol_kv);
    }
  };

  // The leader sets up its own barriers and starts its first loads before
  // the CTA-wide barrier, so they are in flight during the prologue.  The
  // tensor-map prefetches go first (their fetch overlaps the barrier set-up),
  // and Q, the load from HBM, before K and V, which come from L2 after the
  // first CTA of a head has read them.
  pdl_launch_dependents();
  if (leader) {
    if (mine > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_o);
    }
    mbar_init(B_QFULL, 1);
    mbar_init(B_QFULL + 8, 1);
    mbar_init(B_KVFULL, 1);
    mbar_init(B_SFULL, 1);
    mbar_init(B_PFULL, 4);  // one arrival per warp
    mbar_init(B_OFULL, 1);
    mbar_init(B_OSTAGED, 4);
    mbar_init(B_DRAIN, 1);
    fence_barrier_init();
    pdl_wait();  // the inputs are complete from here on
    FA_SWT(wg == 0, 16);
    if (mine > 0) {
      pol_q = l2_policy_evict_first();
      pol_kv = l2_policy_evict_last();
      for (int j = 0; j < p.ns && j < mine; ++j) issue_q(j);
      q_issued = mine < p.ns ? mine : p.ns;
      FA_SWT(wg == 0, 17);
      const SwTile x0 = sw_decode(t0 + wg, p);
      issue_kv(x0);
      kv_cur = x0.kv;
      kv_loads = 1;
      FA_SWT(wg == 0, 18);
    }
    FA_SWT(wg == 0, 15);
  }
  pdl_wait();
  if (threadIdx.x == 0) *abort_flag = 0;
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wctx{abort_flag, status_word, p.timeout_ns, 1u};
  FA_SWT(threadIdx.x == 0, 1);
  // every lane tracks the K/V loads the same way as the leader
  if (!leader && mine > 0) {
    kv_cur = sw_decode(t0 + wg, p).kv;
    kv_loads = 1;
  }

  const int r = (warp & 3) * 32 + lane;  // query row within the tile == TMEM lane
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t tS = tmem + 128 * wg, tO = tS + 64;
  const uint32_t tSl = tS + lane_base, tOl = tO + lane_base;
  const uint32_t idesc_s = idesc_f16(IS_BF16, false, 128, (uint32_t)p.n_s);
  constexpr uint32_t IDESC_PV = idesc_f16(IS_BF16, true, 128, 64);
  const float sl2 = p.scale_log2;
  const int nc = (p.n_s + 31) >> 5;  // 32-key chunks of S
  bool ok = true;

  for (int j = 0; j < mine && ok; ++j) {
    const SwTile x = sw_decode(t0 + wg + SW_WGS * j, p);
    const int s = j % p.ns;
    const uint32_t ph = (uint32_t)(j & 1);
    // ---------------------------------------------------------------- S = Q K^T
    if (lead_warp) {
      ok = __all_sync(0xffffffffu, mbar_wait(B_QFULL + 8 * s, (uint32_t)((j / p.ns) & 1), wctx));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(B_KVFULL, (uint32_t)((kv_loads - 1) & 1), wctx));
      if (ok) {
        tc_fence_after();
        const uint64_t dQ = smem_desc_sw128(rq + s * SW_Q_BYTES, 16, 1024);
        const uint64_t dK = smem_desc_sw128(rk, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) sh_mma_ss(tS, dQ + 2 * kk, dK + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
        mma_commit_elect(B_SFULL);
      }
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(B_SFULL, ph, wctx));
    if (!ok) break;
    FA_SWT(leader && j == 0, 2 + wg);
    tc_fence_after();
    // ---------------------------------------------------------------- softmax
    const int row = x.qt * 128 + r;
    const int lim = p.causal ? (row + 1 < p.Nkv ? row + 1 : p.Nkv) : p.Nkv;  // visible keys [0, lim)
    int lim_hi = p.Nkv;  // largest lim of the warp's rows: groups at or past it are all masked
    if (p.causal) {
      const int top = x.qt * 128 + (warp & 3) * 32 + 32;
      lim_hi = top < p.Nkv ? top : p.Nkv;
    }
    // Groups of 8 keys every row of the warp sees (k + 8 <= lim_lo) skip the
    // per-key mask; groups no row sees (k >= lim_hi) skip the loads and exps.
    int lim_lo = p.Nkv;
    if (p.causal) {
      const int bot = x.qt * 128 + (warp & 3) * 32 + 1;
      lim_lo = bot < p.Nkv ? bot : p.Nkv;
    }
    // One pass over S, 32 keys at a time.  The reference max m2 (log2 units)
    // is the row max of the first chunk, so a later chunk's
    // p = 2^(s * scale * log2 e - m2) may reach 2^8, well inside the range of
    // 16-bit P and of the fp32 sum.  A row whose chunk max passes m2 + 8 takes it as its new
    // reference, and the P it has already written is rescaled in tensor
    // memory (a warp-uniform branch that random scores practically never take).
    auto max8 = [&](const float* v8, int k0, float& mx0, float& mx1, auto MASKc) {
      constexpr bool MASK = decltype(MASKc)::value;
      float v[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = (!MASK || k0 + t < lim) ? v8[t] : -INFINITY;
      mx0 = fmax3(mx0, v[0], v[1]);
      mx1 = fmax3(mx1, v[2], v[3]);
      mx0 = fmax3(mx0, v[4], v[5]);
      mx1 = fmax3(mx1, v[6], v[7]);
    };
    const uint64_t scale2 = f2_pack(sl2, sl2);
    float m2 = 0.f;
    uint64_t acc_a = 0ull, acc_b = 0ull;
    // p for 8 keys, packed to 16 bits in pk4[0..4)
    auto exp8 = [&](const float* v8, int k0, uint32_t* pk4, uint64_t negm2, auto MASKc) {
      constexpr bool MASK = decltype(MASKc)::value;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float s0 = (!MASK || k0 + 2 * t < lim) ? v8[2 * t] : -INFINITY;
        const float s1 = (!MASK || k0 + 2 * t + 1 < lim) ? v8[2 * t + 1] : -INFINITY;
        const uint64_t x2 = f2_fma(f2_pack(s0, s1), scale2, negm2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        if (t & 1)
          acc_b = f2_add(acc_b, f2_pack(p0, p1));
        else
          acc_a = f2_add(acc_a, f2_pack(p0, p1));
        pk4[t] = sh_pack2<T>(p0, p1);
      }
    };
#pragma unroll 1
    for (int c = 0; c < nc; ++c) {
      uint32_t pk[16];
      if (32 * c < lim_hi) {
        float sc[32];
        tmem_ld32(tSl + 32 * c, sc);
        FA_SWT(warp == 0 && lane == 0 && j == 0 && c < 2, 26 + 3 * c);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int k0 = 32 * c + 8 * g;
          if (k0 + 8 <= lim_lo)
            max8(sc + 8 * g, k0, mx0, mx1, std::false_type{});
          else if (k0 < lim_hi)
            max8(sc + 8 * g, k0, mx0, mx1, std::true_type{});
        }
        const float mc2 = fmaxf(mx0, mx1) * sl2;
        if (c == 0) {
          m2 = mc2;  // finite: every row sees key 0
        } else {
          const bool up = mc2 > m2 + 8.f;
          if (__any_sync(0xffffffffu, up)) {
            const float nm2 = up ? mc2 : m2;
            const float f = ex2(m2 - nm2);  // 1 for rows that keep their reference
            tmem_wait_st();                 // the P stores of earlier chunks have landed
#pragma unroll 1
            for (int cc = 0; cc < c; ++cc) {
              uint32_t w[16];
              sw_tmem_ld16(tSl + 16 * cc, w);
#pragma unroll
              for (int t = 0; t < 16; ++t) w[t] = sw_scale_pk<T>(w[t], f);
              sh_tmem_st16(tSl + 16 * cc, w);
            }
            const uint64_t f2 = f2_pack(f, f);
            acc_a = f2_fma(acc_a, f2, 0ull);
            acc_b = f2_fma(acc_b, f2, 0ull);
            m2 = nm2;
          }
        }
        const uint64_t negm2 = f2_pack(-m2, -m2);
        FA_SWT(warp == 0 && lane == 0 && j == 0 && c < 2, 27 + 3 * c);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int k0 = 32 * c + 8 * g;
          if (k0 + 8 <= lim_lo) {
            exp8(sc + 8 * g, k0, pk + 4 * g, negm2, std::false_type{});
          } else if (k0 < lim_hi) {
            exp8(sc + 8 * g, k0, pk + 4 * g, negm2, std::true_type{});
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) pk[4 * g + t] = 0u;
          }
        }
      } else {
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = 0u;
      }
      FA_SWT(warp == 0 && lane == 0 && j == 0 && c < 2, 28 + 3 * c);
      sh_tmem_st16(tSl + 16 * c, pk);
    }
    FA_SWT(lane == 0 && j == 0 && (warp == 0 || warp == 12), warp == 0 ? 21 : 24);
    float l;
    {
      float a0, a1, b0, b1;
      f2_unpack(acc_a, a0, a1);
      f2_unpack(acc_b, b0, b1);
      l = (a0 + a1) + (b0 + b1);
    }
    tmem_wait_st();
    tc_fence_before();
    if (p.fault_mode != 1) mbar_arrive_warp(B_PFULL);
    // ---------------------------------------------------------------- O = P V
    if (lead_warp) {
      ok = __all_sync(0xffffffffu, mbar_wait(B_PFULL, ph, wctx));
      FA_SWT(lane == 0 && wg == 0 && j == 0, 22);
      if (ok) {
        tc_fence_after();
        const uint64_t dV = smem_desc_sw128(rv, SW_Q_BYTES, 1024);
        for (int kk = 0; kk < p.n_s / 16; ++kk)
          sh_mma_ts(tO, tS + 8 * kk, dV + (uint64_t)((kk * 2048) >> 4), IDESC_PV, kk > 0 ? 1u : 0u);
        mma_commit_elect(B_OFULL);
      }
    }
    ok = __all_sync(0xffffffffu, ok && mbar_wait(B_OFULL, ph, wctx));
    if (!ok) break;
    FA_SWT(leader && j == 0, 6 + wg);
    tc_fence_after();
    // K and V of the next tile, once this tile's MMAs no longer read the slot
    if (j + 1 < mine) {
      const SwTile xn = sw_decode(t0 + wg + SW_WGS * (j + 1), p);
      if (xn.kv != kv_cur) {
        if (leader) issue_kv(xn);
        kv_cur = xn.kv;
        ++kv_loads;
      }
    }
    // ---------------------------------------------------------------- epilogue
    // O / l into the tile's Q stage in the 128-byte-swizzled layout (16-byte
    // piece q of row r at r * 128 + (q ^ (r % 8)) * 16), then one TMA store.
    const float inv_l = 1.f / l;
    const uint32_t qs = rq + s * SW_Q_BYTES;
    {
      float ov[64];
      tmem_ld64(tOl, ov);
      const uint32_t rowb = qs + r * 128;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float* o8 = ov + 8 * q;
        st_shared_v4(rowb + ((q ^ (r & 7)) << 4), sh_pack2<T>(o8[0] * inv_l, o8[1] * inv_l),
                     sh_pack2<T>(o8[2] * inv_l, o8[3] * inv_l), sh_pack2<T>(o8[4] * inv_l, o8[5] * inv_l),
                     sh_pack2<T>(o8[6] * inv_l, o8[7] * inv_l));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive_warp(B_OSTAGED);
    FA_SWT(warp == 0 && lane == 0 && j == 0, 25);
    if (row < p.Nq && p.lse != nullptr &&
        FA_INDEX_OK(status_word, ((long long)x.b * p.H + x.h) * p.Nq + row < (long long)p.B * p.H * p.Nq))
      p.lse[((long long)x.b * p.H + x.h) * p.Nq + row] = (m2 + __log2f(l)) * 0.69314718055994530942f;
    if (lead_warp) {
      // the store reads the stage; the next S may overwrite O once every warp has read it
      if (lane == 0) {
        ok = mbar_wait(B_OSTAGED, ph, wctx);
        if (ok) {
          if (p.bsnd)
            sh_tma_store_4d(&tm_o, qs, 0, x.h, x.qt * 128, x.b);
          else
            sh_tma_store_4d(&tm_o, qs, 0, x.qt * 128, x.h, x.b);
          sh_bulk_commit();
          if (q_issued < mine) {  // refill this stage once the store has read it
            sh_bulk_wait_read0();
            issue_q(q_issued);
            ++q_issued;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      tc_fence_after();
    }
  }
  FA_SWT(leader, 10 + wg);

  if (lead_warp) {
    // Every MMA this warp issued finishes, and every copy its leader started
    // lands or is read, before the CTA frees tensor memory and exits.
    mma_commit_elect(B_DRAIN);
    WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
    volatile int no_abort = 0;
    drain.abort_flag = &no_abort;
    mbar_wait(B_DRAIN, 0, drain);
    if (lane == 0 && mine > 0) {
      // the last Q load into each stage, and the last K/V load
      for (int s = 0; s < p.ns; ++s) {
        int last = -1;
        for (int j = s; j < q_issued; j += p.ns) last = j;
        if (last >= 0) mbar_wait(B_QFULL + 8 * s, (uint32_t)((last / p.ns) & 1), drain);
      }
      mbar_wait(B_KVFULL, (uint32_t)((kv_loads - 1) & 1), drain);
      // the stores have read their stages; their writes complete with the grid
      sh_bulk_wait_read0();
    }
    __syncwarp();
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
  FA_SWT(threadIdx.x == 0, 14);
}

}  // namespace fa
