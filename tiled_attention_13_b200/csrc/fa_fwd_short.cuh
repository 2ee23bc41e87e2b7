// fa_fwd_short.cuh -- tensor-core attention forward for short key sequences,
// Nkv <= 128 (every query tile sees a single KV tile), bf16 or fp16 inputs,
// fp32 accumulation, head dim D in {64, 128}.
//
// The case the pages single out is the AIGC cross-attention of page 3 ("ops-nn
// efficient attention for AIGC", section 四: 4096 latent-image tokens attend to
// 77 text tokens).  With one KV tile there is no online rescaling: each row's
// softmax is exact in one pass (page 1, "CANN ops-transformer
// FlashAttentionScore", section 在线 Softmax 的数学原理拆解, with a single
// block), so the work per query tile is S = Q K^T, one softmax, O = P V and the
// write of O.  The arithmetic is small next to the bytes: Q is read and O
// written once (about 74 FLOP per byte for the 77-key case), so the kernel is
// an HBM stream, and its design is about keeping the loads and stores of many
// query tiles in flight rather than about the tensor pipe.
//
// B200 mapping:
//   grid        <= #SM persistent CTAs; CTA c owns a contiguous range of query
//               tiles (b, h, qt), qt fastest, so consecutive tiles share K/V.
//               No work counter: the schedule is static (all tiles cost the
//               same), and the kernel uses no memory beyond its operands.
//   warp 9      TMA producer: Q tiles into a ring of KQ stages; K and V of the
//               current (batch, K/V head) into one of two slots, loaded again
//               only when the head changes.  Rows past Nkv read as zeros.
//   warp 8      TMEM allocator and MMA issuer (whole warp, elect.sync):
//               S_b = Q K^T (N = Nkv rounded up to 16), then, once the softmax
//               has written P, O_b = P V over ceil(Nkv / 16) key steps.
//   warps 0-7   two softmax/epilogue warpgroups; warpgroup b takes the CTA's
//               tiles b, b + 2, ... in TMEM buffer b.  A thread owns one query
//               row (one TMEM lane): row max, p = 2^(s * scale * log2 e - m),
//               l = sum p, P packed to 16 bits over the S columns it has read.
//               After P V: O / l is written in the 128-byte-swizzled layout
//               into the shared-memory stage the tile's Q came from, and one
//               thread stores it with a TMA tensor store (rows past Nq are
//               clipped by the tensor map), then frees the stage.  LSE =
//               (m + log2 l) ln 2.
//
//   TMEM (512 columns): buffer b at 256 b: S [0, 128), O [128, 128 + D).
//   Two buffers let one warpgroup's softmax overlap the other's epilogue and
//   the MMAs of both.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "ptx.cuh"
#include "tc_common.cuh"

namespace fa {

// Optional timeline (compile with -DFA_TRACE_SHORT): %globaltimer stamps of
// a few events of every CTA, readable through fa_debug_short_trace_read().
#ifdef FA_TRACE_SHORT
constexpr int SHT_CTAS = 160, SHT_EV = 16;
__device__ unsigned long long g_trace_short[SHT_CTAS * SHT_EV];
#define FA_SHT(cond, ev)                                                         \
  do {                                                                           \
    if ((cond) && blockIdx.x < SHT_CTAS) g_trace_short[blockIdx.x * SHT_EV + (ev)] = globaltimer_ns(); \
  } while (0)
#else
#define FA_SHT(cond, ev) \
  do {                   \
  } while (0)
#endif

constexpr int SH_WARP_MMA = 8;
constexpr int SH_WARP_TMA = 9;
constexpr int SH_THREADS = 32 * 10;
constexpr int SH_MAX_NKV = 128;

template <int D>
struct ShCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;           // 128 rows x D 16-bit values
  static constexpr int CHUNKS = D / 64;                    // 128-byte-wide column chunks per tile
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int KQ = (D == 64) ? 8 : 3;             // Q / O-staging stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = KQ * TILE_BYTES;            // 2 K slots
  static constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;     // 2 V slots
  static constexpr int OFF_BAR = OFF_V + 2 * TILE_BYTES;
  // q_full[KQ] q_empty[KQ] kv_full[2] kv_empty[2] s_full[2] p_full[2] o_full[2] o_staged[2] drain
  static constexpr int NBAR = 2 * KQ + 12 + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 /*tmem slot + abort*/ + 1024 /*align slack*/;
  static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory of sm_100");
};

struct ShParams {
  float* lse;        // [B, H, Nq] or nullptr
  int B, H, Nq, Nkv;
  int bsnd;          // 1: [B, N, H, D] rows, 0: [B, H, N, D]
  int causal;        // key j visible to query i iff j <= i
  float scale_log2;  // softmax scale * log2(e)
  int qtiles;        // ceil(Nq / 128)
  int n_tiles;       // B * H * qtiles
  int kv_group;      // query heads per K/V head
  int n_s;           // S columns computed: Nkv rounded up to 16
  int kv_steps;      // 16-key steps of P V: ceil(Nkv / 16)
  uint64_t timeout_ns;
  int fault_mode;
};

// Query tile t -> (b, h, qt) and the key of its K/V (batch, K/V head).
struct ShTile {
  int b, h, qt, kv;
};
__host__ __device__ __forceinline__ ShTile sh_decode(int t, const ShParams& p) {
  ShTile x;
  const int bh = t / p.qtiles;
  x.qt = t - bh * p.qtiles;
  x.b = bh / p.H;
  x.h = bh - x.b * p.H;
  x.kv = x.b * (p.H / p.kv_group) + x.h / p.kv_group;
  return x;
}

// Tiles [t0, t1) of CTA c out of G: contiguous, sizes differing by at most one.
__host__ __device__ __forceinline__ void sh_range(int c, int G, int n_tiles, int& t0, int& t1) {
  t0 = (int)(((long long)c * n_tiles) / G);
  t1 = (int)(((long long)(c + 1) * n_tiles) / G);
}


template <int D, typename T>
__global__ void __launch_bounds__(SH_THREADS, 1)
    fa_fwd_short_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        ShParams p, unsigned int* status_word) {
  using C = ShCfg<D>;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int KQ = C::KQ;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment: the 128-byte swizzle pattern is anchored there.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  const int B_QFULL = 0, B_QEMPTY = KQ, B_KVFULL = 2 * KQ, B_KVEMPTY = 2 * KQ + 2, B_SFULL = 2 * KQ + 4,
            B_PFULL = 2 * KQ + 6, B_OFULL = 2 * KQ + 8, B_OSTAGED = 2 * KQ + 10, B_DRAIN = 2 * KQ + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int t0, t1;
  sh_range(blockIdx.x, gridDim.x, p.n_tiles, t0, t1);
  const int n = t1 - t0;  // this CTA's tiles, >= 1
  FA_SHT(threadIdx.x == 0, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < KQ; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_KVFULL + i), 1);
      mbar_init(bar(B_KVEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + i), 4);  // one arrival per warp of the warpgroup
      mbar_init(bar(B_OFULL + i), 1);
      mbar_init(bar(B_OSTAGED + i), 4);
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == SH_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == SH_WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wctx{abort_flag, status_word, p.timeout_ns, 1u};
  FA_SHT(threadIdx.x == 0, 1);

  if (warp == SH_WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      int cur_kv = -1, kv_loads = 0;
      int q_last[KQ];    // last tile index loaded into each stage (-1: none)
      int kv_last[2];    // last load count of each K/V slot (-1: none)
      for (int s = 0; s < KQ; ++s) q_last[s] = -1;
      kv_last[0] = kv_last[1] = -1;
      for (int i = 0; i < n; ++i) {
        const ShTile x = sh_decode(t0 + i, p);
        if (x.kv != cur_kv) {
          const int slot = kv_loads & 1;
          if (!mbar_wait(bar(B_KVEMPTY + slot), ((kv_loads >> 1) & 1) ^ 1, wctx)) break;
          mbar_arrive_expect_tx(bar(B_KVFULL + slot), 2 * C::TILE_BYTES);
          const int hk = x.h / p.kv_group;
          const uint32_t kd = sbase + C::OFF_K + slot * C::TILE_BYTES, vd = sbase + C::OFF_V + slot * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd) {
              tma_load_4d(kd + c * C::CHUNK_BYTES, &tm_k, bar(B_KVFULL + slot), c * 64, hk, 0, x.b, pol_kv);
              tma_load_4d(vd + c * C::CHUNK_BYTES, &tm_v, bar(B_KVFULL + slot), c * 64, hk, 0, x.b, pol_kv);
            } else {
              tma_load_4d(kd + c * C::CHUNK_BYTES, &tm_k, bar(B_KVFULL + slot), c * 64, 0, hk, x.b, pol_kv);
              tma_load_4d(vd + c * C::CHUNK_BYTES, &tm_v, bar(B_KVFULL + slot), c * 64, 0, hk, x.b, pol_kv);
            }
          }
          kv_last[slot] = kv_loads;
          cur_kv = x.kv;
          ++kv_loads;
        }
        const int s = i % KQ;
        if (!mbar_wait(bar(B_QEMPTY + s), ((i / KQ) & 1) ^ 1, wctx)) break;
        mbar_arrive_expect_tx(bar(B_QFULL + s), C::TILE_BYTES);
        const uint32_t qd = sbase + C::OFF_Q + s * C::TILE_BYTES;
        const int row0 = x.qt * 128;
        for (int c = 0; c < C::CHUNKS; ++c) {
          if (p.bsnd)
            tma_load_4d(qd + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + s), c * 64, x.h, row0, x.b, pol_q);
          else
            tma_load_4d(qd + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + s), c * 64, row0, x.h, x.b, pol_q);
        }
        q_last[s] = i;
      }
      FA_SHT(true, 11);
      // Every copy this thread started lands before the CTA may exit.
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      for (int s = 0; s < KQ; ++s)
        if (q_last[s] >= 0) mbar_wait(bar(B_QFULL + s), (q_last[s] / KQ) & 1, drain);
      for (int sl = 0; sl < 2; ++sl)
        if (kv_last[sl] >= 0) mbar_wait(bar(B_KVFULL + sl), (kv_last[sl] >> 1) & 1, drain);
    }
    __syncwarp();
  } else if (warp == SH_WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = idesc_f16(IS_BF16, false, 128, (uint32_t)p.n_s);
    constexpr uint32_t IDESC_PV = idesc_f16(IS_BF16, true, 128, D);
    const uint64_t dQ0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dK0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
    // Event-driven issue: P V of tile jp as soon as its P is written, S of
    // tile js as soon as its Q (and, on a head change, its K/V) has landed and
    // its TMEM buffer is free (P V of tile js - 2 issued: the tensor pipe runs
    // a CTA's MMAs in issue order, so S(js) overwrites P(js - 2) only after it
    // was read).  P V comes first when both are ready.  Polls are warp-wide;
    // a stretch with nothing ready is bounded like every other wait.
    auto ready = [&](int b, uint32_t ph) { return __all_sync(0xffffffffu, mbar_poll(bar(b), ph)); };
    int js = 0, jp = 0;
    int s_kv = -1, s_loads = 0;  // K/V slot bookkeeping of the S side
    int v_kv = -1, v_loads = 0;  // and of the P V side
    uint64_t idle_since = 0;
    bool ok = true;
    while (jp < n) {
      bool did = false;
      if (jp < js && ready(B_PFULL + (jp & 1), (jp >> 1) & 1)) {
        const int b = jp & 1;
        const ShTile x = sh_decode(t0 + jp, p);
        if (x.kv != v_kv) {
          v_kv = x.kv;
          ++v_loads;
        }
        const int slot = (v_loads - 1) & 1;
        tc_fence_after();
        const uint32_t tS = tmem + 256 * b, tO = tS + 128;
        const uint64_t dV = dV0 + (uint64_t)((slot * C::TILE_BYTES) >> 4);
        for (int kk = 0; kk < p.kv_steps; ++kk)
          sh_mma_ts(tO, tS + 8 * kk, dV + (uint64_t)((kk * 2048) >> 4), IDESC_PV, kk > 0 ? 1u : 0u);
        mma_commit_elect(bar(B_OFULL + b));
        FA_SHT(lane == 0 && jp == 0, 3);
        FA_SHT(lane == 0 && jp == n - 1, 4);
        // the K/V slot is free once the last tile that reads it is done
        if (jp + 1 == n || sh_decode(t0 + jp + 1, p).kv != x.kv) mma_commit_elect(bar(B_KVEMPTY + slot));
        ++jp;
        did = true;
      } else if (js < n && js < jp + 2) {
        const ShTile x = sh_decode(t0 + js, p);
        const bool new_kv = x.kv != s_kv;
        const int st = js % KQ;
        if ((!new_kv || ready(B_KVFULL + (s_loads & 1), (s_loads >> 1) & 1)) && ready(B_QFULL + st, (js / KQ) & 1)) {
          if (new_kv) {
            s_kv = x.kv;
            ++s_loads;
          }
          const int slot = (s_loads - 1) & 1;
          tc_fence_after();
          const uint32_t tS = tmem + 256 * (js & 1);
          const uint64_t dQ = dQ0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
          const uint64_t dK = dK0 + (uint64_t)((slot * C::TILE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = (uint64_t)(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4);
            sh_mma_ss(tS, dQ + o, dK + o, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit_elect(bar(B_SFULL + (js & 1)));
          FA_SHT(lane == 0 && js == 0, 2);
          ++js;
          did = true;
        }
      }
      if (did) {
        idle_since = 0;
        continue;
      }
      // nothing was ready: back off, and give up on abort or after the wait limit
      poll_backoff();
      const uint64_t now = globaltimer_ns();
      if (idle_since == 0) idle_since = now;
      const int give_up = __shfl_sync(0xffffffffu, (*abort_flag != 0 || now - idle_since > p.timeout_ns) ? 1 : 0, 0);
      if (give_up) {
        if (lane == 0 && *abort_flag == 0) {
          *abort_flag = 1;
          atomicOr(status_word, 1u);
        }
        ok = false;
        break;
      }
    }
    (void)ok;
    // Let every MMA this warp issued finish before the CTA frees TMEM.
    mma_commit_elect(bar(B_DRAIN));
    {
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_DRAIN), 0, drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int b = warp >> 2;               // warpgroup = TMEM buffer
    const int r = (warp & 3) * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + 256 * b, tO = tS + 128;
    const float sl2 = p.scale_log2;
    const int nc = (p.Nkv + 31) >> 5;  // 32-key chunks holding keys
    const bool storer = (warp & 3) == 0 && lane == 0;
    bool ok = true;
    for (int i = b; i < n && ok; i += 2) {
      const ShTile x = sh_decode(t0 + i, p);
      const int row = x.qt * 128 + r;
      const uint32_t ph = (uint32_t)((i >> 1) & 1);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + b), ph, wctx));
      if (!ok) break;
      FA_SHT(storer && i == 0, 5);
      FA_SHT(storer && i == 1, 10);
      tc_fence_after();
      const int lim = p.causal ? (row + 1 < p.Nkv ? row + 1 : p.Nkv) : p.Nkv;  // visible keys [0, lim)
      float m2, l;
      uint64_t acc2 = 0ull;
      // exps of 32 keys from registers to packed P columns [16c, 16c + 16)
      auto exps32 = [&](const float* sc, int c, uint64_t scale2, uint64_t negm2) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float s0 = 32 * c + 2 * t < lim ? sc[2 * t] : -INFINITY;
          const float s1 = 32 * c + 2 * t + 1 < lim ? sc[2 * t + 1] : -INFINITY;
          const uint64_t x2 = f2_fma(f2_pack(s0, s1), scale2, negm2);
          float x0, x1;
          f2_unpack(x2, x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          acc2 = f2_add(acc2, f2_pack(p0, p1));
          pk[t] = sh_pack2<T>(p0, p1);
        }
        sh_tmem_st16(tS + 16 * c, pk);
      };
      // Up to 96 keys: one pass, the scores loaded together and kept in
      // registers.  More: two passes over tensor memory, 32 columns at a time
      // (the row max, then the exps; P for keys [32c, 32c + 32) goes to packed
      // columns [16c, 16c + 16), which pass 2 has already read by then).
      auto one_pass = [&](auto NCc) {
        constexpr int NC = decltype(NCc)::value;
        float sc[32 * NC];
        if constexpr (NC == 1)
          tmem_ld32(tS, *reinterpret_cast<float(*)[32]>(sc));
        else if constexpr (NC == 2)
          tmem_ld64(tS, *reinterpret_cast<float(*)[64]>(sc));
        else
          tmem_ld96(tS, sc);
        float mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < 32 * NC; ++t) mx = fmaxf(mx, t < lim ? sc[t] : -INFINITY);
        m2 = mx * sl2;  // finite: every row sees key 0
        const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m2, -m2);
#pragma unroll
        for (int c = 0; c < NC; ++c) exps32(sc + 32 * c, c, scale2, negm2);
      };
      if (nc == 1) {
        one_pass(std::integral_constant<int, 1>{});
      } else if (nc == 2) {
        one_pass(std::integral_constant<int, 2>{});
      } else if (nc == 3) {
        one_pass(std::integral_constant<int, 3>{});
      } else {
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < nc; ++c) {
          float sc[32];
          tmem_ld32(tS + 32 * c, sc);
#pragma unroll
          for (int t = 0; t < 32; ++t) mx = fmaxf(mx, 32 * c + t < lim ? sc[t] : -INFINITY);
        }
        m2 = mx * sl2;
        const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m2, -m2);
#pragma unroll 1
        for (int c = 0; c < nc; ++c) {
          float sc[32];
          tmem_ld32(tS + 32 * c, sc);
          exps32(sc, c, scale2, negm2);
        }
      }
      {
        float a0, a1;
        f2_unpack(acc2, a0, a1);
        l = a0 + a1;
      }
      tmem_wait_st();
      tc_fence_before();
      if (p.fault_mode != 1) mbar_arrive_warp(bar(B_PFULL + b));
      FA_SHT(storer && i == 0, 6);
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL + b), ph, wctx));
      if (!ok) break;
      FA_SHT(storer && i == 0, 7);
      tc_fence_after();
      const float inv_l = 1.f / l;
      // O / l into the tile's Q stage (its MMAs are done), 128-byte swizzle:
      // 16-byte chunk j of row r of a 64-column chunk sits at r*128 + (j ^ (r % 8))*16.
      const int s = i % KQ;
      const uint32_t qs = sbase + C::OFF_Q + s * C::TILE_BYTES;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float ov[32];
        tmem_ld32(tO + 32 * c, ov);
        const uint32_t rowb = qs + (c >> 1) * C::CHUNK_BYTES + r * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float* o8 = ov + 8 * j;
          const int piece = 4 * (c & 1) + j;
          st_shared_v4(rowb + ((piece ^ (r & 7)) << 4), sh_pack2<T>(o8[0] * inv_l, o8[1] * inv_l),
                       sh_pack2<T>(o8[2] * inv_l, o8[3] * inv_l), sh_pack2<T>(o8[4] * inv_l, o8[5] * inv_l),
                       sh_pack2<T>(o8[6] * inv_l, o8[7] * inv_l));
        }
      }
      // Each warp makes its writes visible to the async proxy and signals;
      // one thread waits (bounded) for the four warps and stores the tile.
      fence_proxy_async_smem();
      mbar_arrive_warp(bar(B_OSTAGED + b));
      if (storer && !mbar_wait(bar(B_OSTAGED + b), ph, wctx)) ok = false;
      if (storer && ok) {
        const int row0 = x.qt * 128;
        for (int g = 0; g < C::CHUNKS; ++g) {
          if (p.bsnd)
            sh_tma_store_4d(&tm_o, qs + g * C::CHUNK_BYTES, g * 64, x.h, row0, x.b);
          else
            sh_tma_store_4d(&tm_o, qs + g * C::CHUNK_BYTES, g * 64, row0, x.h, x.b);
        }
        sh_bulk_commit();
        FA_SHT(i == 0, 8);
        sh_bulk_wait_read0();  // the stage may be refilled once the store has read it
        FA_SHT(i == 0, 9);
        mbar_arrive(bar(B_QEMPTY + s));
      }
      if (row < p.Nq && p.lse != nullptr &&
          FA_INDEX_OK(status_word, ((long long)x.b * p.H + x.h) * p.Nq + row < (long long)p.B * p.H * p.Nq))
        p.lse[((long long)x.b * p.H + x.h) * p.Nq + row] = (m2 + __log2f(l)) * 0.69314718055994530942f;
    }
    if (storer) sh_bulk_wait0();  // this thread's stores are complete before the CTA exits
    FA_SHT(storer && b == 0, 12);
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == SH_WARP_MMA) tmem_dealloc(tmem, 512);
  FA_SHT(threadIdx.x == 0, 13);
}

}  // namespace fa
