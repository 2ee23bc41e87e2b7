// fa_fwd_tc2.cuh -- tensor-core attention forward for sm_100a with one query
// row per softmax thread: bf16 or fp16 inputs, fp32 accumulation, head dim D
// in {64, 128}, contiguous K/V, causal or not, grouped K/V heads.
//
// Method: as the two-tile kernel (fa_fwd_tc.cuh): page 1, "CANN
// ops-transformer FlashAttentionScore", section 分块 Tiling 的计算骨架 (every
// query tile walks its K/V tiles with the online softmax) and page 3, "ops-nn
// efficient attention for AIGC", section 2.2 (unnormalised accumulator, one
// division by l at the end), in the exp2 domain with a lazily moved reference
// max (moved only when a step's max exceeds it by more than 2^8).
//
// What differs from the two-tile kernel is the softmax's thread layout.  There
// a row's 128 scores are split between two warpgroups, which must agree on
// the reference max through shared memory every step.  Here one thread owns
// one query row and all 128 scores of a step:
//
//   warps 0-3   softmax and epilogue of query tile 0 of the unit
//   warps 4-7   softmax and epilogue of query tile 1
//   warp 8      TMEM allocator and MMA issuer (whole warp, elect.sync)
//   warp 9      ticket claims, unit decode (the two-tile kernel's L2-chunked,
//               heaviest-first order), TMA loads of Q0, Q1 and the K/V ring
//
// so a row's max is thread-local, each sub-partition holds one warp of each
// tile (one tile's exps overlap the other tile's MMAs and row work), and the
// P of a step is handed over in two halves (keys 0-63, then 64-127) so that
// the first half of P V runs while the second half's exps are computed.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1
// [256+D,256+2D); P_i (16-bit pairs) for keys 0-63 overwrites S_i columns
// [0,32), keys 64-127 columns [32,64), after the thread has read all of S_i.
// MMA order per KV step j (tile i = 0, 1): O_i += P_i(j-1) V_(j-1) (two
// halves, each as soon as it is handed over), then S_i(j) = Q_i K_j^T; the
// tensor pipe runs a CTA's MMAs in issue order, so S_i(j) overwrites P_i(j-1)
// only after P V has read it, and O_i is quiescent when S_i(j) is signalled
// (the softmax may rescale it in place).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "tc_common.cuh"
#include "fa_fwd_tc.cuh"     // TcParams, Unit, decode_unit, SchedSlot
#include "ptx.cuh"

namespace fa {

constexpr int T2_SOFTMAX_WARPS = 8;
constexpr int T2_WARP_MMA = 8;
constexpr int T2_WARP_TMA = 9;
constexpr int T2_THREADS = 32 * 10;
#ifndef FA_T2_POLY_EVERY
#define FA_T2_POLY_EVERY 4
#endif
// > 0: on steps without masked scores, one exp pair in T2_POLY_EVERY is
// computed on the FMA pipe (exp2_poly_x2) instead of the SFU; 4 measured best
constexpr int T2_POLY_EVERY = FA_T2_POLY_EVERY;
constexpr int T2_POLY_MOD = T2_POLY_EVERY > 0 ? T2_POLY_EVERY : 1;

template <int D>
struct T2Cfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int KST = (D == 128) ? 2 : 4;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
  static constexpr int OFF_UNIT = OFF_V + KST * TILE_BYTES;
  static constexpr int UNIT_SLOTS = 4;
  static constexpr int OFF_BAR = OFF_UNIT + 64 * UNIT_SLOTS;
  // q_full[2] q_empty[2] k_full/k_empty/v_full/v_empty[KST] s_full[2] p_a[2] p_b[2] o_full[2]
  // u_full[SLOTS] u_empty[SLOTS] drain
  static constexpr int NBAR = 4 + 4 * KST + 8 + 2 * UNIT_SLOTS + 1;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory of sm_100");
  static constexpr uint32_t TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + D;
};

template <int D, typename T>
__global__ void __launch_bounds__(T2_THREADS, 1)
    fa_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, TcParams p, unsigned int* status_word) {
  using C = T2Cfg<D>;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int KST = C::KST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + C::OFF_UNIT);
  const int B_QFULL = 0, B_QEMPTY = 2, B_KFULL = 4, B_KEMPTY = 4 + KST, B_VFULL = 4 + 2 * KST,
            B_VEMPTY = 4 + 3 * KST, B_SFULL = 4 + 4 * KST, B_PA = B_SFULL + 2, B_PB = B_SFULL + 4,
            B_OFULL = B_SFULL + 6, B_UFULL = B_SFULL + 8, B_UEMPTY = B_UFULL + C::UNIT_SLOTS,
            B_DRAIN = B_UEMPTY + C::UNIT_SLOTS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto ring_put = [&](int slot, int tk, const Unit& w) {
    volatile int* e = unit_ring + 16 * slot;
    e[0] = tk; e[1] = w.b; e[2] = w.h; e[3] = w.qt0; e[4] = w.active1; e[5] = w.n0; e[6] = w.n1;
  };
  auto ring_get = [&](int slot, Unit& w) -> int {
    volatile const int* e = unit_ring + 16 * slot;
    w.b = e[1]; w.h = e[2]; w.qt0 = e[3]; w.active1 = e[4]; w.n0 = e[5]; w.n1 = e[6];
    w.lo0 = 0; w.s1 = 0;
    return e[0];
  };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_QFULL + i), 1);
      mbar_init(bar(B_QEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PA + i), 4);  // one arrival per warp of the tile's warpgroup
      mbar_init(bar(B_PB + i), 4);
      mbar_init(bar(B_OFULL + i), 1);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int i = 0; i < C::UNIT_SLOTS; ++i) {
      mbar_init(bar(B_UFULL + i), 1);
      mbar_init(bar(B_UEMPTY + i), 1 + T2_SOFTMAX_WARPS);  // MMA warp + softmax warps
    }
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == T2_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == T2_WARP_TMA && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wctx{abort_flag, status_word, p.timeout_ns, 1u};

  if (warp == T2_WARP_TMA) {
    // ------------------------------------------------------------ tickets and TMA loads
    if (lane == 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t q_phase[2] = {0, 0};
      int st = 0;
      uint32_t kv_phase = 0;
      uint32_t k_issued[KST], v_issued[KST], q_issued[2];
      bool k_pend[KST], v_pend[KST], q_pend[2];
      for (int s = 0; s < KST; ++s) { k_pend[s] = v_pend[s] = false; k_issued[s] = v_issued[s] = 0; }
      q_pend[0] = q_pend[1] = false; q_issued[0] = q_issued[1] = 0;
      bool ok = true;
      int uslot = 0;
      uint32_t uphase = 0;
      while (ok) {
        const unsigned int t = atomicAdd(&p.sched->next, 1u);
        const int tk = (t < (unsigned int)p.n_units) ? (int)t : -1;
        const Unit w = decode_unit(tk < 0 ? 0 : tk, p);
        if (!mbar_wait(bar(B_UEMPTY + uslot), uphase ^ 1, wctx)) break;
        ring_put(uslot, tk, w);
        mbar_arrive(bar(B_UFULL + uslot));
        if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
        if (tk < 0) break;
        for (int i = 0; i < 2 && ok; ++i) {
          if (i == 1 && !w.active1) break;
          if (!mbar_wait(bar(B_QEMPTY + i), q_phase[i] ^ 1, wctx)) { ok = false; break; }
          const uint32_t dst = sbase + C::OFF_Q + i * C::TILE_BYTES;
          mbar_arrive_expect_tx(bar(B_QFULL + i), C::TILE_BYTES);
          const int row0 = (w.qt0 + i) * 128;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd)
              tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + i), c * 64, w.h, row0, w.b, pol_q);
            else
              tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + i), c * 64, row0, w.h, w.b, pol_q);
          }
          q_pend[i] = true; q_issued[i] = q_phase[i];
          q_phase[i] ^= 1;
        }
        const int N = w.n0 > w.n1 ? w.n0 : w.n1;
        const int hk = w.h / p.kv_group;
        for (int j = 0; j < N && ok; ++j) {
          const int kv0 = j * 128;
          if (!mbar_wait(bar(B_KEMPTY + st), kv_phase ^ 1, wctx)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(B_KFULL + st), C::TILE_BYTES);
          const uint32_t kdst = sbase + C::OFF_K + st * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd)
              tma_load_4d(kdst + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + st), c * 64, hk, kv0, w.b, pol_kv);
            else
              tma_load_4d(kdst + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + st), c * 64, kv0, hk, w.b, pol_kv);
          }
          k_pend[st] = true; k_issued[st] = kv_phase;
          if (!mbar_wait(bar(B_VEMPTY + st), kv_phase ^ 1, wctx)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(B_VFULL + st), C::TILE_BYTES);
          const uint32_t vdst = sbase + C::OFF_V + st * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd)
              tma_load_4d(vdst + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + st), c * 64, hk, kv0, w.b, pol_kv);
            else
              tma_load_4d(vdst + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + st), c * 64, kv0, hk, w.b, pol_kv);
          }
          v_pend[st] = true; v_issued[st] = kv_phase;
          if (++st == KST) { st = 0; kv_phase ^= 1; }
        }
      }
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      for (int s = 0; s < KST; ++s) {
        if (k_pend[s]) mbar_wait(bar(B_KFULL + s), k_issued[s], drain);
        if (v_pend[s]) mbar_wait(bar(B_VFULL + s), v_issued[s], drain);
      }
      for (int i = 0; i < 2; ++i)
        if (q_pend[i]) mbar_wait(bar(B_QFULL + i), q_issued[i], drain);
    }
    __syncwarp();
  } else if (warp == T2_WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_S = idesc_f16(IS_BF16, false, 128, 128);
    constexpr uint32_t IDESC_PV = idesc_f16(IS_BF16, true, 128, D);
    const uint64_t dQ[2] = {smem_desc_sw128(sbase + C::OFF_Q, 16, 1024),
                            smem_desc_sw128(sbase + C::OFF_Q + C::TILE_BYTES, 16, 1024)};
    const uint64_t dK0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
    uint32_t q_phase[2] = {0, 0}, kv_phase = 0, pa_phase[2] = {0, 0}, pb_phase[2] = {0, 0};
    int st = 0;
    bool ok = true;
    const uint32_t tS[2] = {tmem + C::TMEM_S0, tmem + C::TMEM_S1};
    const uint32_t tO[2] = {tmem + C::TMEM_O0, tmem + C::TMEM_O1};
    auto wait_all = [&](int b, uint32_t ph) { return __all_sync(0xffffffffu, mbar_wait(bar(b), ph, wctx)); };
    int uslot = 0;
    uint32_t uphase = 0;
    while (ok) {
      if (!wait_all(B_UFULL + uslot, uphase)) break;
      Unit w;
      const int tk = ring_get(uslot, w);
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      const int n[2] = {w.n0, w.n1};
      const int N = w.n0 > w.n1 ? w.n0 : w.n1;
      for (int i = 0; i < 2 && ok; ++i) {
        if (n[i] == 0) continue;
        if (!wait_all(B_QFULL + i, q_phase[i])) ok = false;
        q_phase[i] ^= 1;
      }
      int st_prev = 0;
      uint32_t ph_prev = 0;
      for (int j = 0; j <= N && ok; ++j) {
        bool k_ready = false;
        if (j > 0 && !wait_all(B_VFULL + st_prev, ph_prev)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dK = dK0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
        const uint64_t dV = dV0 + (uint64_t)((st_prev * C::TILE_BYTES) >> 4);
        for (int i = 0; i < 2 && ok; ++i) {
          if (n[i] == 0) continue;
          if (j >= 1 && j - 1 < n[i]) {
            // O_i += P_i(j-1) V_(j-1): keys 0-63 (k-steps 0-3), then 64-127
            if (!wait_all(B_PA + i, pa_phase[i])) { ok = false; break; }
            pa_phase[i] ^= 1;
            tc_fence_after();
            mma_ts4_elect(tO[i], tS[i], dV, tS[i] + 8, dV + (2048 >> 4), tS[i] + 16, dV + (4096 >> 4), tS[i] + 24,
                          dV + (6144 >> 4), IDESC_PV, j - 1 > 0 ? 1u : 0u);
            if (!wait_all(B_PB + i, pb_phase[i])) { ok = false; break; }
            pb_phase[i] ^= 1;
            tc_fence_after();
            mma_ts4_elect(tO[i], tS[i] + 32, dV + (8192 >> 4), tS[i] + 40, dV + (10240 >> 4), tS[i] + 48,
                          dV + (12288 >> 4), tS[i] + 56, dV + (14336 >> 4), IDESC_PV, 1u);
            if (j - 1 == n[i] - 1) mma_commit_elect(bar(B_OFULL + i));
            // V_(j-1) is free once the last tile that reads it is done
            const bool t1_uses = n[1] > 0 && j - 1 < n[1];
            if (i == 1 || !t1_uses) mma_commit_elect(bar(B_VEMPTY + st_prev));
          }
          if (j < n[i]) {
            if (!k_ready) {
              if (!wait_all(B_KFULL + st, kv_phase)) { ok = false; break; }
              k_ready = true;
              tc_fence_after();
            }
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c) {
              const uint64_t o0 = (uint64_t)((c * C::CHUNK_BYTES) >> 4);
              mma_ss4_elect(tS[i], dQ[i] + o0, dK + o0, dQ[i] + o0 + 2, dK + o0 + 2, dQ[i] + o0 + 4, dK + o0 + 4,
                            dQ[i] + o0 + 6, dK + o0 + 6, IDESC_S, c > 0 ? 1u : 0u);
            }
            mma_commit_elect(bar(B_SFULL + i));
            if (j == n[i] - 1) mma_commit_elect(bar(B_QEMPTY + i));
          }
        }
        if (!ok) break;
        if (j < N) mma_commit_elect(bar(B_KEMPTY + st));
        st_prev = st;
        ph_prev = kv_phase;
        if (j < N) {
          if (++st == KST) { st = 0; kv_phase ^= 1; }
        }
      }
    }
    mma_commit_elect(bar(B_DRAIN));
    {
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_DRAIN), 0, drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-7)
    const int tile = warp >> 2;
    const int r = (warp & 3) * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (tile ? C::TMEM_S1 : C::TMEM_S0);
    const uint32_t tO = tmem + lane_base + (tile ? C::TMEM_O1 : C::TMEM_O0);
    const float sl2 = p.scale_log2;
    uint32_t s_phase = 0, o_phase = 0;
    bool ok = true;
    int uslot = 0;
    uint32_t uphase = 0;
    while (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_UFULL + uslot), uphase, wctx));
      if (!ok) break;
      Unit w;
      const int tk = ring_get(uslot, w);
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      const int n = tile ? w.n1 : w.n0;
      if (n == 0) continue;
      const int qt = w.qt0 + tile;
      const int row = qt * 128 + r;
      const int lim_c = p.causal ? (row + 1 < p.Nkv ? row + 1 : p.Nkv) : p.Nkv;  // visible keys [0, lim_c)
      float m_ref = -INFINITY;  // reference max (log2 domain)
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + tile), s_phase, wctx));
        if (!ok) break;
        s_phase ^= 1;
        tc_fence_after();
        const int col0 = j * 128;
        const bool need_mask = (col0 + 128 > p.Nkv) || (p.causal && col0 + 127 > qt * 128);
        // Pass 1: the row max, 64 scores at a time (the whole row would not
        // fit the register budget of 320 threads).
        float mxa = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float s[64];
          tmem_ld64(tS + 64 * hh, s);
          if (need_mask) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (col0 + 64 * hh + c >= lim_c) s[c] = -INFINITY;
          }
          float mx[4] = {fmaxf(s[0], s[4]), fmaxf(s[1], s[5]), fmaxf(s[2], s[6]), fmaxf(s[3], s[7])};
#pragma unroll
          for (int c = 8; c < 64; c += 8)
#pragma unroll
            for (int t = 0; t < 4; ++t) mx[t] = fmax3(mx[t], s[c + t], s[c + 4 + t]);
          mxa = fmax3(mxa, fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        }
        const float cand = mxa * sl2;
        const bool moved = cand > m_ref + TC_RESCALE_THRESHOLD;
        const float m_new = moved ? cand : m_ref;
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          // O is quiescent: its last P V finished before S(j) was signalled
          const float corr = moved ? ex2(m_ref - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float ov[32];
            tmem_ld32(tO + c, ov);
            uint32_t ow[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) ow[t] = __float_as_uint(ov[t] * corr);
            tmem_st32(tO + c, ow);
          }
        }
        if (moved) l *= ex2(m_ref - m_new);  // 0 when m_ref = -inf
        m_ref = m_new;
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-mu, -mu);
        uint64_t acc2[2] = {0ull, 0ull};
        // Pass 2, per half (keys 0-63, then 64-127): the scores again, the
        // exps, P to packed columns [32 hh, 32 hh + 32) (S columns this thread
        // has read), hand-over.  A 16-key group masked for every row of the
        // warp is written as zeros without exps.
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float s[64];
          tmem_ld64(tS + 64 * hh, s);
          auto group16 = [&](int g, auto use_poly) {
            uint32_t pk[8];
            const int k0 = col0 + 64 * hh + 16 * g;
            if (need_mask && __all_sync(0xffffffffu, k0 >= lim_c)) {
#pragma unroll
              for (int t = 0; t < 8; ++t) pk[t] = 0u;
            } else {
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                float v0 = s[16 * g + 2 * t], v1 = s[16 * g + 2 * t + 1];
                if (need_mask) {
                  if (k0 + 2 * t >= lim_c) v0 = -INFINITY;
                  if (k0 + 2 * t + 1 >= lim_c) v1 = -INFINITY;
                }
                const uint64_t x2 = f2_fma(f2_pack(v0, v1), scale2, negm2);
                float p0, p1;
                if (decltype(use_poly)::value && T2_POLY_EVERY > 0 && (t % T2_POLY_MOD) == T2_POLY_MOD - 1) {
                  exp2_poly_x2(x2, p0, p1);
                } else {
                  float x0, x1;
                  f2_unpack(x2, x0, x1);
                  p0 = ex2(x0);
                  p1 = ex2(x1);
                }
                acc2[t & 1] = f2_add(acc2[t & 1], f2_pack(p0, p1));
                pk[t] = sh_pack2<T>(p0, p1);
              }
            }
            tmem_st8(tS + 32 * hh + 8 * g, pk);
          };
          if (need_mask) {
#pragma unroll
            for (int g = 0; g < 4; ++g) group16(g, std::false_type{});
          } else {
#pragma unroll
            for (int g = 0; g < 4; ++g) group16(g, std::true_type{});
          }
          tmem_wait_st();
          tc_fence_before();
          if (p.fault_mode != 1) mbar_arrive_warp(bar((hh == 0 ? B_PA : B_PB) + tile));
        }
        {
          float a0, a1;
          f2_unpack(f2_add(acc2[0], acc2[1]), a0, a1);
          l += a0 + a1;
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL + tile), o_phase, wctx));
      if (!ok) break;
      o_phase ^= 1;
      tc_fence_after();
      const float inv_l = 1.f / l;
      // This row of O as 16-bit pairs: 16-byte chunk k = pk[4k .. 4k+3].
      constexpr int NC = D / 8;  // chunks per row: 16 (d = 128) or 8 (d = 64)
      uint32_t pk[D / 2];
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld32(tO + c, ov);
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[c / 2 + t] = sh_pack2<T>(ov[2 * t] * inv_l, ov[2 * t + 1] * inv_l);
      }
      // Transpose the chunks within groups of NC lanes (XOR butterfly of
      // shuffles): lane i of a group then holds chunk i of each of the group's
      // NC rows, so that one store instruction writes whole row segments.
      auto stage = [&](auto DDc) {
        constexpr int dd = decltype(DDc)::value;
        const bool up = (lane & dd) != 0;
#pragma unroll
        for (int k = 0; k < NC; ++k) {
          if (k & dd) continue;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t send = up ? pk[4 * k + m] : pk[4 * (k ^ dd) + m];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, dd);
            if (up)
              pk[4 * k + m] = recv;
            else
              pk[4 * (k ^ dd) + m] = recv;
          }
        }
      };
      if constexpr (NC == 16) stage(std::integral_constant<int, 8>{});
      stage(std::integral_constant<int, 4>{});
      stage(std::integral_constant<int, 2>{});
      stage(std::integral_constant<int, 1>{});
      {
        const int ci = lane % NC;                                          // chunk this lane stores
        const int rbase = qt * 128 + (warp & 3) * 32 + (lane / NC) * NC;   // first row of its group
        const long long rstride = p.bsnd ? (long long)p.H * D : (long long)D;
        T* obase = reinterpret_cast<T*>(p.o) +
                   (p.bsnd ? ((long long)w.b * p.Nq * p.H + w.h) * D : ((long long)w.b * p.H + w.h) * p.Nq * D) +
                   8 * ci;
#ifdef FA_CHECKS
        const long long o_total = (long long)p.B * p.H * p.Nq * D;
        const long long o_off = obase - reinterpret_cast<T*>(p.o);
#endif
#pragma unroll
        for (int k = 0; k < NC; ++k) {
          const int rk = rbase + k;
          if (rk < p.Nq && FA_INDEX_OK(status_word, o_off + rk * rstride >= 0 && o_off + rk * rstride + 8 <= o_total))
            *reinterpret_cast<uint4*>(obase + rk * rstride) = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (row < p.Nq && p.lse != nullptr &&
          FA_INDEX_OK(status_word, ((long long)w.b * p.H + w.h) * p.Nq + row < (long long)p.B * p.H * p.Nq))
        p.lse[((long long)w.b * p.H + w.h) * p.Nq + row] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
    }
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == T2_WARP_MMA) tmem_dealloc(tmem, 512);
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&p.sched->done, 1u) == gridDim.x - 1) {
      atomicExch(&p.sched->next, 0u);
      atomicExch(&p.sched->done, 0u);
    }
  }
}

}  // namespace fa
