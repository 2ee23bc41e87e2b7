// fa_fwd_tile1.cuh -- tensor-core attention forward with one 128-row query
// tile per work unit, bf16 or fp16 inputs, fp32 accumulation, head dim D in
// {64, 128, 256}.  It serves the two cases the two-tile kernel does not:
//
//   D = 256   (page 1, "CANN ops-transformer FlashAttentionScore", section
//             分块 Tiling 的计算骨架: head dims of 64-256; section 分块参数的
//             物理约束 works the d = 256 case): a 128 x 256 query tile and its
//             128 x 256 fp32 accumulator leave room in shared and tensor
//             memory for one query tile per CTA, not two.
//   BLOCK     block-sparse masks (page 1, section 总结: SparseFlashAttention
//             skips the key blocks a sparse mask marks as not needed): query
//             tile qt of (b, h) visits only the 128-key tiles kt with
//             block_mask[b, h, qt, kt] != 0, intersected with the causal
//             range when causal is set.
//
// Method: the same online softmax as the two-tile kernel (page 3, "ops-nn
// efficient attention for AIGC", section 2.2: unnormalised accumulator, one
// division by l at the end), in the exp2 domain with a lazily moved reference
// max (moved only when a step's max exceeds it by more than 2^8).
//
// B200 mapping:
//   work unit   one (batch, head, 128-row query tile); a persistent grid of
//               <= #SM CTAs takes units from a per-launch ticket counter, in
//               chunks of heads whose K/V fit in L2, heaviest (latest causal)
//               tiles first within a chunk.
//   warp 5      ticket claims and the unit's step list (for BLOCK: the whole
//               warp reads the mask row 32 entries at a time and packs it into
//               a bit set), handed to the other roles through a two-slot
//               shared-memory ring; lane 0 then loads Q and the K tiles (TMA).
//   warp 6      V tiles (TMA), decoupled from the K loads so that a K tile is
//               never held up behind a V tile that waits for its P V.
//   warp 4      TMEM allocator and MMA issuer (whole warp, elect.sync).  S is
//               double-buffered in TMEM: S(j+1) = Q K_(j+1)^T runs while the
//               softmax works on S(j).  Issue is event-driven: P V of the
//               oldest step whose P is written first, else the next S.
//   warps 0-3   softmax and epilogue, one query row (one TMEM lane) per
//               thread, all 128 scores of a step in registers: no exchange
//               between threads.  When a row's reference max moves (rare
//               after the first steps), the thread waits for the previous
//               step's P V to finish and rescales its row of O in TMEM.
//
//   TMEM (512 columns): S0 [0, 128), S1 [128, 256), O [256, 256 + D).  P of a
//   step (16-bit pairs) overwrites the first 64 columns of its S buffer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "tc_common.cuh"
#include "fa_fwd_tc.cuh"     // SchedSlot
#include "ptx.cuh"

namespace fa {

constexpr int T1_WARP_MMA = 4;
constexpr int T1_WARP_SCHED = 5;  // ticket claims, step lists, Q and K loads
constexpr int T1_WARP_V = 6;
constexpr int T1_THREADS = 32 * 7;
constexpr int T1_MAX_WORDS = 128;  // BLOCK: bit-set words per unit, i.e. at most 4096 key tiles (Nkv <= 524288)
constexpr float T1_RESCALE_THRESHOLD = 8.0f;  // log2 units
// d = 256: one exp pair in 4 on the FMA pipe on steps without masked scores
// (measured 1250 against 1178 TFLOP/s on the 8K d = 256 workload); the
// block-sparse d <= 128 instantiations measured slightly slower with it.
// FA_T1_POLY_EVERY overrides the choice for every head dim.
#ifdef FA_T1_POLY_EVERY
template <int D>
constexpr int t1_poly_every() { return FA_T1_POLY_EVERY; }
#else
template <int D>
constexpr int t1_poly_every() { return D == 256 ? 4 : 0; }
#endif

template <int D>
struct T1Cfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int CHUNKS = D / 64;
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int QST = (D == 256) ? 1 : 2;           // Q stages
  static constexpr int KST = (D == 256) ? 1 : (D == 128 ? 2 : 4);  // K and V stages each
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = QST * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
  static constexpr int OFF_RING = OFF_V + KST * TILE_BYTES;
  static constexpr int RING_INTS = 16 + T1_MAX_WORDS;       // header + bit set
  static constexpr int OFF_BAR = OFF_RING + 2 * RING_INTS * 4;
  // u_full[2] u_empty[2] q_full[QST] q_empty[QST] k_full[KST] k_empty[KST]
  // v_full[KST] v_empty[KST] s_full[2] p_full[2] pv_done[2] o_full o_free drain
  static constexpr int NBAR = 4 + 2 * QST + 4 * KST + 6 + 3;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory of sm_100");
};

struct T1Params {
  void* o;
  float* lse;
  int B, H, Nq, Nkv;
  int bsnd, causal;
  float scale_log2;
  int qtiles, kvtiles;
  int n_units;       // B * H * qtiles
  int chunk_heads;   // (batch, head) pairs per scheduling chunk
  int kv_group;      // query heads per K/V head
  // BLOCK: block_mask[b * mask_sb + h * mask_sh + qt * kvtiles + kt] != 0
  // when query tile qt sees key tile kt (strides in elements; 0 broadcasts).
  const uint8_t* block_mask;
  long long mask_sb, mask_sh;
  SchedSlot* sched;
  uint64_t timeout_ns;
  int fault_mode;
};

struct T1Unit {
  int b, h, qt;
};

// Ticket t -> (b, h, qt): chunks of chunk_heads (batch, head) pairs, the
// latest query tiles (the heaviest under a causal mask) first within a chunk.
__host__ __device__ __forceinline__ T1Unit t1_decode(int t, const T1Params& p) {
  T1Unit u;
  const int BH = p.B * p.H;
  const int per_chunk = p.chunk_heads * p.qtiles;
  const int chunk = t / per_chunk;
  const int idx = t - chunk * per_chunk;
  const int h0 = chunk * p.chunk_heads;
  const int g = (BH - h0 < p.chunk_heads) ? (BH - h0) : p.chunk_heads;
  u.qt = p.qtiles - 1 - idx / g;
  const int bh = h0 + idx % g;
  u.b = bh / p.H;
  u.h = bh - u.b * p.H;
  return u;
}

// Key tiles query tile qt may see: all of them, or up to its last row's
// position under the causal mask.
__host__ __device__ __forceinline__ int t1_kv_limit(int qt, const T1Params& p) {
  int lim = p.Nkv;
  if (p.causal) {
    const long long e = (long long)(qt + 1) * 128;
    if (e < lim) lim = (int)e;
  }
  return (lim + 127) / 128;
}

template <int D, typename T, bool BLOCK>
__global__ void __launch_bounds__(T1_THREADS, 1)
    fa_fwd_t1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, T1Params p, unsigned int* status_word) {
  using C = T1Cfg<D>;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int QST = C::QST, KST = C::KST;
  constexpr int T1_POLY_EVERY = t1_poly_every<D>();
  constexpr int T1_POLY_MOD = T1_POLY_EVERY > 0 ? T1_POLY_EVERY : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  volatile int* ring = reinterpret_cast<volatile int*>(smem + C::OFF_RING);
  const int B_UFULL = 0, B_UEMPTY = 2, B_QFULL = 4, B_QEMPTY = 4 + QST, B_KFULL = 4 + 2 * QST,
            B_KEMPTY = B_KFULL + KST, B_VFULL = B_KFULL + 2 * KST, B_VEMPTY = B_KFULL + 3 * KST,
            B_SFULL = B_KFULL + 4 * KST, B_PFULL = B_SFULL + 2, B_PVDONE = B_SFULL + 4, B_OFULL = B_SFULL + 6,
            B_OFREE = B_OFULL + 1, B_DRAIN = B_OFULL + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_UFULL + i), 1);
      mbar_init(bar(B_UEMPTY + i), 6);  // MMA warp, 4 softmax warps, V warp
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + i), 4);
      mbar_init(bar(B_PVDONE + i), 1);
    }
    for (int s = 0; s < QST; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    mbar_init(bar(B_OFULL), 1);
    mbar_init(bar(B_OFREE), 4);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == T1_WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == T1_WARP_SCHED && lane == 0) {
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

  // Ring entry: [0] ticket (-1: no more work), [1] b, [2] h, [3] qt, [4] steps,
  // [16 ...] BLOCK bit set of the key tiles to visit.
  auto ring_get = [&](int slot, T1Unit& u, int& n) -> int {
    volatile const int* e = ring + C::RING_INTS * slot;
    u.b = e[1]; u.h = e[2]; u.qt = e[3]; n = e[4];
    return e[0];
  };
  // Step iterator: the key tile of each step of a unit, in increasing order.
  struct Steps {
    volatile const int* words;
    int w;
    uint32_t bits;
    int next_plain;
  };
  auto steps_begin = [&](int slot) {
    Steps s;
    s.words = ring + C::RING_INTS * slot + 16;
    s.w = 0;
    s.bits = BLOCK ? (uint32_t)s.words[0] : 0u;
    s.next_plain = 0;
    return s;
  };
  auto steps_next = [&](Steps& s) -> int {
    if constexpr (!BLOCK) {
      return s.next_plain++;
    } else {
      while (s.bits == 0u) s.bits = (uint32_t)s.words[++s.w];
      const int k = s.w * 32 + (__ffs(s.bits) - 1);
      s.bits &= s.bits - 1u;
      return k;
    }
  };

  if (warp == T1_WARP_SCHED) {
    // ------------------------------------------------------------ tickets, step lists, Q and K
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    int uslot = 0;
    uint32_t uphase = 0;
    int gq = 0, gk = 0;  // Q and K loads issued so far (stage and phase)
    bool ok = true;
    while (ok) {
      unsigned int t = 0;
      if (lane == 0) t = atomicAdd(&p.sched->next, 1u);
      t = __shfl_sync(0xffffffffu, t, 0);
      const int tk = (t < (unsigned int)p.n_units) ? (int)t : -1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_UEMPTY + uslot), uphase ^ 1, wctx))) break;
      volatile int* e = ring + C::RING_INTS * uslot;
      const T1Unit u = t1_decode(tk < 0 ? 0 : tk, p);
      int n = 0;
      if (tk >= 0) {
        const int lim = t1_kv_limit(u.qt, p);
        if constexpr (BLOCK) {
          const uint8_t* row = p.block_mask + (long long)u.b * p.mask_sb + (long long)u.h * p.mask_sh +
                               (long long)u.qt * p.kvtiles;
          const int nw = (lim + 31) / 32;
          for (int w = 0; w < nw; ++w) {
            const int kt = w * 32 + lane;
            const bool vis = kt < lim && row[kt] != 0;
            const uint32_t bits = __ballot_sync(0xffffffffu, vis);
            if (lane == 0) e[16 + w] = (int)bits;
            n += __popc(bits);
          }
        } else {
          n = lim;
        }
      }
      if (lane == 0) {
        e[0] = tk; e[1] = u.b; e[2] = u.h; e[3] = u.qt; e[4] = n;
        mbar_arrive(bar(B_UFULL + uslot));  // release: the entry is visible to the waiters
      }
      __syncwarp();
      const int my_slot = uslot;
      if (++uslot == 2) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      if (n == 0) continue;
      if (lane == 0) {
        const int qs = gq % QST;
        if (!mbar_wait(bar(B_QEMPTY + qs), ((gq / QST) & 1) ^ 1, wctx)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(bar(B_QFULL + qs), C::TILE_BYTES);
          const uint32_t dst = sbase + C::OFF_Q + qs * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd)
              tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + qs), c * 64, u.h, u.qt * 128, u.b, pol_q);
            else
              tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + qs), c * 64, u.qt * 128, u.h, u.b, pol_q);
          }
          ++gq;
          const int hk = u.h / p.kv_group;
          Steps st = steps_begin(my_slot);
          for (int j = 0; j < n; ++j) {
            const int kt = steps_next(st);
            const int ks = gk % KST;
            if (!mbar_wait(bar(B_KEMPTY + ks), ((gk / KST) & 1) ^ 1, wctx)) { ok = false; break; }
            mbar_arrive_expect_tx(bar(B_KFULL + ks), C::TILE_BYTES);
            const uint32_t kd = sbase + C::OFF_K + ks * C::TILE_BYTES;
            for (int c = 0; c < C::CHUNKS; ++c) {
              if (p.bsnd)
                tma_load_4d(kd + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + ks), c * 64, hk, kt * 128, u.b, pol_kv);
              else
                tma_load_4d(kd + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + ks), c * 64, kt * 128, hk, u.b, pol_kv);
            }
            ++gk;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      // Every copy this thread started lands before the CTA may exit.
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      for (int i = 1; i <= QST && gq - i >= 0; ++i) {
        const int g = gq - i;
        mbar_wait(bar(B_QFULL + g % QST), (g / QST) & 1, drain);
      }
      for (int i = 1; i <= KST && gk - i >= 0; ++i) {
        const int g = gk - i;
        mbar_wait(bar(B_KFULL + g % KST), (g / KST) & 1, drain);
      }
    }
    __syncwarp();
  } else if (warp == T1_WARP_V) {
    // ------------------------------------------------------------ V loads
    const uint64_t pol_kv = l2_policy_evict_last();
    int uslot = 0;
    uint32_t uphase = 0;
    int gv = 0;
    bool ok = true;
    while (ok) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_UFULL + uslot), uphase, wctx))) break;
      T1Unit u;
      int n = 0;
      const int tk = ring_get(uslot, u, n);
      Steps st = steps_begin(uslot);
      // the step list is read while this warp still holds the slot
      if (lane == 0 && tk >= 0) {
        const int hk = u.h / p.kv_group;
        for (int j = 0; j < n; ++j) {
          const int kt = steps_next(st);
          const int vs = gv % KST;
          if (!mbar_wait(bar(B_VEMPTY + vs), ((gv / KST) & 1) ^ 1, wctx)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(B_VFULL + vs), C::TILE_BYTES);
          const uint32_t vd = sbase + C::OFF_V + vs * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c) {
            if (p.bsnd)
              tma_load_4d(vd + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + vs), c * 64, hk, kt * 128, u.b, pol_kv);
            else
              tma_load_4d(vd + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + vs), c * 64, kt * 128, hk, u.b, pol_kv);
          }
          ++gv;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == 2) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
    }
    if (lane == 0) {
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      for (int i = 1; i <= KST && gv - i >= 0; ++i) {
        const int g = gv - i;
        mbar_wait(bar(B_VFULL + g % KST), (g / KST) & 1, drain);
      }
    }
    __syncwarp();
  } else if (warp == T1_WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_S = idesc_f16(IS_BF16, false, 128, 128);
    constexpr uint32_t IDESC_PV = idesc_f16(IS_BF16, true, 128, D);
    const uint64_t dQ0 = smem_desc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dK0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
    const uint32_t tO = tmem + 256;
    auto ready = [&](int b, uint32_t ph) { return __all_sync(0xffffffffu, mbar_poll(bar(b), ph)); };
    int uslot = 0;
    uint32_t uphase = 0;
    int gs = 0, gp = 0, gq = 0;  // S steps, P V steps and query tiles so far (all units)
    int uw = 0;                  // units with at least one step so far
    bool ok = true;
    while (ok) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_UFULL + uslot), uphase, wctx))) break;
      T1Unit u;
      int n = 0;
      const int tk = ring_get(uslot, u, n);
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == 2) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      if (n == 0) continue;
      const int qs = gq % QST;
      if (!__all_sync(0xffffffffu, mbar_wait(bar(B_QFULL + qs), (gq / QST) & 1, wctx))) { ok = false; break; }
      const uint64_t dQ = dQ0 + (uint64_t)((qs * C::TILE_BYTES) >> 4);
      int js = 0, jp = 0;
      uint64_t idle_since = 0;
      while (jp < n) {
        bool did = false;
        // P V of step jp: its P is written, its V has landed and, on the
        // unit's first step, the previous unit's O has been read out.
        if (jp < js && ready(B_PFULL + (gp & 1), (gp >> 1) & 1) &&
            ready(B_VFULL + gp % KST, (gp / KST) & 1) && (jp > 0 || uw == 0 || ready(B_OFREE, (uw - 1) & 1))) {
          tc_fence_after();
          const uint32_t tS = tmem + 128 * (gp & 1);
          const uint64_t dV = dV0 + (uint64_t)(((gp % KST) * C::TILE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            sh_mma_ts(tO, tS + 8 * kk, dV + (uint64_t)((kk * 2048) >> 4), IDESC_PV, (jp > 0 || kk > 0) ? 1u : 0u);
          mma_commit_elect(bar(B_PVDONE + (gp & 1)));
          mma_commit_elect(bar(B_VEMPTY + gp % KST));
          if (jp == n - 1) mma_commit_elect(bar(B_OFULL));
          ++jp;
          ++gp;
          did = true;
        } else if (js < n && js < jp + 2 && ready(B_KFULL + gs % KST, (gs / KST) & 1)) {
          // S of step js into buffer gs & 1 (free: P V of step js - 2 was issued)
          tc_fence_after();
          const uint32_t tS = tmem + 128 * (gs & 1);
          const uint64_t dK = dK0 + (uint64_t)(((gs % KST) * C::TILE_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = (uint64_t)(((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4);
            sh_mma_ss(tS, dQ + o, dK + o, IDESC_S, kk > 0 ? 1u : 0u);
          }
          mma_commit_elect(bar(B_SFULL + (gs & 1)));
          mma_commit_elect(bar(B_KEMPTY + gs % KST));
          if (js == n - 1) mma_commit_elect(bar(B_QEMPTY + qs));
          ++js;
          ++gs;
          did = true;
        }
        if (did) {
          idle_since = 0;
          continue;
        }
        poll_backoff();  // nothing was ready
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
      ++gq;
      ++uw;
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
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int r = warp * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tO = tmem + lane_base + 256;
    const float sl2 = p.scale_log2;
    int uslot = 0;
    uint32_t uphase = 0;
    int g = 0;   // steps so far (all units): S buffer and barrier phases
    int uw = 0;  // units with at least one step so far
    bool ok = true;
    while (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_UFULL + uslot), uphase, wctx));
      if (!ok) break;
      T1Unit u;
      int n = 0;
      const int tk = ring_get(uslot, u, n);
      Steps st = steps_begin(uslot);
      if (tk < 0) {
        mbar_arrive_warp(bar(B_UEMPTY + uslot));
        break;
      }
      // the key tiles of the unit's steps (read before the slot is released)
      const int row = u.qt * 128 + r;
      const bool valid = row < p.Nq;
      const long long orow = p.bsnd ? (((long long)u.b * p.Nq + row) * p.H + u.h) * D
                                    : (((long long)u.b * p.H + u.h) * p.Nq + row) * D;
      T* optr = reinterpret_cast<T*>(p.o) + orow;
      const long long lidx = ((long long)u.b * p.H + u.h) * p.Nq + row;
      if (n == 0) {
        // BLOCK: no key tile visible to this query tile: O = 0, LSE = -inf
        mbar_arrive_warp(bar(B_UEMPTY + uslot));
        if (++uslot == 2) { uslot = 0; uphase ^= 1; }
        if (valid && FA_INDEX_OK(status_word, lidx < (long long)p.B * p.H * p.Nq)) {
#pragma unroll
          for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(optr + c) = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse != nullptr) p.lse[lidx] = -INFINITY;
        }
        continue;
      }
      float m_ref = -INFINITY;  // reference max (log2 domain)
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int kt = steps_next(st);
        if (j == n - 1) {  // every step's key tile is known: release the slot
          mbar_arrive_warp(bar(B_UEMPTY + uslot));
          if (++uslot == 2) { uslot = 0; uphase ^= 1; }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + (g & 1)), (g >> 1) & 1, wctx));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + lane_base + 128 * (g & 1);
        float sc[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<float(*)[32]>(sc + 32 * c));
        const int col0 = kt * 128;
        int lim = p.causal ? (row + 1 < p.Nkv ? row + 1 : p.Nkv) : p.Nkv;
        const bool masked = __any_sync(0xffffffffu, col0 + 127 >= lim);
        if (masked) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (col0 + c >= lim) sc[c] = -INFINITY;
        }
        float mx[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
        for (int c = 4; c < 128; c += 8)
#pragma unroll
          for (int t = 0; t < 4; ++t) mx[t] = fmax3(mx[t], sc[c + t], c + 4 + t < 128 ? sc[c + 4 + t] : sc[c + t]);
        const float cand = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2;
        const bool moved = cand > m_ref + T1_RESCALE_THRESHOLD;
        const float m_new = moved ? cand : m_ref;
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          // O is rescaled in place once the previous step's P V has finished
          ok = __all_sync(0xffffffffu, mbar_wait(bar(B_PVDONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, wctx));
          if (!ok) break;
          tc_fence_after();
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
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        const uint64_t scale2 = f2_pack(sl2, sl2), negm2 = f2_pack(-mu, -mu);
        uint64_t acc2[2] = {0ull, 0ull};
        // With T1_POLY_EVERY > 0, on steps without masked scores one exp pair
        // in T1_POLY_EVERY is computed on the FMA pipe (exp2_poly_x2: masked
        // scores of -inf must not reach it).
        auto exps = [&](auto use_poly) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const uint64_t x2 = f2_fma(f2_pack(sc[32 * c + 2 * t], sc[32 * c + 2 * t + 1]), scale2, negm2);
              float p0, p1;
              if (decltype(use_poly)::value && (t % T1_POLY_MOD) == T1_POLY_MOD - 1) {
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
            sh_tmem_st16(tS + 16 * c, pk);
          }
        };
        if (T1_POLY_EVERY > 0 && !masked)
          exps(std::integral_constant<bool, (T1_POLY_EVERY > 0)>{});
        else
          exps(std::false_type{});
        {
          float a0, a1;
          f2_unpack(f2_add(acc2[0], acc2[1]), a0, a1);
          l += a0 + a1;
        }
        m_ref = m_new;
        tmem_wait_st();
        tc_fence_before();
        if (p.fault_mode != 1) mbar_arrive_warp(bar(B_PFULL + (g & 1)));
        ++g;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL), uw & 1, wctx));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = valid && FA_INDEX_OK(status_word, lidx < (long long)p.B * p.H * p.Nq);
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld32(tO + c, ov);
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[t] = sh_pack2<T>(ov[2 * t] * inv_l, ov[2 * t + 1] * inv_l);
        if (store) {
#pragma unroll
          for (int t = 0; t < 4; ++t)
            *reinterpret_cast<uint4*>(optr + c + 8 * t) = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive_warp(bar(B_OFREE));  // O may take the next unit's first P V
      if (store && p.lse != nullptr) p.lse[lidx] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
      ++uw;
    }
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == T1_WARP_MMA) tmem_dealloc(tmem, 512);
  if (threadIdx.x == 0) {
    // The last CTA out returns this launch's ticket counter to zero.
    __threadfence();
    if (atomicAdd(&p.sched->done, 1u) == gridDim.x - 1) {
      atomicExch(&p.sched->next, 0u);
      atomicExch(&p.sched->done, 0u);
    }
  }
}

}  // namespace fa
