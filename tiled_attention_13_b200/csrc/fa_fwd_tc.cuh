// fa_fwd_tc.cuh -- tensor-core (tcgen05 + TMEM + TMA) attention forward for
// sm_100a, bf16 or fp16 inputs, fp32 accumulation, head dim D in {64, 128}.
//
// Method (page 1, "CANN ops-transformer FlashAttentionScore", section 分块
// Tiling 的计算骨架: every Q tile walks all of its K/V tiles and merges them
// with the online softmax; page 3, "ops-nn efficient attention for AIGC",
// section 2.2: unnormalised accumulator o = o * corr + exp(S - m_new) V,
// divided by l once at the end; section 3.2: causal block skip).
//
// B200 mapping (the pages' Cube/Vector/UB design is prior art only):
//
//   work unit   one (batch, head, pair of 128-row Q tiles); a persistent grid
//               of <= #SM CTAs takes units from a per-launch ticket counter
//               (atomicAdd), in chunks of heads whose K/V fit in L2 and,
//               within a chunk, heaviest causal pairs first.
//   warps 0-15  four softmax warpgroups: (tile 0, keys 0-63), (tile 0, keys
//               64-127), (tile 1, keys 0-63), (tile 1, keys 64-127).  A thread
//               owns one query row (= one TMEM lane) and half of its 128 scores
//               per KV tile; the two halves of a row agree on the reference max
//               through shared memory (lazily, see below).  Each warpgroup also
//               writes its half of O (chunks transposed across lanes by
//               shuffles, so that stores cover whole row segments).
//   warp 16     TMEM allocator and the MMA issuer (whole warp, elect.sync)
//   warp 17     ticket claims and unit decode (handed to the other roles through
//               a shared-memory ring), TMA producer (Q tiles, K/V ring of KST
//               stages)
//
//   TMEM (512 columns x 128 lanes, fp32):  S0 [0,128)  S1 [128,256)
//   O0 [256, 256+D)  O1 [256+D, 256+2D).  P_i (bf16/fp16 pairs) for keys
//   0-63 overwrites S_i columns [0,32), for keys 64-127 columns [64,96): each
//   half writes only columns it has already read.
//
//   MMA order per KV step j (tile i = 0, 1):  O_i += P_i(j-1) V_(j-1) in two
//   parts as the softmax hands them over (keys 0-31 of each half, then keys
//   32-63), then S_i(j) = Q_i K_j^T, then commit -> s_full[i].  The tensor
//   pipe executes a CTA's MMAs in issue order, so S_i(j) overwrites P_i(j-1)
//   only after the P V product has read it, and when s_full[i] fires O_i is
//   quiescent (the softmax may rescale it in place).
//
//   The two tiles run half a step apart (the MMA issue order staggers them):
//   one tile's exps, on two warps per SM sub-partition, overlap the other
//   tile's MMAs.  Built with FA_POLY_EVERY=n > 0, one exp pair in n of the
//   tiles without masked scores is computed on the FMA pipe instead of the
//   SFU (off by default: with the scores held in registers it measured
//   slower than SFU-only exps).
//
//   Online softmax in the exp2 domain: x = s * scale * log2(e).  The running
//   reference max m is only moved when a tile's max exceeds it by more than
//   2^8 (then O and l are rescaled by 2^(m_old - m_new)); otherwise P may
//   reach 2^8, which bf16/fp16 and the fp32 sums hold exactly as well.  The
//   final O = o / l and LSE = (m + log2 l) ln 2 are the same numbers either
//   way: the reference max cancels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "ptx.cuh"

namespace fa {

// Optional timeline instrumentation (compile with -DFA_TRACE): SM-clock
// stamps of each role's phases for the first work unit of CTA 0, readable
// through fa_debug_trace_read().  Compiles to nothing otherwise.
#ifdef FA_TRACE
// [stream][j][event]: streams 0-15 = softmax warps, 16-17 = MMA for tile 0/1
constexpr int TRACE_J = 64, TRACE_EV = 8, TRACE_STREAMS = 18;
__device__ unsigned long long g_trace[TRACE_STREAMS * TRACE_J * TRACE_EV];
#define FA_TR(cond, stream, j, ev)                                                           \
  do {                                                                                       \
    if ((cond) && blockIdx.x == 0 && (j) < TRACE_J)                                          \
      g_trace[((stream) * TRACE_J + (j)) * TRACE_EV + (ev)] = (unsigned long long)clock64(); \
  } while (0)
#else
#define FA_TR(cond, tile, j, ev) \
  do {                           \
  } while (0)
#endif
// Unit-indexed variant (compile with -DFA_TRACE_UNITS): one row per work unit
// of CTA 0, events per role.  Streams: 0 producer, 1 MMA, 2 softmax warp 0.
#ifdef FA_TRACE_UNITS
constexpr int TRU_N = 64, TRU_EV = 8;
__device__ unsigned long long g_trace_units[3 * TRU_N * TRU_EV];
#define FA_TRU(cond, stream, k, ev)                                                               \
  do {                                                                                            \
    if ((cond) && blockIdx.x == 0 && (k) < TRU_N)                                                 \
      g_trace_units[((stream) * TRU_N + (k)) * TRU_EV + (ev)] = (unsigned long long)clock64();   \
  } while (0)
#else
#define FA_TRU(cond, stream, k, ev) \
  do {                              \
  } while (0)
#endif

constexpr int TC_SOFTMAX_WARPS = 16;
constexpr int WARP_MMA = 16;
constexpr int WARP_TMA = 17;
constexpr int TC_THREADS = 32 * 18;
constexpr int TC_BM = 128;                    // query rows per Q tile
constexpr int TC_BN = 128;                    // keys per KV tile
constexpr float TC_RESCALE_THRESHOLD = 8.0f;  // log2 units
#ifndef FA_POLY_EVERY
#define FA_POLY_EVERY 0
#endif
constexpr int TC_POLY_EVERY = FA_POLY_EVERY;  // > 0: one exp pair in TC_POLY_EVERY on the FMA pipe
constexpr int TC_POLY_MOD = TC_POLY_EVERY > 0 ? TC_POLY_EVERY : 1;


template <int D>
struct TcCfg {
  static constexpr int TILE_BYTES = TC_BM * D * 2;          // one 128 x D tile of 16-bit values
  static constexpr int CHUNKS = D / 64;                     // 128-byte-wide column chunks per tile
  static constexpr int CHUNK_BYTES = TC_BM * 128;           // 128 rows x 128 bytes
  static constexpr int KST = (D == 128) ? 2 : 4;            // K/V ring depth
  static constexpr int OFF_Q = 0;                           // Q0, Q1
  static constexpr int OFF_K = 2 * TILE_BYTES;              // KST K tiles
  static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;    // KST V tiles
  static constexpr int OFF_RED = OFF_V + KST * TILE_BYTES;  // [tile][parity][half][row] fp32 exchange
  static constexpr int RED_BYTES = 2 * 2 * 2 * TC_BM * 4;
  static constexpr int OFF_UNIT = OFF_RED + RED_BYTES;      // ring of decoded work units (16 ints each)
  static constexpr int UNIT_SLOTS = 4;
  static constexpr int OFF_BAR = OFF_UNIT + 64 * UNIT_SLOTS;  // barriers
  static constexpr int NBAR = 2 + 2 + 4 * KST + 2 + 4 + 2 + 1 + 2 + 2 * UNIT_SLOTS;
  static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 /*tmem slot + abort*/ + 1024 /*align slack*/;
  static constexpr int TMEM_S0 = 0, TMEM_S1 = 128, TMEM_O0 = 256, TMEM_O1 = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
};

// Work-ticket counter of one launch.  `next` hands out tickets; the last CTA
// to finish (counted by `done`) puts both back to zero for the launch that
// reuses the slot.
struct SchedSlot {
  unsigned int next;
  unsigned int done;
};

struct TcParams {
  // O and LSE; under split-KV (the kernel's SPLIT instantiation) the fp32
  // per-slice results instead: o -> o_part [n_splits, B, H, Nq, D] and
  // lse -> lse_part [n_splits, B, H, Nq], each slice's rows normalised over
  // that slice alone, combined afterwards by the merge kernel.
  void* o;
  float* lse;
  int B, H, Nq, Nkv;
  int bsnd;          // 1: [B, N, H, D] rows, 0: [B, H, N, D]
  int causal;
  float scale_log2;  // softmax scale * log2(e)
  int n_pairs;       // ceil(ceil(Nq / 128) / 2)
  int n_units;       // B * H * n_pairs
  int chunk_heads;   // (batch, head) pairs per scheduling chunk (L2 working set)
  int kv_group;      // query heads per K/V head: query head h reads K/V head h / kv_group
  // Paged K/V (the kernel's PAGED instantiation): the K and V tensor maps cover caches of
  // [num_blocks, block_size, Hkv, d]; key n of batch entry b lives in
  // physical block block_table[b * max_blocks + n / block_size], row
  // n % block_size.  block_size is a power of two >= 16.
  const int* block_table;
  int block_size, max_blocks, num_blocks;
  // The one mode-specific pair of ints (the parameter block keeps its size:
  // a larger one changed the register allocation of every instantiation).
  //   band (BAND): key j is visible to query row i iff
  //     i - pre_tokens <= j <= i + next_tokens (and j < Nkv);
  //   split (SPLIT): the KV tiles are cut into n_splits slices of
  //     split_tiles tiles (the last may be shorter, none is empty), one unit
  //     per (batch, head, Q-tile pair, slice).
  union {
    struct {
      int pre_tokens, next_tokens;
    } band;
    struct {
      int n_splits, split_tiles;
    } split;
  };
  SchedSlot* sched;  // this launch's work-ticket counter
  uint64_t timeout_ns;
  int fault_mode;
};

// Per-unit geometry shared by every role (pure integer arithmetic; the
// decode functions below also compile for the host, where a test checks the
// schedule's coverage).
struct Unit {
  int b, h, qt0;      // qt0 = first Q tile index (even), second = qt0 + 1
  int active1;        // second Q tile has at least one valid row
  int n0, n1;         // KV tiles for tile 0 / tile 1 (0 if inactive)
  int lo0, s1;        // band / split: first KV tile of tile 0; tile 1 starts s1 tiles later (else 0, 0)
};

__host__ __device__ __forceinline__ int kv_tiles_for(int qt, int Nkv, int causal) {
  int lim = Nkv;
  if (causal) {
    long long e = (long long)(qt + 1) * TC_BM;
    if (e < lim) lim = (int)e;
  }
  return (lim + TC_BN - 1) / TC_BN;
}

// Ticket t -> unit.  Tickets walk the (batch, head) pairs in chunks of
// chunk_heads, so the K/V of the heads in flight stay in L2; inside a chunk
// the heaviest causal Q-tile pairs come first (longest-processing-time order)
// and the heads of one pair are adjacent.
__host__ __device__ __forceinline__ Unit decode_unit(int t, const TcParams& p) {
  Unit w;
  const int BH = p.B * p.H;
  const int per_chunk = p.chunk_heads * p.n_pairs;  // <= n_units < 2^31
  const int chunk = t / per_chunk;
  const int idx = t - chunk * per_chunk;
  const int h0 = chunk * p.chunk_heads;
  const int g = (BH - h0 < p.chunk_heads) ? (BH - h0) : p.chunk_heads;
  const int pair = p.n_pairs - 1 - idx / g;
  const int bh = h0 + idx % g;
  w.b = bh / p.H;
  w.h = bh % p.H;
  w.qt0 = 2 * pair;
  w.active1 = ((long long)(w.qt0 + 1) * TC_BM < (long long)p.Nq) ? 1 : 0;
  w.n0 = kv_tiles_for(w.qt0, p.Nkv, p.causal);
  w.n1 = w.active1 ? kv_tiles_for(w.qt0 + 1, p.Nkv, p.causal) : 0;
  return w;
}

// KV tile range [lo, hi) of Q tile qt under a band: the keys its rows can see,
// [qt*128 - pre, qt*128 + 127 + next], cut to [0, Nkv).
__host__ __device__ __forceinline__ int band_lo(int qt, const TcParams& p) {
  const long long k = (long long)qt * TC_BM - p.band.pre_tokens;
  return k <= 0 ? 0 : (int)(k / TC_BN);
}
__host__ __device__ __forceinline__ int band_hi(int qt, const TcParams& p) {
  long long k = (long long)qt * TC_BM + TC_BM + p.band.next_tokens;  // one past the last visible key
  if (k > p.Nkv) k = p.Nkv;
  return (int)((k + TC_BN - 1) / TC_BN);
}

// Split-KV ticket t -> unit and its slice index sp.  The (batch, head)
// chunks are walked as in decode_unit; a head's units are its (Q-tile pair,
// slice) pairs, the slice index fastest.  Both Q tiles of a pair take the
// same slice of KV tiles (no mask but the sequence end).
__host__ __device__ __forceinline__ Unit decode_unit_split(int t, const TcParams& p, int& sp) {
  Unit w;
  const int BH = p.B * p.H;
  const int per_chunk = p.chunk_heads * p.n_pairs * p.split.n_splits;  // <= n_units < 2^31
  const int chunk = t / per_chunk;
  const int idx = t - chunk * per_chunk;
  const int h0 = chunk * p.chunk_heads;
  const int g = (BH - h0 < p.chunk_heads) ? (BH - h0) : p.chunk_heads;
  const int ps = idx / g;
  const int bh = h0 + (idx - ps * g);
  const int pair = ps / p.split.n_splits;
  sp = ps - pair * p.split.n_splits;
  w.b = bh / p.H;
  w.h = bh % p.H;
  w.qt0 = 2 * pair;
  w.active1 = ((long long)(w.qt0 + 1) * TC_BM < (long long)p.Nq) ? 1 : 0;
  const int nt = (p.Nkv + TC_BN - 1) / TC_BN;
  w.lo0 = sp * p.split.split_tiles;
  const int n = (nt - w.lo0 < p.split.split_tiles) ? nt - w.lo0 : p.split.split_tiles;
  w.n0 = n;
  w.n1 = w.active1 ? n : 0;
  w.s1 = 0;
  return w;
}

template <bool BAND, bool SPLIT>
__host__ __device__ __forceinline__ Unit decode_unit_t(int t, const TcParams& p, int& sp) {
  if constexpr (SPLIT) return decode_unit_split(t, p, sp);
  Unit w = decode_unit(t, p);
  w.lo0 = 0;
  w.s1 = 0;
  if constexpr (BAND) {
    const int lo0 = band_lo(w.qt0, p);
    w.lo0 = lo0;
    w.n0 = band_hi(w.qt0, p) - lo0;
    if (w.active1) {
      const int lo1 = band_lo(w.qt0 + 1, p);
      w.s1 = lo1 - lo0;
      w.n1 = band_hi(w.qt0 + 1, p) - lo1;
    }
  }
  return w;
}

template <typename T>
struct Pack;
template <>
struct Pack<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t two(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
};
template <>
struct Pack<__half> {
  static __device__ __forceinline__ uint32_t two(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
};

template <int D, typename T, bool PAGED = false, bool BAND = false, bool SPLIT = false>
__global__ void __launch_bounds__(TC_THREADS, 1)
    fa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, TcParams p, unsigned int* status_word) {
  using C = TcCfg<D>;
  static_assert(!(BAND && SPLIT), "a band and split-KV are separate instantiations");
  // A band or a split walks each unit over its own range of KV tiles.
  constexpr bool WALK = BAND || SPLIT;
  constexpr bool IS_BF16 = std::is_same<T, __nv_bfloat16>::value;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment: the 128-byte swizzle pattern is anchored there.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + C::OFF_UNIT);
  // barrier indices
  const int B_QFULL = 0, B_QEMPTY = 2, B_KFULL = 4, B_KEMPTY = 4 + C::KST, B_VFULL = 4 + 2 * C::KST,
            B_VEMPTY = 4 + 3 * C::KST, B_SFULL = 4 + 4 * C::KST, B_PFULL = B_SFULL + 2, B_OFULL = B_PFULL + 4,
            B_DRAIN = B_OFULL + 2, B_XCHG = B_DRAIN + 1, B_UFULL = B_XCHG + 2,
            B_UEMPTY = B_UFULL + C::UNIT_SLOTS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  // Unit ring slot: ticket (-1 = no more work) and the decoded unit.
  // A split's slice index rides in e[9], outside Unit.
  auto ring_put = [&](int slot, int tk, const Unit& w, int sp) {
    volatile int* e = unit_ring + 16 * slot;
    e[0] = tk; e[1] = w.b; e[2] = w.h; e[3] = w.qt0; e[4] = w.active1; e[5] = w.n0; e[6] = w.n1;
    e[7] = w.lo0; e[8] = w.s1;
    if constexpr (SPLIT) e[9] = sp;
  };
  auto ring_get = [&](int slot, Unit& w) -> int {
    volatile const int* e = unit_ring + 16 * slot;
    w.b = e[1]; w.h = e[2]; w.qt0 = e[3]; w.active1 = e[4]; w.n0 = e[5]; w.n1 = e[6];
    w.lo0 = WALK ? e[7] : 0;
    w.s1 = WALK ? e[8] : 0;
    return e[0];
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_QFULL + i), 1);
      mbar_init(bar(B_QEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + 2 * i), 8);      // P keys 0-31 and 64-95: one arrival per warp of the tile
      mbar_init(bar(B_PFULL + 2 * i + 1), 8);  // P keys 32-63 and 96-127
      mbar_init(bar(B_OFULL + i), 1);
      mbar_init(bar(B_XCHG + i), 8);
    }
    for (int s = 0; s < C::KST; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    for (int i = 0; i < C::UNIT_SLOTS; ++i) {
      mbar_init(bar(B_UFULL + i), 1);
      mbar_init(bar(B_UEMPTY + i), 1 + TC_SOFTMAX_WARPS);  // MMA warp + softmax warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == WARP_TMA && lane == 0) {
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

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    // Lane 0 claims the tickets, keeps the unit ring and the barriers, and
    // issues every Q copy and a contiguous K/V tile's copies.  A paged K/V
    // tile takes up to TC_BN / 16 sub-boxes, one per cache block: there the
    // whole warp runs the loop (warp-uniform control flow) and lane u reads
    // sub-box u's table entry and issues its copies, so that the table reads
    // overlap and the copies go out in parallel rather than one by one.
    const unsigned pmask = PAGED ? 0xffffffffu : 1u;  // the lanes that run the loop
    if (PAGED || lane == 0) {
      const bool lead = PAGED ? lane == 0 : true;  // a compile-time true for contiguous K/V
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t q_phase[2] = {0, 0};
      int st = 0;
      uint32_t kv_phase = 0;
      // outstanding-load bookkeeping for the drain at exit (every lane keeps
      // the same copy)
      uint32_t k_issued[C::KST], v_issued[C::KST], q_issued[2];
      bool k_pend[C::KST], v_pend[C::KST], q_pend[2];
      for (int s = 0; s < C::KST; ++s) { k_pend[s] = v_pend[s] = false; k_issued[s] = v_issued[s] = 0; }
      q_pend[0] = q_pend[1] = false; q_issued[0] = q_issued[1] = 0;
      bool ok = true;
      int uslot = 0;
      uint32_t uphase = 0;
      int n_claimed = 0;
      (void)n_claimed;
      auto wait_p = [&](uint32_t bb, uint32_t ph) {
        if constexpr (PAGED)
          return __all_sync(pmask, mbar_wait(bb, ph, wctx));
        else
          return mbar_wait(bb, ph, wctx);
      };
      // One 128-key K or V tile from a paged cache: TC_BN / pbox sub-boxes of
      // pbox = min(block size, 128) rows, sub-box u from physical block
      // phys_u of lane u.  Blocks past the sequence read at block index
      // num_blocks, outside the tensor map, which the copy fills with zeros.
      constexpr int PSUB = TC_BN / 16;  // sub-boxes per tile at the smallest block size
      const int pbox = PAGED ? (p.block_size < TC_BN ? p.block_size : TC_BN) : TC_BN;
      const int pvalid = PAGED ? (p.Nkv + p.block_size - 1) / p.block_size : 0;
      const bool sub_lane = lane < PSUB && lane * pbox < TC_BN;  // this lane owns sub-box `lane`
      int phys_u = 0;
      // the tile's table entry of this lane's sub-box, used for both K and V
      auto paged_lookup = [&](int kv0, int b) {
        int ph = p.num_blocks;
        if (sub_lane) {
          const int lb = (kv0 + lane * pbox) / p.block_size;
          if (lb < pvalid && FA_INDEX_OK(status_word, lb < p.max_blocks && b < p.B))
            ph = p.block_table[(long long)b * p.max_blocks + lb];
        }
        phys_u = ph;
      };
      auto paged_load = [&](uint32_t dst, const CUtensorMap* tm, uint32_t b_full, int kv0, int hk, uint64_t pol) {
        if (sub_lane) {
          const int off = (kv0 + lane * pbox) % p.block_size;
          for (int c = 0; c < C::CHUNKS; ++c)
            tma_load_4d(dst + c * C::CHUNK_BYTES + lane * pbox * 128, tm, b_full, c * 64, hk, off, phys_u, pol);
        }
      };
      while (ok) {
        // claim the next ticket and hand it to the other roles
        // (decoded here once: its integer divisions stay off the other roles)
        unsigned int t = 0;
        if (lead) t = atomicAdd(&p.sched->next, 1u);
        if constexpr (PAGED) t = __shfl_sync(pmask, t, 0);
        const int tk = (t < (unsigned int)p.n_units) ? (int)t : -1;
        int sp = 0;
        const Unit w = decode_unit_t<BAND, SPLIT>(tk < 0 ? 0 : tk, p, sp);
        if (!wait_p(bar(B_UEMPTY + uslot), uphase ^ 1)) break;
        if (lead) {
          ring_put(uslot, tk, w, sp);
          mbar_arrive(bar(B_UFULL + uslot));
        }
        if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
        if (tk < 0) break;
        FA_TRU(lead, 0, n_claimed, 0);
        for (int i = 0; i < 2 && ok; ++i) {
          if (i == 1 && !w.active1) break;
          if (!wait_p(bar(B_QEMPTY + i), q_phase[i] ^ 1)) { ok = false; break; }
          if (lead) {
            const uint32_t dst = sbase + C::OFF_Q + i * C::TILE_BYTES;
            mbar_arrive_expect_tx(bar(B_QFULL + i), C::TILE_BYTES);
            const int row0 = (w.qt0 + i) * TC_BM;
            for (int c = 0; c < C::CHUNKS; ++c) {
              if (p.bsnd)
                tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + i), c * 64, w.h, row0, w.b, pol_q);
              else
                tma_load_4d(dst + c * C::CHUNK_BYTES, &tm_q, bar(B_QFULL + i), c * 64, row0, w.h, w.b, pol_q);
            }
          }
          q_pend[i] = true; q_issued[i] = q_phase[i];
          q_phase[i] ^= 1;
        }
        FA_TRU(lead, 0, n_claimed, 1);
        const int N = w.n0 > w.s1 + w.n1 ? w.n0 : w.s1 + w.n1;  // KV tiles lo0 .. lo0 + N - 1
        const int hk = w.h / p.kv_group;  // this unit's K/V head
        for (int j = 0; j < N && ok; ++j) {
          const int kv0 = (w.lo0 + j) * TC_BN;
          if constexpr (PAGED) paged_lookup(kv0, w.b);  // before the wait: the read overlaps it
          if (!wait_p(bar(B_KEMPTY + st), kv_phase ^ 1)) { ok = false; break; }
          if (lead) mbar_arrive_expect_tx(bar(B_KFULL + st), C::TILE_BYTES);
          const uint32_t kdst = sbase + C::OFF_K + st * C::TILE_BYTES;
          if constexpr (PAGED) {
            __syncwarp();  // lane 0's expected byte count is set before any lane's copy
            paged_load(kdst, &tm_k, bar(B_KFULL + st), kv0, hk, pol_kv);
          } else {
            for (int c = 0; c < C::CHUNKS; ++c) {
              if (p.bsnd)
                tma_load_4d(kdst + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + st), c * 64, hk, kv0, w.b, pol_kv);
              else
                tma_load_4d(kdst + c * C::CHUNK_BYTES, &tm_k, bar(B_KFULL + st), c * 64, kv0, hk, w.b, pol_kv);
            }
          }
          k_pend[st] = true; k_issued[st] = kv_phase;
          if (!wait_p(bar(B_VEMPTY + st), kv_phase ^ 1)) { ok = false; break; }
          if (lead) mbar_arrive_expect_tx(bar(B_VFULL + st), C::TILE_BYTES);
          const uint32_t vdst = sbase + C::OFF_V + st * C::TILE_BYTES;
          if constexpr (PAGED) {
            __syncwarp();
            paged_load(vdst, &tm_v, bar(B_VFULL + st), kv0, hk, pol_kv);
          } else {
            for (int c = 0; c < C::CHUNKS; ++c) {
              if (p.bsnd)
                tma_load_4d(vdst + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + st), c * 64, hk, kv0, w.b, pol_kv);
              else
                tma_load_4d(vdst + c * C::CHUNK_BYTES, &tm_v, bar(B_VFULL + st), c * 64, kv0, hk, w.b, pol_kv);
            }
          }
          v_pend[st] = true; v_issued[st] = kv_phase;
          FA_TRU(lead && j == N - 1, 0, n_claimed, 2);
          if (++st == C::KST) { st = 0; kv_phase ^= 1; }
        }
        ++n_claimed;
      }
      // Every copy this warp started lands before the CTA may exit (their
      // barriers complete on their own; the waits are bounded regardless).
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      for (int s = 0; s < C::KST; ++s) {
        if (k_pend[s]) mbar_wait(bar(B_KFULL + s), k_issued[s], drain);
        if (v_pend[s]) mbar_wait(bar(B_VFULL + s), v_issued[s], drain);
      }
      for (int i = 0; i < 2; ++i)
        if (q_pend[i]) mbar_wait(bar(B_QFULL + i), q_issued[i], drain);
    }
    __syncwarp();
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this role (warp-uniform control flow, descriptors in
    // uniform registers); elect.sync picks the one lane that issues each
    // tcgen05 instruction.  Only the start-address field of a descriptor
    // changes between MMAs, by compile-time offsets.
    constexpr uint32_t IDESC_S = idesc_f16(IS_BF16, false, 128, 128);
    constexpr uint32_t IDESC_PV = idesc_f16(IS_BF16, true, 128, D);
    const uint64_t dQ[2] = {smem_desc_sw128(sbase + C::OFF_Q, 16, 1024),
                            smem_desc_sw128(sbase + C::OFF_Q + C::TILE_BYTES, 16, 1024)};
    const uint64_t dK0 = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV0 = smem_desc_sw128(sbase + C::OFF_V, C::CHUNK_BYTES, 1024);
    uint32_t q_phase[2] = {0, 0}, kv_phase = 0, p_phase[4] = {0, 0, 0, 0};
    int st = 0;
    bool ok = true;
    const uint32_t tS[2] = {tmem + C::TMEM_S0, tmem + C::TMEM_S1};
    const uint32_t tO[2] = {tmem + C::TMEM_O0, tmem + C::TMEM_O1};
    auto wait_all = [&](int b, uint32_t ph) { return __all_sync(0xffffffffu, mbar_wait(bar(b), ph, wctx)); };
    int uslot = 0;
    uint32_t uphase = 0;
    bool first_unit_m = true;
    int n_units_m = 0;
    (void)n_units_m;
    while (ok) {
      if (!wait_all(B_UFULL + uslot, uphase)) break;
      Unit w;
      const int tk = ring_get(uslot, w);
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      const bool u_first = first_unit_m;
      first_unit_m = false;
      (void)u_first;
      FA_TRU(lane == 0, 1, n_units_m, 0);
      // Tile i takes part in KV steps [s_[i], s_[i] + n[i]) of the unit's walk
      // over tiles lo0 .. lo0 + N - 1 (s_ = {0, 0} unless a band shifts tile 1).
      const int n[2] = {w.n0, w.n1};
      const int s_[2] = {0, WALK ? w.s1 : 0};
      const int N = w.n0 > s_[1] + w.n1 ? w.n0 : s_[1] + w.n1;
      for (int i = 0; i < 2 && ok; ++i) {
        if (n[i] == 0) continue;
        if (!wait_all(B_QFULL + i, q_phase[i])) ok = false;
        q_phase[i] ^= 1;
      }
      int st_prev = 0;
      uint32_t ph_prev = 0;
      for (int j = 0; j <= N && ok; ++j) {
        // K_j is needed only by this iteration's S MMAs (waited for just
        // before the first of them), V_(j-1) by its P V.
        bool k_ready = false;
        FA_TR(lane == 0 && u_first, 16, j, 0);
        if (j > 0 && !wait_all(B_VFULL + st_prev, ph_prev)) { ok = false; break; }
        FA_TR(lane == 0 && u_first, 17, j, 0);
        tc_fence_after();
        if (PAGED && j > 0 && ((WALK ? w.lo0 : 0) + j - 1) * TC_BN + TC_BN > p.Nkv) {
          // Rows past Nkv of this V tile hold whatever the cache has there
          // (stale or never written).  Their P is 0, but 0 x NaN would still
          // reach O: clear them before the P V that reads this tile.
          const int r0 = p.Nkv - ((WALK ? w.lo0 : 0) + j - 1) * TC_BN;
          const uint32_t vbase = sbase + C::OFF_V + st_prev * C::TILE_BYTES;
          for (int c = 0; c < C::CHUNKS; ++c)
            for (int i = r0 * 8 + lane; i < TC_BN * 8; i += 32)  // 8 x 16 bytes per 128-byte row
              st_shared_v4(vbase + c * C::CHUNK_BYTES + i * 16, 0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
          __syncwarp();
        }
        const uint64_t dK = dK0 + (uint64_t)((st * C::TILE_BYTES) >> 4);
        const uint64_t dV = dV0 + (uint64_t)((st_prev * C::TILE_BYTES) >> 4);
        for (int i = 0; i < 2 && ok; ++i) {
          if (n[i] == 0) continue;
          if (j >= 1 + s_[i] && j - 1 < s_[i] + n[i]) {
            // O_i += P_i(j-1) V_(j-1), in two parts as the softmax hands them
            // over: part q holds keys [32q, 32q+32) of both key halves, i.e.
            // k-steps {2q, 2q+1, 4+2q, 5+2q}.
            const uint32_t acc0 = (j - 1 > s_[i]) ? 1u : 0u;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              // k-steps 2q, 2q+1 (keys of half 0) and 4+2q, 5+2q (half 1);
              // operands formed before the wait
              const int k0 = 2 * part, k1 = 2 * part + 1, k2 = 4 + 2 * part, k3 = 5 + 2 * part;
              const uint32_t a0 = tS[i] + (k0 >> 2) * 64 + (k0 & 3) * 8, a1 = tS[i] + (k1 >> 2) * 64 + (k1 & 3) * 8,
                             a2 = tS[i] + (k2 >> 2) * 64 + (k2 & 3) * 8, a3 = tS[i] + (k3 >> 2) * 64 + (k3 & 3) * 8;
              const uint64_t b0 = dV + (uint64_t)((k0 * 2048) >> 4), b1 = dV + (uint64_t)((k1 * 2048) >> 4),
                             b2 = dV + (uint64_t)((k2 * 2048) >> 4), b3 = dV + (uint64_t)((k3 * 2048) >> 4);
              if (!wait_all(B_PFULL + 2 * i + part, p_phase[2 * i + part])) { ok = false; break; }
              if (part == 0) FA_TR(lane == 0 && u_first, 16 + i, j - 1, 1);
              p_phase[2 * i + part] ^= 1;
              tc_fence_after();
              mma_ts4_elect(tO[i], a0, b0, a1, b1, a2, b2, a3, b3, IDESC_PV, part == 0 ? acc0 : 1u);
            }
            if (!ok) break;
            if (j - 1 == s_[i] + n[i] - 1) {
              mma_commit_elect(bar(B_OFULL + i));
              FA_TRU(lane == 0, 1, n_units_m, 2 + i);
            }
            // V_(j-1) is free once the last tile's P V has read it.
            const bool t1_uses = n[1] > 0 && j - 1 >= s_[1] && j - 1 < s_[1] + n[1];
            if (i == 1 || !t1_uses) mma_commit_elect(bar(B_VEMPTY + st_prev));
          }
          if (j >= s_[i] && j < s_[i] + n[i]) {
            if (!k_ready) {
              if (!wait_all(B_KFULL + st, kv_phase)) { ok = false; break; }
              k_ready = true;
              tc_fence_after();
            }
            // S_i(j) = Q_i K_j^T
            // d/16 k-steps, four per issue group (one 64-column chunk each)
#pragma unroll
            for (int c = 0; c < C::CHUNKS; ++c) {
              const uint64_t o0 = (uint64_t)((c * C::CHUNK_BYTES) >> 4);
              mma_ss4_elect(tS[i], dQ[i] + o0, dK + o0, dQ[i] + o0 + 2, dK + o0 + 2, dQ[i] + o0 + 4, dK + o0 + 4,
                            dQ[i] + o0 + 6, dK + o0 + 6, IDESC_S, c > 0 ? 1u : 0u);
            }
            mma_commit_elect(bar(B_SFULL + i));
            FA_TR(lane == 0 && u_first, 16 + i, j, 2);
            if (j == s_[i]) FA_TRU(lane == 0, 1, n_units_m, 4 + i);
            if (j == s_[i] + n[i] - 1) mma_commit_elect(bar(B_QEMPTY + i));
          }
        }
        if (!ok) break;
        if (WALK && j >= 1) {
          // a V tile no tile read (cannot happen for adjacent 128-row tiles,
          // whose key ranges overlap or touch): release it all the same
          const bool t0_uses = n[0] > 0 && j - 1 < n[0];
          const bool t1_uses = n[1] > 0 && j - 1 >= s_[1] && j - 1 < s_[1] + n[1];
          if (!t0_uses && !t1_uses) mma_commit_elect(bar(B_VEMPTY + st_prev));
        }
        if (j < N) mma_commit_elect(bar(B_KEMPTY + st));
        FA_TR(lane == 0 && u_first, 16, j, 3);
        st_prev = st;
        ph_prev = kv_phase;
        if (j < N) {
          if (++st == C::KST) { st = 0; kv_phase ^= 1; }
        }
      }
      ++n_units_m;
    }
    // Let every MMA this warp issued finish before the CTA frees TMEM.
    mma_commit_elect(bar(B_DRAIN));
    {
      WaitCtx drain{abort_flag, status_word, p.timeout_ns, 1u};
      volatile int no_abort = 0;
      drain.abort_flag = &no_abort;
      mbar_wait(bar(B_DRAIN), 0, drain);
    }
    __syncwarp();
  } else if (warp < TC_SOFTMAX_WARPS) {
    // ------------------------------------------------------------ softmax + epilogue
    const int tile = warp >> 3;             // warps 0-7: tile 0, warps 8-15: tile 1
    const int half = (warp >> 2) & 1;       // keys [64 half, 64 half + 64) of each KV tile
    const int r = (warp & 3) * 32 + lane;   // query row within the Q tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + (tile ? C::TMEM_S1 : C::TMEM_S0) + 64 * half;
    const uint32_t tO = tmem + lane_base + (tile ? C::TMEM_O1 : C::TMEM_O0) + (D / 2) * half;
    float* red_t = red + tile * (2 * 2 * TC_BM);  // [parity][half][row]
    const float sl2 = p.scale_log2;
    uint32_t s_phase = 0, o_phase = 0, x_phase = 0;
    bool ok = true;
    // One float per row is swapped with the other half of this tile through
    // shared memory (double-buffered by phase parity): publish() writes and
    // arrives, collect() waits (bounded) and reads the partner's value.
    auto publish = [&](float mine) {
      red_t[(x_phase * 2 + half) * TC_BM + r] = mine;
      mbar_arrive_warp(bar(B_XCHG + tile));
    };
    auto collect = [&](float& theirs) -> bool {
      const bool got = __all_sync(0xffffffffu, mbar_wait(bar(B_XCHG + tile), x_phase, wctx));
      if (got) theirs = red_t[(x_phase * 2 + (half ^ 1)) * TC_BM + r];
      x_phase ^= 1;
      return got;
    };
    int uslot = 0;
    uint32_t uphase = 0;
    bool first_unit = true;
    int n_units_s = 0;
    (void)n_units_s;
    while (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_UFULL + uslot), uphase, wctx));
      if (!ok) break;
      Unit w;
      const int tk = ring_get(uslot, w);
      const int sp = SPLIT ? unit_ring[16 * uslot + 9] : 0;  // split-KV: this unit's slice
      mbar_arrive_warp(bar(B_UEMPTY + uslot));
      if (++uslot == C::UNIT_SLOTS) { uslot = 0; uphase ^= 1; }
      if (tk < 0) break;
      FA_TRU(warp == 0 && lane == 0, 2, n_units_s, 0);
      const int n = tile ? w.n1 : w.n0;
      const bool this_first = first_unit;
      first_unit = false;
      if (n == 0) continue;
      const int qt = w.qt0 + tile;
      const int row = qt * TC_BM + r;
      (void)this_first;
      float m_ref = -INFINITY;  // running reference max (log2 domain), identical in both halves
      float l = 0.f;            // this half's share of the row sum
      for (int j = 0; j < n; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_SFULL + tile), s_phase, wctx));
        if (!ok) break;
        FA_TR(this_first && lane == 0, warp, j, 0);
        FA_TRU(warp == 0 && lane == 0 && j == 0, 2, n_units_s, 1);
        s_phase ^= 1;
        tc_fence_after();
        // KV tile of this step (a band or a split starts the tile's walk at lo0 (+ s1))
        const int kt = (WALK ? w.lo0 + (tile ? w.s1 : 0) : 0) + j;
        const int col0 = kt * TC_BN + 64 * half;
        bool need_mask = (kt * TC_BN + TC_BN > p.Nkv) || (p.causal && kt * TC_BN + TC_BN - 1 > qt * TC_BM);
        // visible keys of this row: [lo_c, lim_c)
        int lim_c = p.causal ? (row + 1 < p.Nkv ? row + 1 : p.Nkv) : p.Nkv;
        int lo_c = 0;
        if constexpr (BAND) {
          const long long first = (long long)kt * TC_BN, last = first + TC_BN - 1;
          need_mask = need_mask || first < (long long)qt * TC_BM + TC_BM - 1 - p.band.pre_tokens ||
                      last > (long long)qt * TC_BM + p.band.next_tokens;
          const long long hi = (long long)row + p.band.next_tokens + 1;
          lim_c = hi < p.Nkv ? (int)hi : p.Nkv;
          const long long lo = (long long)row - p.band.pre_tokens;
          lo_c = lo > 0 ? (int)lo : 0;
        }
        // This half's 64 scores stay in registers from the row max through the
        // exps (a second read of them from tensor memory delayed the P stores
        // behind it).
        float mt;
        float s[64];
        {
          tmem_ld64(tS, s);
          FA_TR(this_first && lane == 0, warp, j, 1);
          float mx[4];
          if (!need_mask) {
#pragma unroll
            for (int t = 0; t < 4; ++t) mx[t] = fmaxf(s[t], s[t + 4]);
#pragma unroll
            for (int c = 8; c < 64; c += 8)
#pragma unroll
              for (int t = 0; t < 4; ++t) mx[t] = fmax3(mx[t], s[c + t], s[c + 4 + t]);
          } else {
            // 16-key groups: skipped when masked for every row of the warp,
            // compared key by key only when partly visible.
#pragma unroll
            for (int t = 0; t < 4; ++t) mx[t] = -INFINITY;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int k0 = col0 + 16 * g;
              if (__all_sync(0xffffffffu, k0 >= lim_c || (BAND && k0 + 16 <= lo_c))) continue;
              if (!__all_sync(0xffffffffu, k0 + 16 <= lim_c && (!BAND || k0 >= lo_c))) {
#pragma unroll
                for (int c = 0; c < 16; ++c)
                  if (k0 + c >= lim_c || (BAND && k0 + c < lo_c)) s[16 * g + c] = -INFINITY;
              }
#pragma unroll
              for (int t = 0; t < 4; ++t) mx[t] = fmax3(mx[t], s[16 * g + t], s[16 * g + 4 + t]);
#pragma unroll
              for (int t = 0; t < 4; ++t) mx[t] = fmax3(mx[t], s[16 * g + 8 + t], s[16 * g + 12 + t]);
            }
          }
          mt = fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3]));
        }
        const float* sa = s;       // keys 0-31 of this half
        const float* sb = s + 32;  // keys 32-63
        FA_TR(this_first && lane == 0, warp, j, 2);
        // Reference max (log2 domain).  A warp waits for the other half's
        // candidate now only when one of its rows must move the reference;
        // otherwise it goes ahead with m_ref and checks the partner's
        // candidate after its exps (published long before).  The reference is
        // the exact max when it moves, so the largest P of that step is
        // exactly 1 (no rounding on the dominant weight).
        const float cand = mt * sl2;
        publish(cand);
        const bool waited = __any_sync(0xffffffffu, cand > m_ref + TC_RESCALE_THRESHOLD);
        float m_new = m_ref, m_use = m_ref;
        bool moved = false;
        if (waited) {
          float other = -INFINITY;
          ok = collect(other);
          if (!ok) break;
          const float mx2 = fmaxf(cand, other);
          if (mx2 > m_ref + TC_RESCALE_THRESHOLD) {
            moved = true;
            m_new = m_use = mx2;
          }
        }
        FA_TR(this_first && lane == 0, warp, j, 3);
        FA_TR(this_first && lane == 0, warp, j, 4);
        const float mref_use = (m_use == -INFINITY) ? 0.f : m_use;
        const uint64_t scale2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-mref_use, -mref_use);
        uint64_t acc2[2] = {0ull, 0ull};
        // 8 score pairs -> 8 packed P columns, written over this half's first
        // 32 S columns (already read).  With TC_POLY_EVERY > 0, on tiles
        // without masked scores one pair in TC_POLY_EVERY takes 2^x on the
        // FMA pipe.
        // On tiles with masked scores (never the polynomial form) a group
        // masked for every row of the warp writes zeros without exps, and a
        // partly visible group masks key by key.
        auto sub = [&](const float* sc, int cbase, auto use_poly) {
          uint32_t pk[8];
          const int k0 = col0 + cbase;
          if (!decltype(use_poly)::value && __all_sync(0xffffffffu, k0 >= lim_c || (BAND && k0 + 16 <= lo_c))) {
#pragma unroll
            for (int t = 0; t < 8; ++t) pk[t] = 0u;
            tmem_st8(tS + cbase / 2, pk);
            return;
          }
          const bool part =
              !decltype(use_poly)::value && !__all_sync(0xffffffffu, k0 + 16 <= lim_c && (!BAND || k0 >= lo_c));
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            float v0 = sc[2 * t], v1 = sc[2 * t + 1];
            if (part) {
              if (k0 + 2 * t >= lim_c || (BAND && k0 + 2 * t < lo_c)) v0 = -INFINITY;
              if (k0 + 2 * t + 1 >= lim_c || (BAND && k0 + 2 * t + 1 < lo_c)) v1 = -INFINITY;
            }
            const uint64_t x2 = f2_fma(f2_pack(v0, v1), scale2, negm2);
            float p0, p1;
            if (decltype(use_poly)::value && TC_POLY_EVERY > 0 && (t % TC_POLY_MOD) == TC_POLY_MOD - 1) {
              exp2_poly_x2(x2, p0, p1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            acc2[t & 1] = f2_add(acc2[t & 1], f2_pack(p0, p1));
            pk[t] = Pack<T>::two(p0, p1);
          }
          tmem_st8(tS + cbase / 2, pk);
        };
        // part 0: this half's keys 0-31
        if (need_mask) {
          sub(sa, 0, std::false_type{});
          sub(sa + 16, 16, std::false_type{});
        } else {
          sub(sa, 0, std::true_type{});
          sub(sa + 16, 16, std::true_type{});
        }
        // Settle this step's reference before any of its P is handed over.
        bool redo = false;
        if (!waited) {
          float other = -INFINITY;
          ok = collect(other);
          if (!ok) break;
          const float mx2 = fmaxf(cand, other);
          if (mx2 > m_ref + TC_RESCALE_THRESHOLD) {
            moved = redo = true;
            m_new = mx2;
          }
        }
        FA_TR(this_first && lane == 0, warp, j, 7);
        // Rescale this half of O in place when this warp moved any row's
        // reference max, before this step's P V touches O (O is quiescent:
        // its last P V finished before S_i(j) was signalled).  The factor
        // (and the SFU op) is only formed when a reference moved.
        if (j > 0 && __any_sync(0xffffffffu, moved)) {
          const float corr = moved ? ex2(m_ref - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 2; c += 32) {
            float ov[32];
            tmem_ld32(tO + c, ov);
            uint32_t ow[32];
#pragma unroll
            for (int t = 0; t < 32; ++t) ow[t] = __float_as_uint(ov[t] * corr);
            tmem_st32(tO + c, ow);
          }
        }
        // Hand part 0 to the MMA warp now, unless this warp's P must still be
        // rescaled (the other half moved the reference: rare).
        const bool warp_redo = __any_sync(0xffffffffu, redo);
        if (!warp_redo) {
          tmem_wait_st();
          tc_fence_before();
          if (p.fault_mode != 1) mbar_arrive_warp(bar(B_PFULL + 2 * tile));
        }
        // part 1: keys 32-63
        if (need_mask) {
          sub(sb, 32, std::false_type{});
          sub(sb + 16, 48, std::false_type{});
        } else {
          sub(sb, 32, std::true_type{});
          sub(sb + 16, 48, std::true_type{});
        }
        FA_TR(this_first && lane == 0, warp, j, 5);
        float sum;
        {
          float a0, a1;
          f2_unpack(f2_add(acc2[0], acc2[1]), a0, a1);
          sum = a0 + a1;
        }
        // The other half moved the reference after this half had computed P
        // against m_ref: scale this half's P and row sum by 2^(m_ref - m_new)
        // (rare; one extra rounding of that step's P), then hand over part 0.
        if (warp_redo) {
          const float f = redo ? ex2(m_ref - m_new) : 1.f;
          float pv[32];
          tmem_ld32(tS, pv);
          uint32_t pw[32];
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float2 q2 = Pack<T>::unpack(__float_as_uint(pv[t]));
            pw[t] = Pack<T>::two(q2.x * f, q2.y * f);
          }
          tmem_st32(tS, pw);
          sum *= f;
          tmem_wait_st();
          tc_fence_before();
          if (p.fault_mode != 1) mbar_arrive_warp(bar(B_PFULL + 2 * tile));
        }
        tmem_wait_st();
        tc_fence_before();
        if (p.fault_mode != 1) mbar_arrive_warp(bar(B_PFULL + 2 * tile + 1));
        if (moved) l *= ex2(m_ref - m_new);  // 0 when m_ref = -inf
        m_ref = m_new;
        l += sum;
        FA_TR(this_first && lane == 0, warp, j, 6);
        FA_TRU(warp == 0 && lane == 0 && j == n - 1, 2, n_units_s, 2);
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      float l_other = 0.f;
      publish(l);
      ok = collect(l_other);
      if (!ok) break;
      l += l_other;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(B_OFULL + tile), o_phase, wctx));
      if (!ok) break;
      o_phase ^= 1;
      FA_TRU(warp == 0 && lane == 0, 2, n_units_s, 3);
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool valid = row < p.Nq;
      if constexpr (SPLIT) {
        // This slice's normalised half row of O, in fp32, and the row's LSE
        // over the slice.  The TMEM loads are warp-wide; only the stores
        // depend on the row.
        const long long prow = (((long long)sp * p.B + w.b) * p.H + w.h) * p.Nq + row;
        float* op = static_cast<float*>(p.o) + prow * D + (D / 2) * half;
        const bool pvalid_row =
            valid && FA_INDEX_OK(status_word, prow >= 0 && prow < (long long)p.split.n_splits * p.B * p.H * p.Nq);
#pragma unroll 1
        for (int c = 0; c < D / 2; c += 32) {
          float ov[32];
          tmem_ld32(tO + c, ov);
          if (pvalid_row) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              *reinterpret_cast<float4*>(op + c + 4 * t) =
                  make_float4(ov[4 * t] * inv_l, ov[4 * t + 1] * inv_l, ov[4 * t + 2] * inv_l, ov[4 * t + 3] * inv_l);
          }
        }
        if (pvalid_row && half == 0) p.lse[prow] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
        ++n_units_s;
        continue;
      }
      // This half row of O as bf16/fp16 pairs: 16-byte chunk k = pk[4k..4k+3].
      constexpr int NC = D / 16;  // chunks per half row: 8 (d=128) or 4 (d=64)
      uint32_t pk[D / 4];
#pragma unroll
      for (int c = 0; c < D / 2; c += 32) {
        float ov[32];
        tmem_ld32(tO + c, ov);
#pragma unroll
        for (int t = 0; t < 16; ++t) pk[c / 2 + t] = Pack<T>::two(ov[2 * t] * inv_l, ov[2 * t + 1] * inv_l);
      }
      // Transpose the chunks within groups of NC lanes (XOR butterfly over
      // shuffles): lane i of a group then holds chunk i of each of the
      // group's NC rows, so that one store instruction writes whole
      // contiguous row segments instead of 32 scattered 16-byte pieces.
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
      if constexpr (NC == 8) stage(std::integral_constant<int, 4>{});
      stage(std::integral_constant<int, 2>{});
      stage(std::integral_constant<int, 1>{});
      {
        const int ci = lane % NC;                                    // chunk this lane stores
        const int rbase = qt * TC_BM + (warp & 3) * 32 + (lane / NC) * NC;  // first row of its group
        const long long rstride = p.bsnd ? (long long)p.H * D : (long long)D;
        T* obase = reinterpret_cast<T*>(p.o) +
                   (p.bsnd ? ((long long)w.b * p.Nq * p.H + w.h) * D : ((long long)w.b * p.H + w.h) * p.Nq * D) +
                   (D / 2) * half + 8 * ci;
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
      if (valid && half == 0 && p.lse != nullptr &&
          FA_INDEX_OK(status_word, ((long long)w.b * p.H + w.h) * p.Nq + row < (long long)p.B * p.H * p.Nq)) {
        p.lse[((long long)w.b * p.H + w.h) * p.Nq + row] = (m_ref + __log2f(l)) * 0.69314718055994530942f;
      }
      FA_TRU(warp == 0 && lane == 0, 2, n_units_s, 4);
      ++n_units_s;
    }
    // Any tcgen05.st of this thread has completed before the CTA frees TMEM.
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
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
