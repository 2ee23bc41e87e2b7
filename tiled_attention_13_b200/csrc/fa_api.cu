// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA
// descriptor encoding, launch configuration and the device status word.
//
// One translation unit holds every kernel so that they share the status word
// (a static __device__ variable).  The only device allocation is fa_fwd's
// 8 KB of tile-scheduler counters, made once per device on its first call;
// fa_fwd_noalloc uses a static array instead.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>
#include <utility>

#include "fa.h"

// Causal d = 128 calls on the one-row-per-thread kernel as well (build option,
// for comparison: measured slower than the two-tile kernel with a mask).
#ifndef FA_TC2_CAUSAL
#define FA_TC2_CAUSAL 0
#endif

// Head dim 64 with at most 128 keys on the four-pipeline short-key kernel
// (0: on the two-warpgroup one, for comparison).
#ifndef FA_SHORT_WG
#define FA_SHORT_WG 1
#endif

namespace fa {
// Bit 0: a bounded wait expired.  Written by kernels, read and cleared by
// fa_get_device_status().
__device__ unsigned int g_status_word = 0;
}  // namespace fa

#include "fa_fwd_short.cuh"
#include "fa_fwd_short_wg.cuh"
#include "fa_fwd_simt.cuh"
#include "fa_fwd_tc.cuh"
#include "fa_fwd_tile1.cuh"
#include "fa_fwd_tc2.cuh"
#include "fa_bwd.cuh"
#include "fa_decode.cuh"
#include "fa_splitkv_merge.cuh"

namespace {

constexpr uint32_t kDefaultTimeoutUs = 2000000u;
std::atomic<uint32_t> g_timeout_us{kDefaultTimeoutUs};
std::atomic<int> g_fault_mode{0};

constexpr int kMaxDevices = 64;
constexpr int kSchedSlots = 1024;  // per-device ring of per-launch ticket counters

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  unsigned int* status = nullptr;      // device address of fa::g_status_word
  fa::SchedSlot* sched = nullptr;      // kSchedSlots counters, allocated once
  std::atomic<uint64_t> launches{0};   // picks the counter slot of a launch
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Launch with programmatic stream serialization (FA_PDL != 0): the kernel
// may start while the previous kernel of the stream drains, and waits for it
// (griddepcontrol.wait) before touching global data.
#ifndef FA_PDL
#define FA_PDL 1
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = FA_PDL ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename K>
bool set_smem_attr(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// Shared-memory attributes of the short-key kernels.
bool set_short_attrs() {
  bool ok = true;
  ok &= set_smem_attr(fa::fa_fwd_short_kernel<64, __nv_bfloat16>, fa::ShCfg<64>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_short_kernel<128, __nv_bfloat16>, fa::ShCfg<128>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_short_kernel<64, __half>, fa::ShCfg<64>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_short_kernel<128, __half>, fa::ShCfg<128>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_short_wg_kernel<__nv_bfloat16>, fa::SW_SMEM_MAX);
  ok &= set_smem_attr(fa::fa_fwd_short_wg_kernel<__half>, fa::SW_SMEM_MAX);
  return ok;
}

// Shared-memory attributes of the one-tile kernels (d = 256, block-sparse).
template <typename T>
bool set_t1_attrs_t() {
  bool ok = true;
  ok &= set_smem_attr(fa::fa_fwd_t1_kernel<256, T, false>, fa::T1Cfg<256>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_t1_kernel<64, T, true>, fa::T1Cfg<64>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_t1_kernel<128, T, true>, fa::T1Cfg<128>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_t1_kernel<256, T, true>, fa::T1Cfg<256>::SMEM_BYTES);
  return ok;
}
bool set_t1_attrs() {
#ifdef FA_T1_DENSE
  // build option: plain d = 64 / 128 calls on the one-tile kernel as well
  if (!set_smem_attr(fa::fa_fwd_t1_kernel<64, __nv_bfloat16, false>, fa::T1Cfg<64>::SMEM_BYTES) ||
      !set_smem_attr(fa::fa_fwd_t1_kernel<128, __nv_bfloat16, false>, fa::T1Cfg<128>::SMEM_BYTES) ||
      !set_smem_attr(fa::fa_fwd_t1_kernel<64, __half, false>, fa::T1Cfg<64>::SMEM_BYTES) ||
      !set_smem_attr(fa::fa_fwd_t1_kernel<128, __half, false>, fa::T1Cfg<128>::SMEM_BYTES))
    return false;
#endif
  return set_t1_attrs_t<__nv_bfloat16>() && set_t1_attrs_t<__half>();
}

// Shared-memory attributes of the decode kernels (every row count).
template <int D, typename T, bool PAGED>
bool set_decode_attrs_p() {
  return set_smem_attr(fa::fa_decode_kernel<D, T, 1, PAGED>, fa::DecCfg<D>::SMEM_BYTES) &&
         set_smem_attr(fa::fa_decode_kernel<D, T, 2, PAGED>, fa::DecCfg<D>::SMEM_BYTES) &&
         set_smem_attr(fa::fa_decode_kernel<D, T, 4, PAGED>, fa::DecCfg<D>::SMEM_BYTES) &&
         set_smem_attr(fa::fa_decode_kernel<D, T, 8, PAGED>, fa::DecCfg<D>::SMEM_BYTES);
}
template <int D, typename T>
bool set_decode_attrs() {
  return set_decode_attrs_p<D, T, false>() && set_decode_attrs_p<D, T, true>();
}

// Shared-memory attributes of the backward, decode and one-row two-tile kernels.
bool set_more_attrs() {
  bool ok = true;
  ok &= set_smem_attr(fa::fa_fwd_tc2_kernel<128, __nv_bfloat16>, fa::T2Cfg<128>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_fwd_tc2_kernel<128, __half>, fa::T2Cfg<128>::SMEM_BYTES);
  ok &= set_decode_attrs<64, __nv_bfloat16>() && set_decode_attrs<128, __nv_bfloat16>();
  ok &= set_decode_attrs<64, __half>() && set_decode_attrs<128, __half>();
  ok &= set_smem_attr(fa::fa_bwd_kernel<64, __nv_bfloat16>, fa::BwdCfg<64>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_bwd_kernel<128, __nv_bfloat16>, fa::BwdCfg<128>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_bwd_kernel<64, __half>, fa::BwdCfg<64>::SMEM_BYTES);
  ok &= set_smem_attr(fa::fa_bwd_kernel<128, __half>, fa::BwdCfg<128>::SMEM_BYTES);
  return ok;
}

// Per-device one-time set-up with that device current: properties, the
// status word's device address, kernel shared-memory attributes and the
// driver's tensor-map encoder.
int device_setup(int dev, DeviceInfo** out) {
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
    di.supported = (prop.major == 10 && prop.minor == 0);
    di.num_sms = prop.multiProcessorCount;
    if (di.supported) {
      void* sym = nullptr;
      if (cudaGetSymbolAddress(&sym, fa::g_status_word) != cudaSuccess) return FA_ERR_LAUNCH;
      di.status = static_cast<unsigned int*>(sym);
      bool ok = true;
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16, false, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16, false, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half, false, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half, false, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16, true, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16, true, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half, true, false, true>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half, true, false, true>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_simt_kernel<64>, fa::simt_smem_bytes<64>());
      ok &= set_smem_attr(fa::fa_fwd_simt_kernel<128>, fa::simt_smem_bytes<128>());
      ok &= set_short_attrs();
      ok &= set_t1_attrs();
      ok &= set_more_attrs();
      if (!ok) return FA_ERR_LAUNCH;
      // The tile scheduler's ticket counters: one slot per launch in flight,
      // each put back to zero by the last CTA of its launch.
      void* sp = nullptr;
      if (cudaMalloc(&sp, kSchedSlots * sizeof(fa::SchedSlot)) != cudaSuccess) return FA_ERR_LAUNCH;
      if (cudaMemset(sp, 0, kSchedSlots * sizeof(fa::SchedSlot)) != cudaSuccess ||
          cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(sp);
        return FA_ERR_LAUNCH;
      }
      di.sched = static_cast<fa::SchedSlot*>(sp);
      if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          return FA_ERR_LAUNCH;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
    }
    di.ready = true;
  }
  if (!di.supported) return FA_ERR_NO_DEVICE;
  *out = &di;
  return FA_OK;
}

// 4-D tensor map over a [B, H, N, D] (BHND) or [B, N, H, D] (BSND) 16-bit
// tensor, box = 64 columns x box_rows rows of one (b, h), 128-byte swizzle,
// out-of-range rows read as zero.
bool make_tmap(CUtensorMap* tm, const void* base, bool bf16, bool bsnd, int64_t B, int64_t H, int64_t N,
               int64_t D, uint32_t box_rows = 128) {
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  const cuuint64_t es = 2;
  if (!bsnd) {
    dims[0] = D; dims[1] = N; dims[2] = H; dims[3] = B;
    strides[0] = D * es; strides[1] = N * D * es; strides[2] = H * N * D * es;
    box[0] = 64; box[1] = box_rows; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = N; dims[3] = B;
    strides[0] = D * es; strides[1] = H * D * es; strides[2] = N * H * D * es;
    box[0] = 64; box[1] = 1; box[2] = box_rows; box[3] = 1;
  }
  CUresult r = g_encode(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D tensor map over a paged cache [num_blocks, block_size, Hkv, D] of 16-bit
// values: dims (D, Hkv, block_size, num_blocks), box = 64 columns x
// min(block_size, 128) rows of one (block, head), 128-byte swizzle, reads
// outside the cache (e.g. block index num_blocks) fill with zeros.
bool make_tmap_paged(CUtensorMap* tm, const void* base, bool bf16, int64_t Hkv, int64_t bs, int64_t num_blocks,
                     int64_t D, int64_t box_rows = 128) {
  const cuuint64_t es = 2;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)bs, (cuuint64_t)num_blocks};
  cuuint64_t strides[3] = {D * es, Hkv * D * es, bs * Hkv * D * es};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)(bs < box_rows ? bs : box_rows), 1}, estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(tm, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The band of fa_fwd_band: key j visible to query i iff i - pre <= j <= i + next.
struct Band {
  int pre_tokens, next_tokens;
};

// A paged K/V cache as fa_fwd_paged receives it.
struct PagedKV {
  const int* block_table;  // [B, max_blocks] physical block of each logical block
  int64_t block_size, num_blocks, max_blocks;
};

// Split-KV as launch_tc receives it: the plan and the caller's workspace,
// o_part [n_splits, B, H, Nq, D] then lse_part [n_splits, B, H, Nq], fp32.
struct SplitKV {
  int n_splits, split_tiles;
  float* o_part;
  float* lse_part;
};

// The split-KV plan: the KV tiles of every (batch, head, Q-tile pair) cut
// into n_splits slices of split_tiles tiles, the last possibly shorter and
// none empty.  requested > 0 asks for that many slices (at most one per KV
// tile).  requested <= 0 picks the count with a wave model of the persistent
// grid: base_units * n_splits equal units over num_sms CTAs take
// ceil(units / num_sms) waves of (split_tiles + 1) tile steps each, the + 1
// standing for a unit's fixed cost (its Q load, the pipeline's fill and the
// epilogue); the first count with the lowest cost wins, trying up to about
// four units per SM.
// CTAs that run at once, for the split plan: decoding-shaped calls (Nq <= 8
// rows; at most 8 rows per K/V head go to the CUDA-core decode kernel, which
// fits two CTAs on an SM) count two per SM, others one.
int64_t plan_slots(int64_t Nq, int num_sms) {
  return Nq <= fa::DEC_ROWS ? (int64_t)fa::DEC_CTAS_PER_SM * num_sms : (int64_t)num_sms;
}

void split_plan(int64_t base_units, int64_t kv_tiles, int requested, int num_sms, int* n_splits,
                int* split_tiles) {
  int64_t S = 1;
  if (requested > 0) {
    S = requested < kv_tiles ? requested : kv_tiles;
  } else if (base_units > 0 && num_sms > 0) {
    int64_t smax = (4 * (int64_t)num_sms + base_units - 1) / base_units;
    if (smax > kv_tiles) smax = kv_tiles;
    if (smax > 4096) smax = 4096;
    int64_t best_cost = INT64_MAX;
    for (int64_t c = 1; c <= smax; ++c) {
      const int64_t t = (kv_tiles + c - 1) / c;
      const int64_t sc = (kv_tiles + t - 1) / t;
      const int64_t waves = (base_units * sc + num_sms - 1) / num_sms;
      const int64_t cost = waves * (t + 1);
      if (cost < best_cost) {
        best_cost = cost;
        S = c;
      }
    }
  }
  if (S < 1) S = 1;
  const int64_t t = (kv_tiles + S - 1) / S;
  *split_tiles = (int)t;
  *n_splits = (int)((kv_tiles + t - 1) / t);
}

// (batch, head) pairs per scheduling chunk: enough that the chunk's K and V
// (2 * Nkv * D * 2 bytes per K/V head, shared by `group` consecutive query
// heads) stay within a comfortable share of the 126 MB L2 while every CTA
// works on the chunk.  A whole number of groups when it holds one at all.
int chunk_heads_for(int64_t BH, int64_t Nkv, int64_t D, int64_t group = 1) {
  const double kv_head = 4.0 * (double)Nkv * (double)D;
  const double budget = 40.0 * 1024 * 1024;
  int64_t g = (int64_t)(budget / kv_head) * group;
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return (int)g;
}

template <int D, typename T>
int launch_tc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
              int64_t Hkv, int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream,
              DeviceInfo& di, const PagedKV* pg = nullptr, const Band* band = nullptr,
              const SplitKV* sk = nullptr) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D)) return FA_ERR_LAUNCH;
  if (pg == nullptr) {
    if (!make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D) || !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D))
      return FA_ERR_LAUNCH;
  } else {
    if (!make_tmap_paged(&tk, k, BF16, Hkv, pg->block_size, pg->num_blocks, D) ||
        !make_tmap_paged(&tv, v, BF16, Hkv, pg->block_size, pg->num_blocks, D))
      return FA_ERR_LAUNCH;
  }
  fa::TcParams p;
  p.o = sk != nullptr ? static_cast<void*>(sk->o_part) : o;  // split: the kernel writes the slices' partials
  p.lse = sk != nullptr ? sk->lse_part : lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
  p.n_pairs = (int)((qtiles + 1) / 2);
  const int64_t units = B * H * (int64_t)p.n_pairs * (sk != nullptr ? sk->n_splits : 1);
  if (units > INT32_MAX) return FA_ERR_UNSUPPORTED;
  p.n_units = (int)units;
  p.chunk_heads = chunk_heads_for(B * H, Nkv, D, H / Hkv);
  p.kv_group = (int)(H / Hkv);
  p.block_table = pg != nullptr ? pg->block_table : nullptr;
  p.block_size = pg != nullptr ? (int)pg->block_size : 0;
  p.max_blocks = pg != nullptr ? (int)pg->max_blocks : 0;
  p.num_blocks = pg != nullptr ? (int)pg->num_blocks : 0;
  if (sk != nullptr) {
    p.split.n_splits = sk->n_splits;
    p.split.split_tiles = sk->split_tiles;
  } else {
    p.band.pre_tokens = band != nullptr ? band->pre_tokens : 0;
    p.band.next_tokens = band != nullptr ? band->next_tokens : 0;
  }
  p.sched = di.sched + (di.launches.fetch_add(1) % kSchedSlots);
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(units < di.num_sms ? units : di.num_sms);
  if (band != nullptr)
    fa::fa_fwd_tc_kernel<D, T, false, true><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(
        tq, tk, tv, p, di.status);
  else if (sk != nullptr && pg == nullptr)
    fa::fa_fwd_tc_kernel<D, T, false, false, true><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(
        tq, tk, tv, p, di.status);
  else if (sk != nullptr)
    fa::fa_fwd_tc_kernel<D, T, true, false, true><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(
        tq, tk, tv, p, di.status);
  else if (pg == nullptr)
    fa::fa_fwd_tc_kernel<D, T, false><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p,
                                                                                                  di.status);
  else
    fa::fa_fwd_tc_kernel<D, T, true><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p,
                                                                                                 di.status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  if (sk != nullptr) {  // combine the slices into O and LSE, in stream order
    const int64_t rows = B * H * Nq;
    const int64_t blocks = (rows + fa::MERGE_ROWS_PER_CTA - 1) / fa::MERGE_ROWS_PER_CTA;
    if (launch_pdl(fa::fa_splitkv_merge_kernel<D, T>, dim3((unsigned int)blocks), dim3(fa::MERGE_THREADS), 0, stream,
                   (const float*)sk->o_part, (const float*)sk->lse_part, static_cast<T*>(o), lse, (int)B, (int)H,
                   (int)Nq, sk->n_splits, bsnd ? 1 : 0) != cudaSuccess)
      return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

// Keys fit one KV tile (Nkv <= 128): the short-key kernel, one pass of
// softmax per query tile, a static schedule and no work counter.  Plain
// (contiguous, causal or not, grouped or not) bf16/fp16 calls.
// The short-key kernel with four query-tile pipelines per CTA (head dim 64).
// K / V tensor maps load n_s = Nkv rounded up to 16 rows; two Q stages per
// pipeline when they fit in shared memory, else one.
template <typename T>
int launch_short_wg(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                    int64_t Hkv, int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream,
                    int num_sms, unsigned int* status) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  const int n_s = (int)((Nkv + 15) / 16) * 16;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, 64) || !make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, 64, n_s) ||
      !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, 64, n_s) || !make_tmap(&to, o, BF16, bsnd, B, H, Nq, 64))
    return FA_ERR_LAUNCH;
  fa::SwParams p;
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.qtiles = (int)((Nq + 127) / 128);
  const int64_t tiles = B * H * (int64_t)p.qtiles;
  if (tiles > INT32_MAX) return FA_ERR_UNSUPPORTED;
  p.n_tiles = (int)tiles;
  p.kv_group = (int)(H / Hkv);
  p.n_s = n_s;
  p.ns = fa::sw_smem_bytes(n_s, 2) <= fa::SW_SMEM_MAX ? 2 : 1;
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  const cudaError_t e = launch_pdl(fa::fa_fwd_short_wg_kernel<T>, dim3(grid), dim3(fa::SW_THREADS),
                                   (size_t)fa::sw_smem_bytes(n_s, p.ns), stream, tq, tk, tv, to, p, status);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

template <int D, typename T>
int launch_short(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                 int64_t Hkv, int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream,
                 int num_sms, unsigned int* status) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
#if FA_SHORT_WG
  if constexpr (D == 64)  // four tile pipelines per CTA
    return launch_short_wg<T>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, stream, num_sms, status);
#endif
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D) || !make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D) ||
      !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D) || !make_tmap(&to, o, BF16, bsnd, B, H, Nq, D))
    return FA_ERR_LAUNCH;
  fa::ShParams p;
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.qtiles = (int)((Nq + 127) / 128);
  const int64_t tiles = B * H * (int64_t)p.qtiles;
  if (tiles > INT32_MAX) return FA_ERR_UNSUPPORTED;
  p.n_tiles = (int)tiles;
  p.kv_group = (int)(H / Hkv);
  p.n_s = (int)((Nkv + 15) / 16) * 16;
  p.kv_steps = (int)((Nkv + 15) / 16);
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  fa::fa_fwd_short_kernel<D, T><<<grid, fa::SH_THREADS, fa::ShCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, to, p,
                                                                                            status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// A block-sparse mask as fa_fwd_block_sparse receives it.
struct BlockMask {
  const uint8_t* mask;  // [.., .., ceil(Nq/128), ceil(Nkv/128)]
  int64_t batch_stride, head_stride;
};

// The one-tile kernel: d = 256 (BLOCK false) or a block-sparse mask (BLOCK
// true, bm the mask).
template <int D, typename T, bool BLOCK>
int launch_t1(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H, int64_t Hkv,
              int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream, int num_sms,
              unsigned int* status, fa::SchedSlot* sched, const BlockMask* bm) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D) || !make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D) ||
      !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D))
    return FA_ERR_LAUNCH;
  fa::T1Params p;
  p.o = o;
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.qtiles = (int)((Nq + 127) / 128);
  p.kvtiles = (int)((Nkv + 127) / 128);
  const int64_t units = B * H * (int64_t)p.qtiles;
  if (units > INT32_MAX - 1024) return FA_ERR_UNSUPPORTED;
  p.n_units = (int)units;
  p.chunk_heads = chunk_heads_for(B * H, Nkv, D, H / Hkv);
  p.kv_group = (int)(H / Hkv);
  p.block_mask = bm != nullptr ? bm->mask : nullptr;
  p.mask_sb = bm != nullptr ? (long long)bm->batch_stride : 0;
  p.mask_sh = bm != nullptr ? (long long)bm->head_stride : 0;
  p.sched = sched;
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(units < num_sms ? units : num_sms);
  fa::fa_fwd_t1_kernel<D, T, BLOCK><<<grid, fa::T1_THREADS, fa::T1Cfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p, status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// The backward workspace: the fp32 dQ accumulator [B, H, Nq, d], then
// LSE * log2(e) and D = rowsum(dO o O), each [B, H, nq_pad] fp32 with nq_pad
// = Nq rounded up to 128; each part starts on a 256-byte boundary.
struct BwdLayout {
  int64_t nq_pad, off_lse2, off_delta, bytes;
};
BwdLayout bwd_layout(int64_t B, int64_t H, int64_t Nq, int64_t d) {
  BwdLayout L;
  auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
  L.nq_pad = (Nq + 127) / 128 * 128;
  L.off_lse2 = up(B * H * Nq * d * 4);
  L.off_delta = L.off_lse2 + up(B * H * L.nq_pad * 4);
  L.bytes = L.off_delta + up(B * H * L.nq_pad * 4);
  return L;
}

template <int D, typename T>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
               void* dq, void* dk, void* dv, void* ws, int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv,
               float scale, int causal, bool bsnd, cudaStream_t stream, unsigned int* status) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv, tdo, tdq;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D) || !make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D) ||
      !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D) || !make_tmap(&tdo, dout, BF16, bsnd, B, H, Nq, D))
    return FA_ERR_LAUNCH;
  const BwdLayout L = bwd_layout(B, H, Nq, D);
  {  // the fp32 dQ accumulator [B, H, Nq, D], for the kernel's reduce-adds: 32 x 32 boxes, 128-byte swizzle
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Nq, (cuuint64_t)H, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)(Nq * D * 4), (cuuint64_t)(H * Nq * D * 4)};
    cuuint32_t box[4] = {32, 32, 1, 1}, estr[4] = {1, 1, 1, 1};
    if (g_encode(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return FA_ERR_LAUNCH;
  }
  fa::BwdParams p;
  p.o = o; p.dout = dout; p.lse = lse;
  p.dq_acc = static_cast<float*>(ws);
  p.lse2 = reinterpret_cast<float*>(static_cast<char*>(ws) + L.off_lse2);
  p.delta = reinterpret_cast<float*>(static_cast<char*>(ws) + L.off_delta);
  p.dq = dq; p.dk = dk; p.dv = dv;
  p.B = (int)B; p.H = (int)H; p.Hkv = (int)Hkv; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.qtiles = (int)((Nq + 127) / 128);
  p.kvtiles = (int)((Nkv + 127) / 128);
  p.nq_pad = (int)L.nq_pad;
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  const int64_t ctas = (int64_t)p.kvtiles * B * Hkv;
  // pre kernel: D / 8 threads per padded query row (it also clears the dQ accumulator)
  const int64_t pre_items = B * H * L.nq_pad * (D / 8), post_items = B * H * Nq * (D / 8);
  if (ctas > INT32_MAX || pre_items > (int64_t)INT32_MAX * 256 || post_items > (int64_t)INT32_MAX * 256)
    return FA_ERR_UNSUPPORTED;
  fa::fa_bwd_pre_kernel<D, T><<<(unsigned int)((pre_items + 255) / 256), 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fa::fa_bwd_kernel<D, T><<<(unsigned int)ctas, fa::BWD_THREADS, fa::BwdCfg<D>::SMEM_BYTES, stream>>>(
      tq, tk, tv, tdo, tdq, p, status);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_LAUNCH;
  fa::fa_bwd_post_kernel<D, T><<<(unsigned int)((post_items + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// The one-row-per-thread two-tile kernel (plain calls: contiguous K/V, causal
// or not, grouped K/V heads).
template <int D, typename T>
int launch_tc2(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H, int64_t Hkv,
               int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream, int num_sms,
               unsigned int* status, fa::SchedSlot* slot) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D) || !make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D) ||
      !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D))
    return FA_ERR_LAUNCH;
  fa::TcParams p;
  p.o = o;
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
  p.n_pairs = (int)((qtiles + 1) / 2);
  const int64_t units = B * H * (int64_t)p.n_pairs;
  if (units > INT32_MAX - 1024) return FA_ERR_UNSUPPORTED;
  p.n_units = (int)units;
  p.chunk_heads = chunk_heads_for(B * H, Nkv, D, H / Hkv);
  p.kv_group = (int)(H / Hkv);
  p.block_table = nullptr;
  p.block_size = p.max_blocks = p.num_blocks = 0;
  p.band.pre_tokens = p.band.next_tokens = 0;
  p.sched = slot;
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(units < num_sms ? units : num_sms);
  fa::fa_fwd_tc2_kernel<D, T><<<grid, fa::T2_THREADS, fa::T2Cfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p, status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// Decoding-shaped split-KV (at most fa::DEC_ROWS query rows per batch and
// K/V head, contiguous K/V): the CUDA-core decode kernel over the plan's
// slices, then the merge when there is more than one slice.
template <int D, typename T>
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                  int64_t Hkv, int64_t Nq, int64_t Nkv, float scale, bool bsnd, cudaStream_t stream,
                  unsigned int* status, const SplitKV* sk, const PagedKV* pg) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tk, tv;
  if (pg != nullptr) {
    if (!make_tmap_paged(&tk, k, BF16, Hkv, pg->block_size, pg->num_blocks, D, fa::DEC_CHUNK) ||
        !make_tmap_paged(&tv, v, BF16, Hkv, pg->block_size, pg->num_blocks, D, fa::DEC_CHUNK))
      return FA_ERR_LAUNCH;
  } else if (!make_tmap(&tk, k, BF16, bsnd, B, Hkv, Nkv, D, fa::DEC_CHUNK) ||
             !make_tmap(&tv, v, BF16, bsnd, B, Hkv, Nkv, D, fa::DEC_CHUNK)) {
    return FA_ERR_LAUNCH;
  }
  fa::DecParams p;
  p.block_table = pg != nullptr ? pg->block_table : nullptr;
  p.max_blocks = pg != nullptr ? (int)pg->max_blocks : 0;
  p.bs_log2 = 0;
  if (pg != nullptr)
    while ((int64_t(1) << p.bs_log2) < pg->block_size) ++p.bs_log2;
  p.q = q;
  p.o = sk != nullptr ? static_cast<void*>(sk->o_part) : o;
  p.lse = sk != nullptr ? sk->lse_part : lse;
  p.B = (int)B; p.H = (int)H; p.Hkv = (int)Hkv; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_splits = sk != nullptr ? sk->n_splits : 1;
  p.split_keys = sk != nullptr ? sk->split_tiles * fa::TC_BN : (int)((Nkv + fa::TC_BN - 1) / fa::TC_BN) * fa::TC_BN;
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  const int64_t ctas = (int64_t)p.n_splits * B * Hkv;
  if (ctas > INT32_MAX) return FA_ERR_UNSUPPORTED;
  const int64_t R = Nq * (H / Hkv);  // rows per (batch, K/V head), at most fa::DEC_ROWS
  const dim3 grid((unsigned int)ctas);
  const int sm = fa::DecCfg<D>::SMEM_BYTES;
  auto kern = pg != nullptr ? (R <= 1   ? fa::fa_decode_kernel<D, T, 1, true>
                               : R <= 2 ? fa::fa_decode_kernel<D, T, 2, true>
                               : R <= 4 ? fa::fa_decode_kernel<D, T, 4, true>
                                        : fa::fa_decode_kernel<D, T, 8, true>)
                            : (R <= 1   ? fa::fa_decode_kernel<D, T, 1, false>
                               : R <= 2 ? fa::fa_decode_kernel<D, T, 2, false>
                               : R <= 4 ? fa::fa_decode_kernel<D, T, 4, false>
                                        : fa::fa_decode_kernel<D, T, 8, false>);
  if (launch_pdl(kern, grid, dim3(fa::DEC_THREADS), (size_t)sm, stream, tk, tv, p, status) != cudaSuccess)
    return FA_ERR_LAUNCH;
  if (sk != nullptr) {
    const int64_t rows = B * H * Nq;
    const int64_t blocks = (rows + fa::MERGE_ROWS_PER_CTA - 1) / fa::MERGE_ROWS_PER_CTA;
    if (launch_pdl(fa::fa_splitkv_merge_kernel<D, T>, dim3((unsigned int)blocks), dim3(fa::MERGE_THREADS), 0, stream,
                   (const float*)sk->o_part, (const float*)sk->lse_part, static_cast<T*>(o), lse, (int)B, (int)H,
                   (int)Nq, sk->n_splits, bsnd ? 1 : 0) != cudaSuccess)
      return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

template <int D>
int launch_simt(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                int64_t Hkv, int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream) {
  fa::SimtParams p;
  p.q = static_cast<const float*>(q);
  p.k = static_cast<const float*>(k);
  p.v = static_cast<const float*>(v);
  p.o = static_cast<float*>(o);
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.Hkv = (int)Hkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.n_qblocks = (int)((Nq + fa::SIMT_ROWS - 1) / fa::SIMT_ROWS);
  const int64_t blocks = B * H * (int64_t)p.n_qblocks;
  if (blocks > INT32_MAX) return FA_ERR_UNSUPPORTED;
  fa::fa_fwd_simt_kernel<D><<<(int)blocks, fa::SIMT_THREADS, fa::simt_smem_bytes<D>(), stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

namespace {

// fa_fwd and fa_fwd_gqa: validation (in the order the header states), then
// the launch.  Hkv == H is ordinary multi-head attention.
int fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
               int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int causal, int layout, int dtype,
               void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (d == 256 && dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // d = 256 is the one-tile kernel's
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;  // nothing to compute
  if (Nkv == 0) return FA_ERR_INVALID_ARG;         // softmax over an empty key set
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse != nullptr && !aligned(lse, 4)))
    return FA_ERR_MISALIGNED;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
#ifdef FA_T1_DENSE
  if (dtype != FA_DTYPE_FP32 && d != 256 && Nkv > fa::SH_MAX_NKV) {
    fa::SchedSlot* slot = di->sched + (di->launches.fetch_add(1) % kSchedSlots);
    if (dtype == FA_DTYPE_BF16)
      return d == 64 ? launch_t1<64, __nv_bfloat16, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                           di->num_sms, di->status, slot, nullptr)
                     : launch_t1<128, __nv_bfloat16, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd,
                                                            s, di->num_sms, di->status, slot, nullptr);
    return d == 64 ? launch_t1<64, __half, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                  di->num_sms, di->status, slot, nullptr)
                   : launch_t1<128, __half, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                   di->num_sms, di->status, slot, nullptr);
  }
#endif
  if (d == 256) {
    fa::SchedSlot* slot = di->sched + (di->launches.fetch_add(1) % kSchedSlots);
    return dtype == FA_DTYPE_BF16
               ? launch_t1<256, __nv_bfloat16, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                               di->num_sms, di->status, slot, nullptr)
               : launch_t1<256, __half, false>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, di->num_sms,
                                        di->status, slot, nullptr);
  }
  if (dtype == FA_DTYPE_FP32) {
    return d == 64 ? launch_simt<64>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s)
                   : launch_simt<128>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s);
  }
  if (Nkv <= fa::SH_MAX_NKV) {  // one KV tile per query tile
    if (dtype == FA_DTYPE_BF16)
      return d == 64 ? launch_short<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                       di->num_sms, di->status)
                     : launch_short<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                        di->num_sms, di->status);
    return d == 64 ? launch_short<64, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                              di->num_sms, di->status)
                   : launch_short<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                               di->num_sms, di->status);
  }
  if (d == 128 && (!causal || FA_TC2_CAUSAL)) {  // the one-row-per-thread kernel: measured faster without a mask
    fa::SchedSlot* slot = di->sched + (di->launches.fetch_add(1) % kSchedSlots);
    return dtype == FA_DTYPE_BF16
               ? launch_tc2<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                                di->num_sms, di->status, slot)
               : launch_tc2<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, di->num_sms,
                                         di->status, slot);
  }
  if (dtype == FA_DTYPE_BF16) {
    return d == 64
               ? launch_tc<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, *di)
               : launch_tc<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, *di);
  }
  return d == 64 ? launch_tc<64, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, *di)
                 : launch_tc<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, *di);
}

// Bytes of split-KV workspace for n_splits slices (none for one slice).
int64_t split_workspace_bytes(int64_t B, int64_t H, int64_t Nq, int64_t d, int n_splits) {
  return n_splits > 1 ? (int64_t)n_splits * B * H * Nq * (d + 1) * 4 : 0;
}

// fa_fwd_splitkv and fa_fwd_paged_splitkv: validation (in the order the
// header states), the plan, then the split kernel and the merge, or the plain
// kernel when the plan has one slice.  pg == nullptr: contiguous K/V.
int splitkv_common(const void* q, const void* k, const void* v, const PagedKV* pg, void* o, float* lse, int64_t B,
                   int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int num_splits,
                   void* workspace, int64_t workspace_bytes, int layout, int dtype, void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0 || workspace_bytes < 0) return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (pg != nullptr && (pg->block_size <= 0 || pg->num_blocks < 0 || pg->max_blocks < 0 ||
                        (pg->block_size & (pg->block_size - 1)) != 0 || pg->block_size < 16))
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // split-KV is the tensor-core kernel's
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;          // nothing to compute
  if (Nkv == 0) return FA_ERR_INVALID_ARG;                // softmax over an empty key set
  if (pg != nullptr && (pg->num_blocks == 0 || pg->max_blocks < (Nkv + pg->block_size - 1) / pg->block_size))
    return FA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || (pg != nullptr && pg->block_table == nullptr))
    return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (pg != nullptr && (pg->block_size > (1 << 20) || pg->num_blocks > INT32_MAX - 1 ||
                        pg->max_blocks > INT32_MAX || B * pg->max_blocks > INT32_MAX))
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse != nullptr && !aligned(lse, 4)) || (pg != nullptr && !aligned(pg->block_table, 4)))
    return FA_ERR_MISALIGNED;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;
  const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
  int S = 1, tiles = 0;
  split_plan(B * H * ((qtiles + 1) / 2), (Nkv + fa::TC_BN - 1) / fa::TC_BN, num_splits,
             (int)plan_slots(Nq, di->num_sms), &S, &tiles);
  const int64_t need = split_workspace_bytes(B, H, Nq, d, S);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return FA_ERR_MISALIGNED;
  }
  const SplitKV sk{S, tiles, static_cast<float*>(workspace),
                   need > 0 ? reinterpret_cast<float*>(static_cast<char*>(workspace) + (int64_t)S * B * H * Nq * d * 4)
                            : nullptr};
  const SplitKV* skp = S > 1 ? &sk : nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  if (Nq * (H / Hkv) <= fa::DEC_ROWS) {  // decoding-shaped: the CUDA-core kernel, contiguous or paged
    if (dtype == FA_DTYPE_BF16)
      return d == 64 ? launch_decode<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, bsnd, s,
                                                        di->status, skp, pg)
                     : launch_decode<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, bsnd, s,
                                                         di->status, skp, pg);
    return d == 64 ? launch_decode<64, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, bsnd, s, di->status, skp,
                                               pg)
                   : launch_decode<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, bsnd, s, di->status, skp,
                                                pg);
  }
  if (dtype == FA_DTYPE_BF16)
    return d == 64 ? launch_tc<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, pg,
                                                  nullptr, skp)
                   : launch_tc<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, pg,
                                                   nullptr, skp);
  return d == 64 ? launch_tc<64, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, pg, nullptr, skp)
                 : launch_tc<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, pg, nullptr,
                                          skp);
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H, int64_t Nq,
           int64_t Nkv, int64_t d, float scale, int causal, int layout, int dtype, void* stream) {
  return fwd_common(q, k, v, o, lse, B, H, H, Nq, Nkv, d, scale, causal, layout, dtype, stream);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
               int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int causal, int layout, int dtype,
               void* stream) {
  return fwd_common(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, d, scale, causal, layout, dtype, stream);
}

int fa_fwd_band(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int64_t pre_tokens,
                int64_t next_tokens, int layout, int dtype, void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0 || pre_tokens < 0 || next_tokens < 0)
    return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // the band path is the tensor-core kernel's
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;          // nothing to compute
  if (Nkv == 0) return FA_ERR_INVALID_ARG;                // softmax over an empty key set
  if (pre_tokens < Nq - Nkv) return FA_ERR_INVALID_ARG;   // the last query rows would see no key
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse != nullptr && !aligned(lse, 4)))
    return FA_ERR_MISALIGNED;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);
  // widths past the sequences change nothing; keep them in int range
  const int64_t cap = Nq + Nkv;
  const Band band{(int)(pre_tokens < cap ? pre_tokens : cap), (int)(next_tokens < cap ? next_tokens : cap)};

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  if (dtype == FA_DTYPE_BF16)
    return d == 64 ? launch_tc<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di,
                                                  nullptr, &band)
                   : launch_tc<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di,
                                                   nullptr, &band);
  return d == 64 ? launch_tc<64, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, nullptr, &band)
                 : launch_tc<128, __half>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, 0, bsnd, s, *di, nullptr,
                                          &band);
}

int fa_bwd_workspace_size(int64_t B, int64_t H, int64_t Nq, int64_t d, int64_t* workspace_bytes) {
  if (B < 0 || H < 0 || Nq < 0 || (d != 64 && d != 128) || workspace_bytes == nullptr) return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256) return FA_ERR_UNSUPPORTED;
  *workspace_bytes = (B == 0 || H == 0 || Nq == 0) ? 0 : bwd_layout(B, H, Nq, d).bytes;
  return FA_OK;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, void* workspace, int64_t workspace_bytes, int64_t B, int64_t H, int64_t Hkv,
           int64_t Nq, int64_t Nkv, int64_t d, float scale, int causal, int layout, int dtype, void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0 || workspace_bytes < 0) return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // the backward is the tensor-core kernel's
  if (B == 0 || H == 0 || (Nq == 0 && Nkv == 0)) return FA_OK;
  if (Nkv == 0) return FA_ERR_INVALID_ARG;  // the forward was not defined
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || dout == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr)
    return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return FA_ERR_MISALIGNED;
  if (Nq > 0) {
    if (workspace == nullptr || workspace_bytes < bwd_layout(B, H, Nq, d).bytes) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
  }
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  if (Nq == 0) {  // no query: dK = dV = 0
    const size_t nb = (size_t)(B * Hkv * Nkv * d * 2);
    if (cudaMemsetAsync(dk, 0, nb, s) != cudaSuccess || cudaMemsetAsync(dv, 0, nb, s) != cudaSuccess)
      return FA_ERR_LAUNCH;
    return FA_OK;
  }
  if (dtype == FA_DTYPE_BF16)
    return d == 64 ? launch_bwd<64, __nv_bfloat16>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nkv,
                                                   scale, causal, bsnd, s, di->status)
                   : launch_bwd<128, __nv_bfloat16>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nkv,
                                                    scale, causal, bsnd, s, di->status);
  return d == 64 ? launch_bwd<64, __half>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nkv, scale,
                                          causal, bsnd, s, di->status)
                 : launch_bwd<128, __half>(q, k, v, o, dout, lse, dq, dk, dv, workspace, B, H, Hkv, Nq, Nkv, scale,
                                           causal, bsnd, s, di->status);
}

int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, const uint8_t* block_mask,
                        int64_t mask_batch_stride, int64_t mask_head_stride, int64_t B, int64_t H, int64_t Hkv,
                        int64_t Nq, int64_t Nkv, int64_t d, float scale, int causal, int layout, int dtype,
                        void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0 || mask_batch_stride < 0 || mask_head_stride < 0)
    return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // the block-sparse path is the tensor-core kernel's
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;          // nothing to compute
  if (Nkv == 0) return FA_ERR_INVALID_ARG;                // softmax over an empty key set
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || block_mask == nullptr) return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256 ||
      (Nkv + 127) / 128 > 32 * fa::T1_MAX_WORDS)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse != nullptr && !aligned(lse, 4)))
    return FA_ERR_MISALIGNED;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  const BlockMask bm{block_mask, mask_batch_stride, mask_head_stride};
  fa::SchedSlot* slot = di->sched + (di->launches.fetch_add(1) % kSchedSlots);
  const int n = di->num_sms;
  unsigned int* sw = di->status;
  if (dtype == FA_DTYPE_BF16) {
    if (d == 64)
      return launch_t1<64, __nv_bfloat16, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
    if (d == 128)
      return launch_t1<128, __nv_bfloat16, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
    return launch_t1<256, __nv_bfloat16, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
  }
  if (d == 64)
    return launch_t1<64, __half, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
  if (d == 128)
    return launch_t1<128, __half, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
  return launch_t1<256, __half, true>(q, k, v, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s, n, sw, slot, &bm);
}

int fa_fwd_paged(const void* q, const void* k_cache, const void* v_cache, const int* block_table, void* o,
                 float* lse, int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                 int64_t block_size, int64_t num_blocks, int64_t max_blocks, float scale, int causal, int layout,
                 int dtype, void* stream) {
  if (B < 0 || H < 0 || Hkv < 0 || Nq < 0 || Nkv < 0 || d <= 0 || block_size <= 0 || num_blocks < 0 ||
      max_blocks < 0)
    return FA_ERR_INVALID_ARG;
  if (H > 0 && (Hkv < 1 || H % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if ((block_size & (block_size - 1)) != 0 || block_size < 16) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;  // the paged path is the tensor-core kernel's
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;          // nothing to compute
  if (Nkv == 0) return FA_ERR_INVALID_ARG;                // softmax over an empty key set
  if (num_blocks == 0 || max_blocks < (Nkv + block_size - 1) / block_size) return FA_ERR_INVALID_ARG;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || o == nullptr)
    return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256 ||
      block_size > (1 << 20) || num_blocks > INT32_MAX - 1 || max_blocks > INT32_MAX || B * max_blocks > INT32_MAX)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(block_table, 4) || (lse != nullptr && !aligned(lse, 4)))
    return FA_ERR_MISALIGNED;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  DeviceInfo* di = nullptr;
  const int st = device_setup(dev, &di);
  if (st != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  const PagedKV pg{block_table, block_size, num_blocks, max_blocks};
  if (dtype == FA_DTYPE_BF16)
    return d == 64 ? launch_tc<64, __nv_bfloat16>(q, k_cache, v_cache, o, lse, B, H, Hkv, Nq, Nkv, scale, causal,
                                                  bsnd, s, *di, &pg)
                   : launch_tc<128, __nv_bfloat16>(q, k_cache, v_cache, o, lse, B, H, Hkv, Nq, Nkv, scale, causal,
                                                   bsnd, s, *di, &pg);
  return d == 64 ? launch_tc<64, __half>(q, k_cache, v_cache, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                         *di, &pg)
                 : launch_tc<128, __half>(q, k_cache, v_cache, o, lse, B, H, Hkv, Nq, Nkv, scale, causal, bsnd, s,
                                          *di, &pg);
}

int fa_splitkv_plan(int64_t B, int64_t H, int64_t Nq, int64_t Nkv, int64_t d, int num_splits, int num_sms,
                    int* splits, int64_t* workspace_bytes) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || (d != 64 && d != 128) || splits == nullptr ||
      workspace_bytes == nullptr)
    return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (num_sms <= 0) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
    DeviceInfo* di = nullptr;
    const int st = device_setup(dev, &di);
    if (st != FA_OK) return st;
    num_sms = di->num_sms;
  }
  int S = 1, tiles = 0;
  if (B > 0 && H > 0 && Nq > 0 && Nkv > 0) {
    const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
    split_plan(B * H * ((qtiles + 1) / 2), (Nkv + fa::TC_BN - 1) / fa::TC_BN, num_splits,
               (int)plan_slots(Nq, num_sms), &S, &tiles);
  }
  *splits = S;
  *workspace_bytes = split_workspace_bytes(B, H, Nq, d, S);
  return FA_OK;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                   int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d, float scale, int num_splits, void* workspace,
                   int64_t workspace_bytes, int layout, int dtype, void* stream) {
  return splitkv_common(q, k, v, nullptr, o, lse, B, H, Hkv, Nq, Nkv, d, scale, num_splits, workspace,
                        workspace_bytes, layout, dtype, stream);
}

int fa_fwd_paged_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* block_table, void* o,
                         float* lse, int64_t B, int64_t H, int64_t Hkv, int64_t Nq, int64_t Nkv, int64_t d,
                         int64_t block_size, int64_t num_blocks, int64_t max_blocks, float scale, int num_splits,
                         void* workspace, int64_t workspace_bytes, int layout, int dtype, void* stream) {
  const PagedKV pg{block_table, block_size, num_blocks, max_blocks};
  return splitkv_common(q, k_cache, v_cache, &pg, o, lse, B, H, Hkv, Nq, Nkv, d, scale, num_splits, workspace,
                        workspace_bytes, layout, dtype, stream);
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dim or size";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: pointer alignment";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH: CUDA launch or descriptor failure";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a bounded device wait expired";
    case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE: no usable sm_100 device";
    case FA_ERR_TOO_LARGE: return "FA_ERR_TOO_LARGE: the problem needs more than fa_fwd_noalloc's fixed scratch";
    case FA_ERR_CHECK: return "FA_ERR_CHECK: a debug build found a computed index out of bounds";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  unsigned int w = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&w, fa::g_status_word, sizeof(w)) != cudaSuccess) return FA_ERR_LAUNCH;
  if (w != 0 && cudaMemcpyToSymbol(fa::g_status_word, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_LAUNCH;
  if (w & 2u) return FA_ERR_CHECK;  // bit 1: a debug build's index check failed
  return (w & 1u) ? FA_ERR_TIMEOUT : FA_OK;
}

uint32_t fa_set_wait_timeout_us(uint32_t us) {
  return g_timeout_us.exchange(us == 0 ? kDefaultTimeoutUs : us);
}

int fa_debug_set_fault(int mode) { return g_fault_mode.exchange(mode); }

int fa_abi_version(void) { return (1 << 16) | 7; }

#ifdef FA_TRACE_SHORT
// which = 0: the two-warpgroup short-key kernel's timeline, 1: the four-pipeline one's
int fa_debug_short_trace_read(unsigned long long* host, int n, int which) {
  const int total = which ? fa::SWT_CTAS * fa::SWT_EV : fa::SHT_CTAS * fa::SHT_EV;
  if (n > total) n = total;
  const cudaError_t e = which ? cudaMemcpyFromSymbol(host, fa::g_trace_short_wg, n * sizeof(unsigned long long))
                              : cudaMemcpyFromSymbol(host, fa::g_trace_short, n * sizeof(unsigned long long));
  return e == cudaSuccess ? n : FA_ERR_LAUNCH;
}
#endif

#ifdef FA_TRACE_BWD
int fa_debug_bwd_trace_read(unsigned long long* host, int n) {
  const int total = fa::BWT_CTAS * fa::BWT_STEPS * fa::BWT_EV;
  if (n > total) n = total;
  return cudaMemcpyFromSymbol(host, fa::g_trace_bwd, n * sizeof(unsigned long long)) == cudaSuccess ? n
                                                                                                    : FA_ERR_LAUNCH;
}
#endif

#ifdef FA_TRACE_UNITS
int fa_debug_trace_units_read(unsigned long long* host, int n) {
  const int total = 3 * fa::TRU_N * fa::TRU_EV;
  if (n > total) n = total;
  if (cudaMemcpyFromSymbol(host, fa::g_trace_units, n * sizeof(unsigned long long)) != cudaSuccess)
    return FA_ERR_LAUNCH;
  return n;
}
#endif

#ifdef FA_TRACE
int fa_debug_trace_read(unsigned long long* host, int n) {
  const int total = fa::TRACE_STREAMS * fa::TRACE_J * fa::TRACE_EV;
  if (n > total) n = total;
  if (cudaMemcpyFromSymbol(host, fa::g_trace, n * sizeof(unsigned long long)) != cudaSuccess) return FA_ERR_LAUNCH;
  static unsigned long long zeros[fa::TRACE_STREAMS * fa::TRACE_J * fa::TRACE_EV];
  cudaMemcpyToSymbol(fa::g_trace, zeros, sizeof(zeros));
  return n;
}
#endif

}  // extern "C"

// ---------------------------------------------------------------- fa_fwd_noalloc
// An entry point for callers that must not allocate device memory at all:
// code running inside a memory pool or arena it does not own, real-time or
// embedded services that reserve all device memory up front, or hosts that
// forbid cudaMalloc after start-up.  fa_fwd's tile scheduler keeps its work
// counters in an 8 KB buffer that it allocates on its first call on a device;
// this variant keeps the counter in a fixed static device array instead, so
// none of its calls allocates anything.
namespace fa {
constexpr int kNoAllocScratchBytes = 256;
constexpr int kNoAllocScratchSlots = kNoAllocScratchBytes / (int)sizeof(SchedSlot);
// One copy per device that loads the library, held until the process exits.
// Every call of fa_fwd_noalloc on a device uses slot 0 (its work-ticket
// counter and its finished-CTA counter, 8 bytes); the rest of the 256 bytes
// is unused padding.  See the header for why overlapping calls race.
static __device__ __align__(256) SchedSlot g_noalloc_scratch[kNoAllocScratchSlots];
static_assert(sizeof(SchedSlot) <= kNoAllocScratchBytes, "the fixed scratch must hold one scheduler slot");
}  // namespace fa

namespace {

struct NoAllocDevice {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  unsigned int* status = nullptr;       // device address of fa::g_status_word
  fa::SchedSlot* scratch = nullptr;     // device address of fa::g_noalloc_scratch
};
NoAllocDevice g_noalloc_dev[kMaxDevices];

// Once per device, with that device current.  Host code only holds a stand-in
// for a __device__ variable's name, so the device address of the scratch
// array comes from cudaGetSymbolAddress.  Nothing here allocates memory.
int noalloc_setup(int dev, NoAllocDevice** out) {
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  NoAllocDevice& nd = g_noalloc_dev[dev];
  if (!nd.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
    nd.supported = (prop.major == 10 && prop.minor == 0);
    nd.num_sms = prop.multiProcessorCount;
    if (nd.supported) {
      void* sym = nullptr;
      if (cudaGetSymbolAddress(&sym, fa::g_status_word) != cudaSuccess) return FA_ERR_LAUNCH;
      nd.status = static_cast<unsigned int*>(sym);
      void* scr = nullptr;
      if (cudaGetSymbolAddress(&scr, fa::g_noalloc_scratch) != cudaSuccess || scr == nullptr)
        return FA_ERR_LAUNCH;
      nd.scratch = static_cast<fa::SchedSlot*>(scr);
      bool ok = true;
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __nv_bfloat16>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __nv_bfloat16>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<64, __half>, fa::TcCfg<64>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_tc_kernel<128, __half>, fa::TcCfg<128>::SMEM_BYTES);
      ok &= set_smem_attr(fa::fa_fwd_simt_kernel<64>, fa::simt_smem_bytes<64>());
      ok &= set_smem_attr(fa::fa_fwd_simt_kernel<128>, fa::simt_smem_bytes<128>());
      ok &= set_short_attrs();
      ok &= set_t1_attrs();
      ok &= set_more_attrs();  // also the one-row two-tile and decode kernels
      if (!ok) return FA_ERR_LAUNCH;
      if (g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          return FA_ERR_LAUNCH;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
    }
    nd.ready = true;
  }
  if (!nd.supported) return FA_ERR_NO_DEVICE;
  *out = &nd;
  return FA_OK;
}

template <int D, typename T>
int launch_tc_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
                      int64_t Nq, int64_t Nkv, float scale, int causal, bool bsnd, cudaStream_t stream,
                      const NoAllocDevice& nd) {
  constexpr bool BF16 = std::is_same<T, __nv_bfloat16>::value;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, BF16, bsnd, B, H, Nq, D) || !make_tmap(&tk, k, BF16, bsnd, B, H, Nkv, D) ||
      !make_tmap(&tv, v, BF16, bsnd, B, H, Nkv, D))
    return FA_ERR_LAUNCH;
  fa::TcParams p;
  p.o = o;
  p.lse = lse;
  p.B = (int)B; p.H = (int)H; p.Nq = (int)Nq; p.Nkv = (int)Nkv;
  p.bsnd = bsnd ? 1 : 0;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
  p.n_pairs = (int)((qtiles + 1) / 2);
  p.n_units = (int)(B * H * (int64_t)p.n_pairs);
  p.chunk_heads = chunk_heads_for(B * H, Nkv, D);
  p.kv_group = 1;        // one K/V head per query head
  p.block_table = nullptr;  // contiguous K/V
  p.block_size = p.max_blocks = p.num_blocks = 0;
  p.band.pre_tokens = p.band.next_tokens = 0;
  p.sched = nd.scratch;  // slot 0 of the static array
  p.timeout_ns = (uint64_t)g_timeout_us.load() * 1000ull;
  p.fault_mode = g_fault_mode.load();
  const int grid = (int)(p.n_units < nd.num_sms ? p.n_units : nd.num_sms);
  // The counter must start at zero: the previous call's last CTA normally
  // leaves it so, but clear it in stream order anyway (no allocation).
  if (cudaMemsetAsync(nd.scratch, 0, sizeof(fa::SchedSlot), stream) != cudaSuccess) return FA_ERR_LAUNCH;
  fa::fa_fwd_tc_kernel<D, T><<<grid, fa::TC_THREADS, fa::TcCfg<D>::SMEM_BYTES, stream>>>(tq, tk, tv, p,
                                                                                         nd.status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace

extern "C" int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                              int64_t H, int64_t Nq, int64_t Nkv, int64_t d, float scale, int causal, int layout,
                              int dtype, void* stream) {
  if (B < 0 || H < 0 || Nq < 0 || Nkv < 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (layout != FA_LAYOUT_BHND && layout != FA_LAYOUT_BSND) return FA_ERR_INVALID_ARG;
  if (dtype != FA_DTYPE_BF16 && dtype != FA_DTYPE_FP16 && dtype != FA_DTYPE_FP32) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (d == 256 && dtype == FA_DTYPE_FP32) return FA_ERR_UNSUPPORTED;
  if (B == 0 || H == 0 || Nq == 0) return FA_OK;
  if (Nkv == 0) return FA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return FA_ERR_INVALID_ARG;
  if (B > INT32_MAX || H > INT32_MAX || B * H > INT32_MAX || Nq > INT32_MAX - 256 || Nkv > INT32_MAX - 256)
    return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse != nullptr && !aligned(lse, 4)))
    return FA_ERR_MISALIGNED;
  // Slot 0 of the fixed scratch holds the 32-bit work-ticket counter: a call
  // fits when it can number all its work units (pairs of 128-row query tiles
  // over every batch and head) plus one closing ticket per CTA.
  const int64_t qtiles = (Nq + fa::TC_BM - 1) / fa::TC_BM;
  const int64_t units = B * H * (d == 256 ? qtiles : (qtiles + 1) / 2);  // d = 256: one query tile per unit
  if (dtype != FA_DTYPE_FP32 && units > (int64_t)INT32_MAX - 1024) return FA_ERR_TOO_LARGE;
  if (!(scale > 0.f) || std::isinf(scale)) scale = 1.0f / std::sqrt((float)d);

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_NO_DEVICE;
  NoAllocDevice* nd = nullptr;
  const int st = noalloc_setup(dev, &nd);
  if (st != FA_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bsnd = layout == FA_LAYOUT_BSND;
  if (dtype == FA_DTYPE_FP32) {  // this kernel uses no scratch at all
    return d == 64 ? launch_simt<64>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s)
                   : launch_simt<128>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s);
  }
  if (d == 256) {  // the one-tile kernel, its ticket counter in slot 0 of the fixed scratch
    if (cudaMemsetAsync(nd->scratch, 0, sizeof(fa::SchedSlot), s) != cudaSuccess) return FA_ERR_LAUNCH;
    return dtype == FA_DTYPE_BF16
               ? launch_t1<256, __nv_bfloat16, false>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s, nd->num_sms,
                                               nd->status, nd->scratch, nullptr)
               : launch_t1<256, __half, false>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s, nd->num_sms,
                                        nd->status, nd->scratch, nullptr);
  }
  if (Nkv <= fa::SH_MAX_NKV) {  // the short-key kernel uses no scratch at all
    if (dtype == FA_DTYPE_BF16)
      return d == 64 ? launch_short<64, __nv_bfloat16>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s,
                                                       nd->num_sms, nd->status)
                     : launch_short<128, __nv_bfloat16>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s,
                                                        nd->num_sms, nd->status);
    return d == 64 ? launch_short<64, __half>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s, nd->num_sms,
                                              nd->status)
                   : launch_short<128, __half>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s, nd->num_sms,
                                               nd->status);
  }
  if (d == 128 && (!causal || FA_TC2_CAUSAL)) {  // as fa_fwd: the one-row-per-thread kernel, its counter in slot 0
    if (cudaMemsetAsync(nd->scratch, 0, sizeof(fa::SchedSlot), s) != cudaSuccess) return FA_ERR_LAUNCH;
    return dtype == FA_DTYPE_BF16
               ? launch_tc2<128, __nv_bfloat16>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s,
                                                nd->num_sms, nd->status, nd->scratch)
               : launch_tc2<128, __half>(q, k, v, o, lse, B, H, H, Nq, Nkv, scale, causal, bsnd, s, nd->num_sms,
                                         nd->status, nd->scratch);
  }
  if (dtype == FA_DTYPE_BF16) {
    return d == 64 ? launch_tc_noalloc<64, __nv_bfloat16>(q, k, v, o, lse, B, H, Nq, Nkv, scale, causal, bsnd, s, *nd)
                   : launch_tc_noalloc<128, __nv_bfloat16>(q, k, v, o, lse, B, H, Nq, Nkv, scale, causal, bsnd, s,
                                                           *nd);
  }
  return d == 64 ? launch_tc_noalloc<64, __half>(q, k, v, o, lse, B, H, Nq, Nkv, scale, causal, bsnd, s, *nd)
                 : launch_tc_noalloc<128, __half>(q, k, v, o, lse, B, H, Nq, Nkv, scale, causal, bsnd, s, *nd);
}
