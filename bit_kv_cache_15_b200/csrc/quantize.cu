// quantize.cu -- KVarN quantise-on-write for whole 128-token tiles (sm_100a).
//
// The four stages of [hypho] "KV-cache 量化终于能跑生产了？KVarN …", section
// 它怎么做到的：四步流水线 (= [lehuy] "KVarN: Backend lượng tử hóa KV-cache …",
// section Cơ chế hoạt động), one (token group, KV head, K|V) tile at a time:
//   1 stage   the fp16 tile is brought into shared memory by the TMA engine
//             (cp.async.bulk.tensor, two 64-channel boxes, 128-byte swizzle so
//             ldmatrix reads are conflict-free).  CTAs are persistent and load
//             the next tile while they compute the current one;
//   2-5       rotate, normalise, quantise and pack: quant_tile.cuh, with R
//             kept in tensor memory between the rotation and quantisation.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kvarn_internal.h"
#include "quant_tile.cuh"

namespace kvarn {
namespace {

using namespace qt;

struct QuantSmem {
  alignas(1024) uint8_t x[2][2][kBox];  // [stage][channel half] swizzled fp16 tile
  QuantScratch s;
  alignas(8) uint64_t bar[2];
  uint32_t tmem;                         // tensor-memory base of this CTA's R stash
  int it_slot[kQThreads];                // per thread: the index of its next tile iteration
  alignas(8) int64_t slot[2];            // [stage] slot_mapping of the tile's first token
  struct {
    int64_t grp;
    int side, h;
  } coord[2];                            // [stage] the tile's coordinates (written by thread 0)
};

// 8-byte asynchronous copy global -> shared (through L1), in its own commit group
__device__ __forceinline__ void fetch_slot(int64_t* dst, const int64_t* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// A CTA allocates kTmemCols tensor-memory columns once; at most kMaxCtasPerSm
// CTAs share an SM's 512 columns, so the allocation never waits.
constexpr int kMaxCtasPerSm = 512 / kTmemCols;

// TMA load of one tile (two 64-channel boxes) into a stage
__device__ __forceinline__ void load_tile(const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int h, int64_t grp) {
  mbar_arrive_expect_tx(bar, 2 * kBox);
  const int t0 = static_cast<int>(grp * kTile);
  const uint64_t pol = l2_evict_first_policy();   // the fp16 input is read once
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;\n" ::"r"(smem_u32(dst + half * kBox)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(64 * half), "r"(h), "r"(t0), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
  }
}

// tile id -> (side, group, head): K tiles first, then V tiles
__device__ __forceinline__ void tile_coords(const QuantArgs& p, int64_t id, int& side, int64_t& grp, int& h) {
  const int64_t per_side = p.num_groups * p.hkv;
  side = id >= per_side ? 1 : 0;
  const int64_t r = id - side * per_side;
  grp = r / p.hkv;
  h = static_cast<int>(r - grp * p.hkv);
}

template <int KB, int VB>
#ifndef KVARN_Q_MIN_CTAS
#define KVARN_Q_MIN_CTAS 3
#endif
__global__ void __launch_bounds__(kQThreads, KVARN_Q_MIN_CTAS) quantize_kernel(const __grid_constant__ CUtensorMap map_k,
                                                            const __grid_constant__ CUtensorMap map_v,
                                                            const __grid_constant__ QuantArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  QuantSmem& sm = *reinterpret_cast<QuantSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int64_t total = 2 * p.num_groups * p.hkv;
  if (tid == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_barrier_init();
  }
  if (tid < 32) tmem_alloc(&sm.tmem);
  sm.it_slot[tid] = 0;
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  // a programmatic dependent launch: the setup above may overlap the previous
  // kernel in the stream; wait for it before the first global-memory access.
  // No early launch_dependents: the next kernel launches as these CTAs exit
  // (waiting CTAs resident beside running ones slowed the step by 10-20 us).
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  if (blockIdx.x < total && tid == 0) {
    int side, h;
    int64_t grp;
    tile_coords(p, blockIdx.x, side, grp, h);
    load_tile(side ? &map_v : &map_k, sm.x[0][0], &sm.bar[0], h, grp);
    fetch_slot(&sm.slot[0], p.slot_mapping + grp * kTile);
    sm.coord[0].grp = grp;
    sm.coord[0].side = side;
    sm.coord[0].h = h;
  }
  for (;;) {
    // The iteration index goes through shared memory (each thread its own
    // word), so that no loop state stays live in registers across the tile,
    // whose passes need all but a few of them.
    const int it = sm.it_slot[tid];
    sm.it_slot[tid] = it + 1;
    const int64_t id = blockIdx.x + static_cast<int64_t>(it) * gridDim.x;
    if (id >= total) break;
    const int stage = it & 1;
    const int64_t nxt = id + gridDim.x;
    if (nxt < total && tid == 0) {   // the other stage was released at the end of the previous tile
      int side, h;
      int64_t grp;
      tile_coords(p, nxt, side, grp, h);
      load_tile(side ? &map_v : &map_k, sm.x[stage ^ 1][0], &sm.bar[stage ^ 1], h, grp);
      fetch_slot(&sm.slot[stage ^ 1], p.slot_mapping + grp * kTile);
      sm.coord[stage ^ 1].grp = grp;
      sm.coord[stage ^ 1].side = side;
      sm.coord[stage ^ 1].h = h;
    }
    // thread 0: this tile's slot (fetched a tile ago) has landed; the barrier
    // below publishes it to the CTA
    if (tid == 0) {
      if (nxt < total) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
      else asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    }
    // every thread polls; the CTA proceeds only if all saw the copy land
    const bool landed = __syncthreads_and(mbar_wait_bounded(&sm.bar[stage], (it >> 1) & 1)) != 0;
    if (!landed) {
      if (tid == 0) report_status(p.status, KVARN_DEV_TIMEOUT);
      // let the copies still in flight land before the shared memory is released
      (void)mbar_wait_bounded(&sm.bar[stage], (it >> 1) & 1);
      if (nxt < total) (void)mbar_wait_bounded(&sm.bar[stage ^ 1], ((it + 1) >> 1) & 1);
      break;
    }
    // the tile's coordinates and slot, published by the barrier above
    const int side = sm.coord[stage].side, h = sm.coord[stage].h;
    const int64_t grp = sm.coord[stage].grp;
    // which paged block: slot_mapping[128 * grp] must start a block of the pool
    // debug builds: the tile's coordinates lie inside the input
    const bool coords_ok = debug_ok(grp >= 0 && grp < p.num_groups && h >= 0 && h < p.hkv, p.status);
    const int64_t slot = coords_ok ? sm.slot[stage] : -1;
    const int64_t blk = slot >> 7;
    if (!coords_ok) {
      // reported as KVARN_DEV_INTERNAL; nothing is written
    } else if (slot < 0 || (slot & 127) != 0 || blk >= p.num_blocks) {
      if (tid == 0) report_status(p.status, KVARN_DEV_BAD_SLOT);
    } else {
      const uint32_t xs = smem_u32(sm.x[stage][0]);
      if (tid == 0) {   // read inside quantize_tile after its first barrier
        TileOut& o = sm.s.out;
        o.codes = p.packed + (blk * p.hkv + h) * (int64_t)(2048 * (p.kb + p.vb)) + (side == 0 ? 0 : 2048 * p.kb);
        o.scales = p.scales + ((blk * p.hkv + h) * 2 + side) * (int64_t)kScaleRec;
        o.dbg = p.dbg != nullptr ? p.dbg + ((grp * p.hkv + h) * 2 + side) * 256 : nullptr;
      }
      if (side == 0) quantize_tile<0, KB, true>(p.iters, sm.s, xs, sm.tmem);
      else quantize_tile<1, VB, true>(p.iters, sm.s, xs, sm.tmem);
    }
    __syncthreads();   // stage `stage` and the shared scratch are free again
  }
  // every path reaches here with the CTA converged (the timeout break is CTA-uniform)
  if (tid == 0) cp_async_wait_all();   // no slot copy outlives the CTA
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  if (tid < 32) tmem_dealloc(sm.tmem);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [num_tokens][hkv][128] fp16 as a 3-D tensor (channel, head, token); box = 64 channels x 1 head x 128 tokens
cudaError_t make_map(CUtensorMap* m, const __half* base, int hkv, int64_t num_tokens) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(num_tokens)};
  const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(hkv) * 256};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<__half*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// CTAs of `fn` that fit on one SM by registers, shared memory and threads.  The
// runtime's occupancy query answers 1 for any kernel that allocates tensor
// memory, whatever its footprint, so the persistent grid is sized from the
// kernel's own resources instead (the tensor-memory bound is applied by the caller).
cudaError_t resident_ctas(const void* fn, int dyn_smem, int dev, int* out) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  int regs_sm = 0, smem_sm = 0, thr_sm = 0, smem_rsv = 0, ctas_sm = 0;
  if ((e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&ctas_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev)) != cudaSuccess) return e;
  const int warps = (kQThreads + 31) / 32;
  const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;   // allocated per warp in units of 256
  int occ = ctas_sm;
  occ = std::min(occ, regs_sm / std::max(1, regs_warp * warps));
  occ = std::min(occ, smem_sm / std::max(1, static_cast<int>(fa.sharedSizeBytes) + dyn_smem + smem_rsv));
  occ = std::min(occ, thr_sm / kQThreads);
  *out = occ;
  return cudaSuccess;
}

template <int KB, int VB>
cudaError_t launch_q(const QuantArgs& p, cudaStream_t stream) {
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  static int ctas_per_sm[64] = {};
  static int sms[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;   // one configured bit per ordinal
  const uint64_t bit = 1ull << dev;
  const int smem = static_cast<int>(sizeof(QuantSmem));
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(quantize_kernel<KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = resident_ctas(reinterpret_cast<const void*>(quantize_kernel<KB, VB>), smem, dev, &occ);
    if (e != cudaSuccess) return e;
    // each resident CTA holds kTmemCols of the SM's 512 tensor-memory columns
    ctas_per_sm[dev] = occ < 1 ? 1 : (occ > kMaxCtasPerSm ? kMaxCtasPerSm : occ);
    sms[dev] = n;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap mk, mv;
  e = make_map(&mk, p.k, p.hkv, p.num_groups * kTile);
  if (e != cudaSuccess) return e;
  e = make_map(&mv, p.v, p.hkv, p.num_groups * kTile);
  if (e != cudaSuccess) return e;
  const int64_t tiles = 2 * p.num_groups * p.hkv;
  const int64_t slots = static_cast<int64_t>(sms[dev]) * ctas_per_sm[dev];
  const unsigned grid = static_cast<unsigned>(tiles < slots ? tiles : slots);
  return launch_pdl(quantize_kernel<KB, VB>, dim3(grid), dim3(kQThreads), static_cast<size_t>(smem), stream, mk, mv, p);
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs& p, cudaStream_t stream) {
#define KVARN_Q_CASE(KB, VB) \
  if (p.kb == KB && p.vb == VB) return launch_q<KB, VB>(p, stream);
  KVARN_Q_CASE(4, 2)
  KVARN_Q_CASE(2, 2)
  KVARN_Q_CASE(4, 4)
  KVARN_Q_CASE(8, 8)
  KVARN_Q_CASE(2, 4)
  KVARN_Q_CASE(4, 8)
  KVARN_Q_CASE(8, 4)
  KVARN_Q_CASE(8, 2)
  KVARN_Q_CASE(2, 8)
#undef KVARN_Q_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kvarn
