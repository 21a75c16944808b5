// baseline.cu -- uncompressed fp16 / fp8 (e4m3) paged decode attention on
// sm_100a: the measurement baselines the KVarN decode is compared with (the
// pages compare against FP16 and FP8 KV caches: [hypho] "KV-cache 量化终于能跑
// 生产了？KVarN …", section 与 TurboQuant 和 FP8 的实测对比).
//
// Cache layout: [num_blocks][Hkv][128 tokens][128 channels], fp16 or e4m3
// (value = code * k_scale / v_scale); token i of sequence b is row i % 128
// of block block_table[b][i / 128]; the last block may be partial.
//
// Same structure as the KVarN decode: grid (num_splits + 1, Hkv, B) with the
// last split index unused here (kept so both kernels share one geometry),
// 4 warps per CTA, each warp streaming 16-token units through a private
// 2-stage ring filled by the TMA engine (128-byte swizzle), mma.m16n8k16 for
// q.K (A = K rows via ldmatrix) and P.V (A = V^T via ldmatrix.trans), online
// softmax per warp, merge per CTA, and the last CTA of a (seq, KV head)
// combines the splits.  e4m3 tiles go to the tensor cores straight from the
// staged bytes: ldmatrix of 8x8 blocks of byte pairs, widened to fp16 in
// registers (cvt.rn.f16x2.e4m3x2), with the k and m orders of the MMAs
// permuted to match (q is loaded in the same k order, and the output
// channels are mapped back when the warps merge).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kvarn_internal.h"

namespace kvarn {
namespace {

constexpr int kBWarps = 4;
constexpr int kBThreads = 32 * kBWarps;
constexpr int kUnit = 16;                       // tokens per warp work unit
constexpr int kHalf16 = kUnit * 128;            // one 64-channel fp16 box: 16 rows x 128 B

template <int FP8>
struct BaseTraits {
  // fp16: stage = K (2 boxes) + V (2 boxes); fp8: stage = K row tile + V row tile (128 B rows)
  static constexpr int kRaw = FP8 ? 2 * kUnit * 128 : 4 * kHalf16;
  static constexpr int kWarpBytes = 2 * kRaw;
  static constexpr int kBarOff = kBWarps * kWarpBytes;
  static constexpr int kSmem = kBarOff + 64;
};

// byte offset of (row t < 16, 16-byte chunk c16 in 0..15) in a 2-box fp16 tile
__device__ __forceinline__ uint32_t off16(int t, int c16) {
  return (c16 >> 3) * kHalf16 + t * 128 + (((c16 & 7) ^ (t & 7)) << 4);
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
  uint32_t y;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(y) : "h"(x));
  return y;
}
// bytes (i, j) of x as an e4m3 pair (byte i to the low half)
__device__ __forceinline__ uint32_t e4m3_bytes_to_f16x2(uint32_t x, unsigned sel) {
  return e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(x, 0u, sel)));
}

__device__ __forceinline__ void tma_3d(const CUtensorMap* map, void* dst, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

template <int FP8>
__device__ void baseline_split(const BaselineArgs& p, const CUtensorMap* mk, const CUtensorMap* mv, uint8_t* smem,
                               int b, int h, int s, int L) {
  using T = BaseTraits<FP8>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, c = lane & 3;
  const int G = p.G;
  const int n_tiles = (L + kTile - 1) / kTile;          // blocks holding tokens
  const int t_begin = s * p.tiles_per_split;
  const int t_end = min(t_begin + p.tiles_per_split, n_tiles);
  if (t_begin >= t_end) return;
  const int tok_begin = t_begin * kTile;
  const int tok_end = min(t_end * kTile, L);
  const int n_units = (tok_end - tok_begin + kUnit - 1) / kUnit;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff) + warp * 2;
  uint8_t* wbase = smem + warp * T::kWarpBytes;
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_barrier_init();
  }
  __syncwarp();

  // q fragments (B operand of q.K), heads >= G are 0.  fp16: b0 = q[g8][16kt +
  // 2c .. +1], b1 = +8.  fp8: the k slots 2c, 2c+1, 2c+8, 2c+9 of block kt
  // are channels 16kt + 4c .. 4c+3 (the order the e4m3 K fragments arrive in)
  uint32_t qb0[8], qb1[8];
  {
    const __half* qp = p.q + ((int64_t)b * p.Hq + h * G + g8) * kHeadDim;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      const int c0 = FP8 ? 16 * kt + 4 * c : 16 * kt + 2 * c;
      const int c1 = FP8 ? c0 + 2 : c0 + 8;
      qb0[kt] = g8 < G ? *reinterpret_cast<const uint32_t*>(qp + c0) : 0u;
      qb1[kt] = g8 < G ? *reinterpret_cast<const uint32_t*>(qp + c1) : 0u;
    }
  }
  const float sl = p.sm_scale * kLog2e * (FP8 ? p.k_scale : 1.f);
  const float vs = FP8 ? p.v_scale : 1.f;
  const int32_t* btab = p.block_table + (int64_t)b * p.max_blocks;
  const int n_mine = warp < n_units ? (n_units - warp + kBWarps - 1) / kBWarps : 0;

  auto issue = [&](int k) {
    const int u = warp + k * kBWarps;
    const int tok = tok_begin + u * kUnit;
    const int32_t blk = btab[tok >> 7];
    const bool ok = blk >= 0 && blk < p.num_blocks;
    if (lane == 0) {
      uint8_t* dst = wbase + (k & 1) * T::kRaw;
      uint64_t* bar = &bars[k & 1];
      // order this warp's earlier generic writes to the stage (zeroed rows) before the async-proxy refill
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      if (ok) {
        const int plane = blk * p.Hkv + h;
        mbar_arrive_expect_tx(bar, T::kRaw);
        if (FP8) {
          tma_3d(mk, dst, bar, 0, tok & 127, plane);
          tma_3d(mv, dst + kUnit * 128, bar, 0, tok & 127, plane);
        } else {
          tma_3d(mk, dst, bar, 0, tok & 127, plane);
          tma_3d(mk, dst + kHalf16, bar, 64, tok & 127, plane);
          tma_3d(mv, dst + 2 * kHalf16, bar, 0, tok & 127, plane);
          tma_3d(mv, dst + 3 * kHalf16, bar, 64, tok & 127, plane);
        }
      } else {
        report_status(p.status, KVARN_DEV_BAD_BLOCK);
        mbar_arrive_expect_tx(bar, 0);
      }
    }
    return ok;
  };

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[i][r] = 0.f;
  float mrun[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
  bool ok0 = n_mine > 0 ? issue(0) : false;
  bool ok1 = n_mine > 1 ? issue(1) : false;
  int k_fail = -1;

  for (int k = 0; k < n_mine; ++k) {
    const int stg = k & 1;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[stg], (k >> 1) & 1))) {
      if (lane == 0) report_status(p.status, KVARN_DEV_TIMEOUT);
      k_fail = k;
      break;
    }
    const bool ok = stg == 0 ? ok0 : ok1;
    const int tok0 = tok_begin + (warp + k * kBWarps) * kUnit;
    const int valid_rows = min(kUnit, L - tok0);          // rows >= valid_rows are past the sequence
    uint8_t* raw = wbase + stg * T::kRaw;
    if (!FP8 && valid_rows < kUnit) {   // zero V rows past the sequence (cache memory there is arbitrary)
      uint8_t* vt16 = raw + 2 * kHalf16;
      for (int idx = lane; idx < kUnit * 16; idx += 32) {
        const int row = idx >> 4, c16 = idx & 15;
        if (row >= valid_rows) *reinterpret_cast<uint4*>(vt16 + off16(row, c16)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    if (ok) {
      // q.K: 16 tokens x 8 heads, K = 128 channels
      float S[4] = {0.f, 0.f, 0.f, 0.f};
      const int mi = lane >> 3;
      if (FP8) {
        // 8x8 blocks of byte pairs: lanes 0-15 address rows 0-15 of chunk kt,
        // lanes 16-31 of chunk kt + 1; a thread gets channels 4c .. 4c+3 of
        // rows g8 and g8 + 8 of each chunk
        const uint32_t kb8 = smem_u32(raw);
        const int lrow = (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int kt = 0; kt < 8; kt += 2) {
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4(kb8 + lrow * 128 + (((kt + (mi >> 1)) ^ (lrow & 7)) << 4), r0, r1, r2, r3);
          mma_f16(S, e4m3_bytes_to_f16x2(r0, 0x10), e4m3_bytes_to_f16x2(r1, 0x10), e4m3_bytes_to_f16x2(r0, 0x32),
                  e4m3_bytes_to_f16x2(r1, 0x32), qb0[kt], qb1[kt]);
          mma_f16(S, e4m3_bytes_to_f16x2(r2, 0x10), e4m3_bytes_to_f16x2(r3, 0x10), e4m3_bytes_to_f16x2(r2, 0x32),
                  e4m3_bytes_to_f16x2(r3, 0x32), qb0[kt + 1], qb1[kt + 1]);
        }
      } else {
        const uint32_t kb = smem_u32(raw);
        const int arow = (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int kt = 0; kt < 8; ++kt) {
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(kb + off16(arow, 2 * kt + (mi >> 1)), a0, a1, a2, a3);
          mma_f16(S, a0, a1, a2, a3, qb0[kt], qb1[kt]);
        }
      }
      // rows g8 and g8 + 8, heads 2c, 2c+1; log2 units; mask tokens past the sequence
      const bool v0 = g8 < valid_rows, v1 = g8 + 8 < valid_rows;
      S[0] = v0 ? S[0] * sl : -INFINITY;
      S[1] = v0 ? S[1] * sl : -INFINITY;
      S[2] = v1 ? S[2] * sl : -INFINITY;
      S[3] = v1 ? S[3] * sl : -INFINITY;
      float mx0 = fmaxf(S[0], S[2]), mx1 = fmaxf(S[1], S[3]);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(mrun[0], mx0), mn1 = fmaxf(mrun[1], mx1);
      const float al0 = ex2_fast(mrun[0] - mn0), al1 = ex2_fast(mrun[1] - mn1);
      mrun[0] = mn0;
      mrun[1] = mn1;
      const float p0 = ex2_fast(S[0] - mn0), p1 = ex2_fast(S[1] - mn1);
      const float p2 = ex2_fast(S[2] - mn0), p3 = ex2_fast(S[3] - mn1);
      lsum[0] = lsum[0] * al0 + (p0 + p2);
      lsum[1] = lsum[1] * al1 + (p1 + p3);
      const uint32_t bv0 = movmatrix_t(pack_f2h2(p0, p1));
      const uint32_t bv1 = movmatrix_t(pack_f2h2(p2, p3));
      if (FP8) {
        // P.V: A = V^T from ldmatrix.trans of the byte-pair blocks: a thread
        // gets tokens 2c, 2c+1 (and 8 + 2c, 9 + 2c) of channels 2 g8 and
        // 2 g8 + 1 of a chunk, which become the MMA rows g8 and g8 + 8 (the
        // merge maps them back).  V past the sequence is zeroed in registers.
        const uint32_t vb8 = smem_u32(raw + kUnit * 128);
        const int lrow = (lane & 7) + 8 * (mi & 1);
        const uint32_t mlo = (2 * c < valid_rows ? 0xffffu : 0u) | (2 * c + 1 < valid_rows ? 0xffff0000u : 0u);
        const uint32_t mhi = (8 + 2 * c < valid_rows ? 0xffffu : 0u) | (9 + 2 * c < valid_rows ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < 8; mt += 2) {
          uint32_t r0, r1, r2, r3;
          ldmatrix_x4_t(vb8 + lrow * 128 + (((mt + (mi >> 1)) ^ (lrow & 7)) << 4), r0, r1, r2, r3);
          const uint32_t rr[4] = {r0, r1, r2, r3};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const uint32_t lo = rr[2 * h2], hi = rr[2 * h2 + 1];   // tokens 0-7, 8-15 of chunk mt + h2
            float o[4] = {0.f, 0.f, 0.f, 0.f};
            mma_f16(o, e4m3_bytes_to_f16x2(lo, 0x20) & mlo, e4m3_bytes_to_f16x2(lo, 0x31) & mlo,
                    e4m3_bytes_to_f16x2(hi, 0x20) & mhi, e4m3_bytes_to_f16x2(hi, 0x31) & mhi, bv0, bv1);
            float* ac = acc[mt + h2];
            ac[0] = fmaf(ac[0], al0, o[0] * vs);
            ac[1] = fmaf(ac[1], al1, o[1] * vs);
            ac[2] = fmaf(ac[2], al0, o[2] * vs);
            ac[3] = fmaf(ac[3], al1, o[3] * vs);
          }
        }
      } else {
        // P.V: A = V^T (rows channels, k = the 16 tokens) via ldmatrix.trans of the V rows
        const uint32_t vb = smem_u32(raw + 2 * kHalf16);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          // matrices: (tokens 0-7, ch 16mt..+7), (tokens 0-7, ch +8..), (tokens 8-15, ch 16mt..), (8-15, +8)
          const int vrow = (lane & 7) + 8 * (mi >> 1);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_t(vb + off16(vrow, 2 * mt + (mi & 1)), a0, a1, a2, a3);
          float o[4] = {0.f, 0.f, 0.f, 0.f};
          mma_f16(o, a0, a1, a2, a3, bv0, bv1);
          acc[mt][0] = fmaf(acc[mt][0], al0, o[0] * vs);
          acc[mt][1] = fmaf(acc[mt][1], al1, o[1] * vs);
          acc[mt][2] = fmaf(acc[mt][2], al0, o[2] * vs);
          acc[mt][3] = fmaf(acc[mt][3], al1, o[3] * vs);
        }
      }
    }
    __syncwarp();
    if (k + 2 < n_mine) {
      const bool okn = issue(k + 2);
      if (stg == 0) ok0 = okn; else ok1 = okn;
    }
  }
  if (k_fail >= 0) {
    (void)mbar_wait_bounded(&bars[k_fail & 1], (k_fail >> 1) & 1);
    if (k_fail + 1 < n_mine) (void)mbar_wait_bounded(&bars[(k_fail + 1) & 1], ((k_fail + 1) >> 1) & 1);
  }

  // merge the warps (same record format as the KVarN decode, original domain)
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], o);
    lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], o);
  }
  __syncthreads();
  float* mS = reinterpret_cast<float*>(smem);
  float* lS = mS + kBWarps * 8;
  float* aS = lS + kBWarps * 8;
  if (g8 == 0) {
    mS[warp * 8 + 2 * c] = mrun[0];
    mS[warp * 8 + 2 * c + 1] = mrun[1];
    lS[warp * 8 + 2 * c] = lsum[0];
    lS[warp * 8 + 2 * c + 1] = lsum[1];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      // MMA row g8 + 8 ri is channel 16 mt + g8 + 8 ri (fp16) or 16 mt + 2 g8 + ri (fp8)
      const int d = FP8 ? 16 * mt + 2 * g8 + ri : 16 * mt + g8 + 8 * ri;
      aS[(warp * 8 + 2 * c) * kHeadDim + d] = acc[mt][2 * ri];
      aS[(warp * 8 + 2 * c + 1) * kHeadDim + d] = acc[mt][2 * ri + 1];
    }
  __syncthreads();
  const int d = tid;
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kBWarps; ++w) M = fmaxf(M, mS[w * 8 + g]);
    float l = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kBWarps; ++w) {
      const float mw = mS[w * 8 + g];
      const float f = mw == -INFINITY ? 0.f : ex2_fast(mw - M);
      l = fmaf(f, lS[w * 8 + g], l);
      a = fmaf(f, aS[(w * 8 + g) * kHeadDim + d], a);
    }
    float* rec = p.ws + (((int64_t)b * p.Hq + h * G + g) * (p.num_splits + 1) + s) * kPartialFloats;
    if (d == 0) {
      rec[0] = M;
      rec[1] = l;
      rec[2] = 0.f;
      rec[3] = 0.f;
    }
    rec[4 + d] = a;
  }
}

__device__ void baseline_combine(const BaselineArgs& p, int b, int h, int L, bool valid) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int g = warp; g < p.G; g += kBWarps) {
    const int j = h * p.G + g;
    __half* o = p.out + ((int64_t)b * p.Hq + j) * kHeadDim + 4 * lane;
    if (!valid || L == 0) {
      *reinterpret_cast<uint2*>(o) = make_uint2(0u, 0u);
      continue;
    }
    const int n_tiles = (L + kTile - 1) / kTile;
    const int nsv = (n_tiles + p.tiles_per_split - 1) / p.tiles_per_split;
    const float* rec = p.ws + ((int64_t)b * p.Hq + j) * (p.num_splits + 1) * kPartialFloats;
    float M = -INFINITY;
    for (int s = 0; s < nsv; ++s) M = fmaxf(M, __ldcg(rec + (int64_t)s * kPartialFloats));
    float l = 0.f, a[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < nsv; ++s) {
      const float* r = rec + (int64_t)s * kPartialFloats;
      const float w = ex2_fast(__ldcg(r) - M);
      l = fmaf(w, __ldcg(r + 1), l);
      const float4 v = __ldcg(reinterpret_cast<const float4*>(r + 4 + 4 * lane));
      a[0] = fmaf(w, v.x, a[0]);
      a[1] = fmaf(w, v.y, a[1]);
      a[2] = fmaf(w, v.z, a[2]);
      a[3] = fmaf(w, v.w, a[3]);
    }
    const float il = 1.f / l;
    *reinterpret_cast<uint2*>(o) = make_uint2(h2_as_u32(__floats2half2_rn(a[0] * il, a[1] * il)),
                                              h2_as_u32(__floats2half2_rn(a[2] * il, a[3] * il)));
  }
}

template <int FP8>
__global__ void __launch_bounds__(kBThreads) baseline_kernel(const __grid_constant__ CUtensorMap mk,
                                                             const __grid_constant__ CUtensorMap mv,
                                                             const __grid_constant__ BaselineArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int last_arrival;
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int L = p.seq_lens[b];
  const bool valid = L >= 0 && L <= kTile * p.max_blocks;
  if (!valid) {
    if (threadIdx.x == 0 && s == 0) report_status(p.status, KVARN_DEV_BAD_SEQ_LEN);
  } else if (s < p.num_splits) {
    baseline_split<FP8>(p, &mk, &mv, smem, b, h, s, L);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_arrival = atomicAdd(p.counters + (int64_t)b * p.Hkv + h, 1) == p.num_splits;
  __syncthreads();
  if (!last_arrival) return;
  __threadfence();
  baseline_combine(p, b, h, L, valid);
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

// cache [planes = num_blocks * Hkv][128 tokens][128 channels]; box = (64 | 128 channels, 16 tokens, 1 plane)
cudaError_t cache_map(CUtensorMap* m, const void* base, int64_t planes, bool fp8) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[3] = {128, 128, static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {128 * esz, 128 * 128 * esz};
  const cuuint32_t box[3] = {fp8 ? 128u : 64u, static_cast<cuuint32_t>(kUnit), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int FP8>
cudaError_t launch_b(const BaselineArgs& p, cudaStream_t stream) {
  using T = BaseTraits<FP8>;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;   // one configured bit per ordinal
  const uint64_t bit = 1ull << dev;
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    e = cudaFuncSetAttribute(baseline_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  const int64_t planes = (p.num_blocks > 0 ? p.num_blocks : 1) * p.Hkv;
  CUtensorMap mk, mv;
  e = cache_map(&mk, p.k_cache, planes, FP8 != 0);
  if (e != cudaSuccess) return e;
  e = cache_map(&mv, p.v_cache, planes, FP8 != 0);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counters, 0, static_cast<size_t>(p.B) * p.Hkv * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(p.num_splits + 1), static_cast<unsigned>(p.Hkv), static_cast<unsigned>(p.B));
  baseline_kernel<FP8><<<grid, kBThreads, T::kSmem, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_baseline(const BaselineArgs& p, cudaStream_t stream) {
  return p.fp8 ? launch_b<1>(p, stream) : launch_b<0>(p, stream);
}

}  // namespace kvarn
