// quantize.cu -- KVarN quantise-on-write for whole 128-token tiles (sm_100a).
//
// The four stages of [hypho] "KV-cache 量化终于能跑生产了？KVarN …", section
// 它怎么做到的：四步流水线 (= [lehuy] "KVarN: Backend lượng tử hóa KV-cache …",
// section Cơ chế hoạt động), one (token group, KV head, K|V) tile at a time:
//   1 stage   the fp16 tile is brought into shared memory by the TMA engine
//             (cp.async.bulk.tensor, two 64-channel boxes, 128-byte swizzle so
//             ldmatrix reads are conflict-free).  CTAs are persistent and load
//             the next tile while they compute the current one;
//   2 rotate  R = X H along channels.  H128 = H8 (x) H16 (Kronecker), so the
//             16-channel factor runs on the tensor cores (mma.m16n8k16 against
//             a +-1 fp16 H16) and the 8-group factor is an in-register
//             butterfly across the eight mma results each lane holds;
//   3 normalise  N passes of channel RMS then token RMS in base-2 log space:
//             A = R*R stays in registers; each pass is packed f32x2 FMAs, a
//             warp reduce-scatter and (for channels) a 4-warp shared sum;
//   4 quantise   Z = (R * fp32(2^-Lt)) * fp32(2^-Lc) from the stored fp16
//             log-scales, one zero/step per tile from min/max, codes =
//             clamp(rne((Z - zero) * (1/step))).
// The K-side rotation uses X as the mma A operand and the V side as the B
// operand, so after stage 2 each lane holds exactly the elements of the
// decode kernel's mma fragments (K: rows tokens; V: rows channels): codes are
// packed in registers and written with 16-byte stores, no cross-lane traffic.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kvarn_internal.h"

namespace kvarn {
namespace {

constexpr int kQThreads = 128;
constexpr int kBox = 128 * 128;       // one 64-channel box: 128 rows of 128 bytes

struct QuantSmem {
  alignas(1024) uint8_t x[2][2][kBox];  // [stage][channel half] swizzled fp16 tile
  float red[4][kHeadDim];                // per-warp channel partial sums
  float u[kHeadDim];                     // channel weights 2^(-2 lc)
  float mt[kTile];                       // fp32(2^-Lt)
  float mc[kHeadDim];                    // fp32(2^-Lc)
  float zmin[4], zmax[4];
  alignas(16) uint8_t rec[kScaleRec];    // staged scale record
  alignas(8) uint64_t bar[2];
  uint32_t tmem;                         // tensor-memory base of this CTA's R stash
};

// Tensor memory holds each tile's rotated R (fp32, 128 lanes x 128 columns =
// 64 KB) from the rotation until quantisation, so R is computed once.  A CTA
// allocates kTmemCols columns once; at most kMaxCtasPerSm CTAs share an SM's
// 512 columns, so the allocation never waits.
constexpr int kTmemCols = 128;
constexpr int kMaxCtasPerSm = 512 / kTmemCols;

// byte offset of (row t, 16-byte chunk c16 in 0..15) inside one stage
__device__ __forceinline__ uint32_t xoff(int t, int c16) {
  return (c16 >> 3) * kBox + t * 128 + (((c16 & 7) ^ (t & 7)) << 4);
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// 1/2 log2 of the mean square (sum / 128), floored at 2^-48
__device__ __forceinline__ float log2_scale(float sum_sq) {
  return 0.5f * (lg2_approx(fmaxf(sum_sq, 4.547473508864641e-13f)) - 7.0f);   // 2^-41
}

// fp16 bit pattern of the Hadamard sign H16[r][c] = (-1)^popcount(r & c).
__device__ __forceinline__ uint32_t h16_bits(int r, int c) {
  return (__popc(r & c) & 1) ? 0xBC00u : 0x3C00u;
}
__device__ __forceinline__ uint32_t h16_pair(int r0, int c0, int r1, int c1) {
  return h16_bits(r0, c0) | (h16_bits(r1, c1) << 16);
}

// In-register 8-point Walsh-Hadamard transforms (Sylvester order) of two
// independent vectors at once: lane .x of v is one vector, lane .y the other.
__device__ __forceinline__ void fwht8x2(float2 (&v)[8]) {
#pragma unroll
  for (int hl = 1; hl < 8; hl <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & hl) == 0) {
        const float2 a = v[i], b = v[i + hl];
        v[i] = __fadd2_rn(a, b);
        v[i + hl] = __fadd2_rn(a, make_float2(-b.x, -b.y));
      }
    }
  }
}

// One reduce-scatter step across lanes (lane ^ mask): the first N/2 entries
// of v end up holding the half this lane keeps, summed with its partner's.
template <int N>
__device__ __forceinline__ void rs_step(float* v, int mask, int lane) {
  const bool up = (lane & mask) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = up ? v[i] : v[i + N / 2];
    const float keep = up ? v[i + N / 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
  }
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ float min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// insert the low `len` bits of x into y at bit `pos`
__device__ __forceinline__ uint32_t bfi(uint32_t x, uint32_t y, int pos, int len) {
  uint32_t r;
  asm("bfi.b32 %0, %1, %2, %3, %4;\n" : "=r"(r) : "r"(x), "r"(y), "r"(pos), "r"(len));
  return r;
}

// ------------------------------------------------------------ tensor memory

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem) {   // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst_smem)),
               "n"(kTmemCols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base) {     // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(base), "n"(kTmemCols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// 32 consecutive columns of this thread's lane <-> v[0..31]
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
      "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]),
      "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]),
      "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]), "=f"(v[8]),
        "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15]), "=f"(v[16]),
        "=f"(v[17]), "=f"(v[18]), "=f"(v[19]), "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]),
        "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// ---------------------------------------------------------------- rotation

// K side: thread holds R at t = 16*(2w+ml) + g + 8*ri, d = 16*a + 8*nb + 2*c + rj
// in R[((ml*8 + a)*2 + nb)*4 + 2*ri + rj]   (g = lane/4, c = lane%4).
__device__ __forceinline__ void rotate_k(uint32_t xs, int warp, int lane, float (&R)[128]) {
  const int g = lane >> 2, c = lane & 3;
  uint32_t hb0[2], hb1[2];
#pragma unroll
  for (int nb = 0; nb < 2; ++nb) {
    const int n = 8 * nb + g;
    hb0[nb] = h16_pair(2 * c, n, 2 * c + 1, n);
    hb1[nb] = h16_pair(2 * c + 8, n, 2 * c + 9, n);
  }
  const int mi = lane >> 3;
#pragma unroll
  for (int ml = 0; ml < 2; ++ml) {
    const int row = 16 * (2 * warp + ml) + (lane & 7) + 8 * (mi & 1);
    float C[8][2][4];
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(xs + xoff(row, 2 * a + (mi >> 1)), a0, a1, a2, a3);
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
        for (int r = 0; r < 4; ++r) C[a][nb][r] = 0.f;
        mma_f16(C[a][nb], a0, a1, a2, a3, hb0[nb], hb1[nb]);
      }
    }
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
      for (int r = 0; r < 4; r += 2) {
        float2 v[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) v[a] = make_float2(C[a][nb][r], C[a][nb][r + 1]);
        fwht8x2(v);
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          R[((ml * 8 + a) * 2 + nb) * 4 + r] = v[a].x;
          R[((ml * 8 + a) * 2 + nb) * 4 + r + 1] = v[a].y;
        }
      }
    }
  }
}

// V side: thread holds R at t = 8*(4w+ntl) + 2*c + rj, d = 16*a + g + 8*ri
// in R[(ntl*8 + a)*4 + 2*ri + rj].
__device__ __forceinline__ void rotate_v(uint32_t xs, int warp, int lane, float (&R)[128]) {
  const int g = lane >> 2, c = lane & 3;
  const uint32_t ha0 = h16_pair(g, 2 * c, g, 2 * c + 1);
  const uint32_t ha1 = h16_pair(g + 8, 2 * c, g + 8, 2 * c + 1);
  const uint32_t ha2 = h16_pair(g, 2 * c + 8, g, 2 * c + 9);
  const uint32_t ha3 = h16_pair(g + 8, 2 * c + 8, g + 8, 2 * c + 9);
  const int mi = lane >> 3;
#pragma unroll
  for (int ntl = 0; ntl < 4; ++ntl) {
    const int row = 8 * (4 * warp + ntl) + (lane & 7);
    float C[8][4];
#pragma unroll
    for (int ap = 0; ap < 4; ++ap) {
      uint32_t r0, r1, r2, r3;
      ldmatrix_x4(xs + xoff(row, 4 * ap + mi), r0, r1, r2, r3);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        C[2 * ap][r] = 0.f;
        C[2 * ap + 1][r] = 0.f;
      }
      mma_f16(C[2 * ap], ha0, ha1, ha2, ha3, r0, r1);
      mma_f16(C[2 * ap + 1], ha0, ha1, ha2, ha3, r2, r3);
    }
#pragma unroll
    for (int r = 0; r < 4; r += 2) {
      float2 v[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) v[a] = make_float2(C[a][r], C[a][r + 1]);
      fwht8x2(v);
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        R[(ntl * 8 + a) * 4 + r] = v[a].x;
        R[(ntl * 8 + a) * 4 + r + 1] = v[a].y;
      }
    }
  }
}

// ---------------------------------------------------------------- the tile

template <int SIDE, int BITS>
__device__ __forceinline__ void quantize_tile(const QuantArgs& p, QuantSmem& sm, uint32_t xs, int64_t grp, int h,
                                              int64_t blk) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;

  // ---- 2. rotate
  float A[128];
  if (SIDE == 0) rotate_k(xs, warp, lane, A); else rotate_v(xs, warp, lane, A);
  // stash R in this warp's 32 TMEM lanes (lane field: bits 31..16, column: 15..0)
  const uint32_t tr = sm.tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_st32(tr + 32 * q, A + 32 * q);
  tmem_wait_st();
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float2 s2 = __fmul2_rn(f2(A[i], A[i + 1]), f2(A[i], A[i + 1]));
    A[i] = s2.x;
    A[i + 1] = s2.y;
  }

  // ---- 3. normalise
  constexpr int NT = SIDE == 0 ? 4 : 8;   // tokens per thread
  float wt[NT];                           // token weights 2^(-2 lt)
#pragma unroll
  for (int i = 0; i < NT; ++i) wt[i] = 1.f;
  float lt_own = 0.f, lc_own = 0.f;

  for (int it = 0; it < p.iters; ++it) {
    // channel pass: partial sums over this thread's tokens
    if (SIDE == 0) {
      float s[32];   // index a*4 + nb*2 + rj
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          float2 acc = f2(0.f, 0.f);
#pragma unroll
          for (int ml = 0; ml < 2; ++ml)
#pragma unroll
            for (int ri = 0; ri < 2; ++ri) {
              const int i = ((ml * 8 + a) * 2 + nb) * 4 + 2 * ri;
              const float w = wt[ml * 2 + ri];
              acc = __ffma2_rn(f2(A[i], A[i + 1]), f2(w, w), acc);
            }
          s[a * 4 + nb * 2] = acc.x;
          s[a * 4 + nb * 2 + 1] = acc.y;
        }
      rs_step<32>(s, 16, lane);
      rs_step<16>(s, 8, lane);
      rs_step<8>(s, 4, lane);
      *reinterpret_cast<float2*>(&sm.red[warp][16 * g + 2 * c]) = f2(s[0], s[1]);
      *reinterpret_cast<float2*>(&sm.red[warp][16 * g + 8 + 2 * c]) = f2(s[2], s[3]);
    } else {
      float s[16];   // index a*2 + ri
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          float2 acc = f2(0.f, 0.f);
#pragma unroll
          for (int ntl = 0; ntl < 4; ++ntl) {
            const int i = (ntl * 8 + a) * 4 + 2 * ri;
            acc = __ffma2_rn(f2(A[i], A[i + 1]), f2(wt[ntl * 2], wt[ntl * 2 + 1]), acc);
          }
          s[a * 2 + ri] = acc.x + acc.y;
        }
      rs_step<16>(s, 2, lane);
      rs_step<8>(s, 1, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int a = 2 * c + (k >> 1), ri = k & 1;
        sm.red[warp][16 * a + g + 8 * ri] = s[k];
      }
    }
    __syncthreads();
    {
      const float tot = (sm.red[0][tid] + sm.red[1][tid]) + (sm.red[2][tid] + sm.red[3][tid]);
      lc_own = log2_scale(tot);
      sm.u[tid] = ex2_fast(-2.f * lc_own);
    }
    __syncthreads();

    // token pass
    if (SIDE == 0) {
      float2 uu[16];   // (a, nb) -> channels 16a + 8nb + 2c + {0,1}
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
          uu[a * 2 + nb] = *reinterpret_cast<const float2*>(&sm.u[16 * a + 8 * nb + 2 * c]);
      float s[4];    // index ml*2 + ri
#pragma unroll
      for (int ml = 0; ml < 2; ++ml)
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          float2 acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};   // 4 chains for ILP
#pragma unroll
          for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              const int i = ((ml * 8 + a) * 2 + nb) * 4 + 2 * ri;
              acc[(a & 1) * 2 + nb] = __ffma2_rn(f2(A[i], A[i + 1]), uu[a * 2 + nb], acc[(a & 1) * 2 + nb]);
            }
          const float2 t01 = __fadd2_rn(acc[0], acc[1]), t23 = __fadd2_rn(acc[2], acc[3]);
          const float2 t = __fadd2_rn(t01, t23);
          s[ml * 2 + ri] = t.x + t.y;
        }
      rs_step<4>(s, 2, lane);
      rs_step<2>(s, 1, lane);
      lt_own = log2_scale(s[0]);
      const float wown = ex2_fast(-2.f * lt_own);
#pragma unroll
      for (int k = 0; k < 4; ++k) wt[k] = __shfl_sync(0xffffffffu, wown, (lane & ~3) | k);
    } else {
      float uu[16];
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) uu[a * 2 + ri] = sm.u[16 * a + g + 8 * ri];
      float s[8];    // index ntl*2 + rj
#pragma unroll
      for (int ntl = 0; ntl < 4; ++ntl) {
        float2 acc[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};   // 2 chains for ILP
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int ri = 0; ri < 2; ++ri) {
            const int i = (ntl * 8 + a) * 4 + 2 * ri;
            const float uv = uu[a * 2 + ri];
            acc[ri] = __ffma2_rn(f2(A[i], A[i + 1]), f2(uv, uv), acc[ri]);
          }
        const float2 t = __fadd2_rn(acc[0], acc[1]);
        s[ntl * 2] = t.x;
        s[ntl * 2 + 1] = t.y;
      }
      rs_step<8>(s, 16, lane);
      rs_step<4>(s, 8, lane);
      rs_step<2>(s, 4, lane);
      lt_own = log2_scale(s[0]);
      const float wown = ex2_fast(-2.f * lt_own);
#pragma unroll
      for (int k = 0; k < 8; ++k) wt[k] = __shfl_sync(0xffffffffu, wown, c | (k << 2));
    }
  }

  // ---- stored fp16 log-scales and their fp32 multipliers
  const int t_own = (SIDE == 0) ? 16 * (2 * warp + ((lane >> 1) & 1)) + g + 8 * (lane & 1)
                                : 8 * (4 * warp + (lane >> 3)) + 2 * c + ((lane >> 2) & 1);
  const __half Lt16 = __float2half_rn(lt_own);
  const __half Lc16 = __float2half_rn(lc_own);
  sm.mt[t_own] = __double2float_rn(exp2(-static_cast<double>(__half2float(Lt16))));
  sm.mc[tid] = __double2float_rn(exp2(-static_cast<double>(__half2float(Lc16))));
  reinterpret_cast<__half*>(sm.rec)[t_own] = Lt16;
  reinterpret_cast<__half*>(sm.rec + 256)[tid] = Lc16;
  if (p.dbg != nullptr) {
    float* d = p.dbg + ((grp * p.hkv + h) * 2 + SIDE) * 256;
    d[t_own] = lt_own;
    d[128 + tid] = lc_own;
  }
  __syncthreads();

  // ---- 4. quantise: R back from tensor memory, Z, zero/step, codes
  float Z[128];
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld32(tr + 32 * q, Z + 32 * q);
  tmem_wait_ld();
  float zlo = 3.402823466e38f, zhi = -3.402823466e38f;
  if (SIDE == 0) {
    float mtv[4];
#pragma unroll
    for (int ml = 0; ml < 2; ++ml)
#pragma unroll
      for (int ri = 0; ri < 2; ++ri) mtv[ml * 2 + ri] = sm.mt[16 * (2 * warp + ml) + g + 8 * ri];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        const float2 mc2 = *reinterpret_cast<const float2*>(&sm.mc[16 * a + 8 * nb + 2 * c]);
#pragma unroll
        for (int ml = 0; ml < 2; ++ml)
#pragma unroll
          for (int ri = 0; ri < 2; ++ri) {
            const int i = ((ml * 8 + a) * 2 + nb) * 4 + 2 * ri;
            const float m = mtv[ml * 2 + ri];
            const float2 z = __fmul2_rn(__fmul2_rn(f2(Z[i], Z[i + 1]), f2(m, m)), mc2);
            Z[i] = z.x;
            Z[i + 1] = z.y;
            zlo = min3(zlo, z.x, z.y);
            zhi = max3(zhi, z.x, z.y);
          }
      }
  } else {
    float2 mtv[4];
#pragma unroll
    for (int ntl = 0; ntl < 4; ++ntl) mtv[ntl] = *reinterpret_cast<const float2*>(&sm.mt[8 * (4 * warp + ntl) + 2 * c]);
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int ri = 0; ri < 2; ++ri) {
        const float mcv = sm.mc[16 * a + g + 8 * ri];
#pragma unroll
        for (int ntl = 0; ntl < 4; ++ntl) {
          const int i = (ntl * 8 + a) * 4 + 2 * ri;
          const float2 z = __fmul2_rn(__fmul2_rn(f2(Z[i], Z[i + 1]), mtv[ntl]), f2(mcv, mcv));
          Z[i] = z.x;
          Z[i + 1] = z.y;
          zlo = min3(zlo, z.x, z.y);
          zhi = max3(zhi, z.x, z.y);
        }
      }
  }
  const float zl = warp_min(zlo);
  const float zh = warp_max(zhi);
  if (lane == 0) {
    sm.zmin[warp] = zl;
    sm.zmax[warp] = zh;
  }
  __syncthreads();
  const float zero = fminf(fminf(sm.zmin[0], sm.zmin[1]), fminf(sm.zmin[2], sm.zmin[3]));
  const float zmx = fmaxf(fmaxf(sm.zmax[0], sm.zmax[1]), fmaxf(sm.zmax[2], sm.zmax[3]));
  constexpr int LB = (1 << BITS) - 1;
  float step = __fdiv_rn(__fsub_rn(zmx, zero), static_cast<float>(LB));
  if (step == 0.f) step = 1.f;
  const float inv = __fdiv_rn(1.f, step);

  // codes: y = (Z - zero) * inv >= 0, rounded to nearest even by adding 1.5 * 2^23
  // (exact for y < 2^22); packed in the fragment order (block bl, register j, half h)
  constexpr int PER = 16 / BITS;          // register pairs per 32-bit word
  constexpr int NW = 64 / PER;            // words per thread (= 4*BITS)
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  uint32_t words[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) words[i] = 0u;
#pragma unroll
  for (int bl = 0; bl < 16; ++bl)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int idx;                             // index of the (h = 0) element; h = 1 is idx + 1
      if (SIDE == 0) {   // bl = ml*8 + a;  j = ri + 2*nb;  h = rj
        const int ml = bl >> 3, a = bl & 7, nb = j >> 1, ri = j & 1;
        idx = ((ml * 8 + a) * 2 + nb) * 4 + 2 * ri;
      } else {           // bl = (ntl>>1)*8 + a;  j = ri + 2*(ntl&1);  h = rj
        const int ntl = 2 * (bl >> 3) + (j >> 1), a = bl & 7, ri = j & 1;
        idx = (ntl * 8 + a) * 4 + 2 * ri;
      }
      const float2 y = __fmul2_rn(__fadd2_rn(f2(Z[idx], Z[idx + 1]), f2(-zero, -zero)), f2(inv, inv));
      const float2 r = __fadd2_rn(y, f2(kMagic, kMagic));
      // 0 <= y <= 2^b - 1 up to rounding, so rne(y) sits in the low BITS bits of r
      const int rho = 4 * bl + j;
      words[rho / PER] = bfi(__float_as_uint(r.x), words[rho / PER], BITS * (rho % PER), BITS);
      words[rho / PER] = bfi(__float_as_uint(r.y), words[rho / PER], BITS * (rho % PER) + 16, BITS);
    }

  // ---- 5. store codes (16-byte chunks, lane-interleaved) and the scale record
  uint8_t* dst = p.packed + (blk * p.hkv + h) * (int64_t)(2048 * (p.kb + p.vb)) + (SIDE == 0 ? 0 : 2048 * p.kb);
#pragma unroll
  for (int cc = 0; cc < BITS; ++cc) {
    const uint4 v4 = make_uint4(words[4 * cc], words[4 * cc + 1], words[4 * cc + 2], words[4 * cc + 3]);
    *reinterpret_cast<uint4*>(dst + ((warp * BITS + cc) * 32 + lane) * 16) = v4;
  }
  if (tid == 0) {
    float* tailp = reinterpret_cast<float*>(sm.rec + 512);
    tailp[0] = zero;
    tailp[1] = step;
    tailp[2] = 0.f;
    tailp[3] = 0.f;
  }
  __syncthreads();
  if (tid < kScaleRec / 16) {
    uint8_t* sdst = p.scales + ((blk * p.hkv + h) * 2 + SIDE) * (int64_t)kScaleRec;
    *reinterpret_cast<uint4*>(sdst + tid * 16) = *reinterpret_cast<const uint4*>(sm.rec + tid * 16);
  }
}

// TMA load of one tile (two 64-channel boxes) into a stage
__device__ __forceinline__ void load_tile(const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int h, int64_t grp) {
  mbar_arrive_expect_tx(bar, 2 * kBox);
  const int t0 = static_cast<int>(grp * kTile);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(smem_u32(dst + half * kBox)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(64 * half), "r"(h), "r"(t0), "r"(smem_u32(bar))
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
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  int64_t id = blockIdx.x;
  if (id < total && tid == 0) {
    int side, h;
    int64_t grp;
    tile_coords(p, id, side, grp, h);
    load_tile(side ? &map_v : &map_k, sm.x[0][0], &sm.bar[0], h, grp);
  }
  for (int it = 0; id < total; ++it, id += gridDim.x) {
    const int stage = it & 1;
    const int64_t nxt = id + gridDim.x;
    if (nxt < total && tid == 0) {   // the other stage was released at the end of the previous tile
      int side, h;
      int64_t grp;
      tile_coords(p, nxt, side, grp, h);
      load_tile(side ? &map_v : &map_k, sm.x[stage ^ 1][0], &sm.bar[stage ^ 1], h, grp);
    }
    int side, h;
    int64_t grp;
    tile_coords(p, id, side, grp, h);
    // every thread polls; the CTA proceeds only if all saw the copy land
    const bool landed = __syncthreads_and(mbar_wait_bounded(&sm.bar[stage], (it >> 1) & 1)) != 0;
    if (!landed) {
      if (tid == 0) report_status(p.status, KVARN_DEV_TIMEOUT);
      // let the copies still in flight land before the shared memory is released
      (void)mbar_wait_bounded(&sm.bar[stage], (it >> 1) & 1);
      if (nxt < total) (void)mbar_wait_bounded(&sm.bar[stage ^ 1], ((it + 1) >> 1) & 1);
      break;
    }
    // which paged block: slot_mapping[128 * grp] must start a block of the pool
    const int64_t slot = p.slot_mapping[grp * kTile];
    const int64_t blk = slot >> 7;
    if (slot < 0 || (slot & 127) != 0 || blk >= p.num_blocks) {
      if (tid == 0) report_status(p.status, KVARN_DEV_BAD_SLOT);
    } else {
      const uint32_t xs = smem_u32(sm.x[stage][0]);
      if (side == 0) quantize_tile<0, KB>(p, sm, xs, grp, h, blk);
      else quantize_tile<1, VB>(p, sm, xs, grp, h, blk);
    }
    __syncthreads();   // stage `stage` and the shared scratch are free again
  }
  // every path reaches here with the CTA converged (the timeout break is CTA-uniform)
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
  const uint64_t bit = 1ull << (dev & 63);
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
    ctas_per_sm[dev & 63] = occ < 1 ? 1 : (occ > kMaxCtasPerSm ? kMaxCtasPerSm : occ);
    sms[dev & 63] = n;
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap mk, mv;
  e = make_map(&mk, p.k, p.hkv, p.num_groups * kTile);
  if (e != cudaSuccess) return e;
  e = make_map(&mv, p.v, p.hkv, p.num_groups * kTile);
  if (e != cudaSuccess) return e;
  const int64_t tiles = 2 * p.num_groups * p.hkv;
  const int64_t slots = static_cast<int64_t>(sms[dev & 63]) * ctas_per_sm[dev & 63];
  const unsigned grid = static_cast<unsigned>(tiles < slots ? tiles : slots);
  quantize_kernel<KB, VB><<<grid, kQThreads, smem, stream>>>(mk, mv, p);
  return cudaGetLastError();
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
