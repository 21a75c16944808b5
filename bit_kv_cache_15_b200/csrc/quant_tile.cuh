// quant_tile.cuh -- one KVarN tile quantised by one 128-thread CTA (sm_100a).
//
// The four stages of [hypho] "KV-cache 量化终于能跑生产了？KVarN …", section
// 它怎么做到的：四步流水线 (= [lehuy] "KVarN: Backend lượng tử hóa KV-cache …",
// section Cơ chế hoạt động) after the tile is staged in shared memory:
//   2 rotate  R = X H along channels.  H128 = H8 (x) H16 (Kronecker), so the
//             16-channel factor runs on the tensor cores (mma.m16n8k16 against
//             a +-1 fp16 H16) and the 8-group factor is an in-register
//             butterfly across the eight mma results each lane holds;
//   3 normalise  N passes of channel RMS then token RMS in base-2 log space:
//             A = R*R stays in registers; each pass is packed f32x2 FMAs and
//             a sum of the per-thread partials through shared memory
//             (channels: over the 16 threads of the CTA that hold a channel;
//             tokens: over the 8 lanes of a warp that hold a token);
//   4 quantise   Z = (R * fp32(2^-Lt)) * fp32(2^-Lc) from the stored fp16
//             log-scales, one zero/step per tile from min/max, codes =
//             clamp(rne((Z - zero) / step)), the quotient formed in fp32 as
//             Z * (1/step) - zero * (1/step) (one FMA per element);
//   5 pack    codes in the decode's mma fragment order, 16-byte stores.
// The rotation uses H16 as the mma A operand and X as the B operand, so after
// stage 2 each lane holds exactly the elements of the decode kernel's V-side
// mma fragments (rows channels): V codes are packed in registers with no
// cross-lane traffic, and K codes (rows tokens) are packed the same way and
// then moved to the K fragment order by one movmatrix transpose per packed
// 32-bit word.
// Used by the quantise-on-write kernel and by the decode kernel's append path.
#pragma once
#include "common.cuh"
#include "kvarn_internal.h"

namespace kvarn {
namespace qt {

constexpr int kQThreads = 128;
constexpr int kBox = 128 * 128;       // one 64-channel box: 128 rows of 128 bytes

// Row stride (floats) of the channel-pass exchange: 128 + 4, so that the 8
// lanes of a quarter-warp writing 16 bytes each (4 rows x 2 column blocks) hit
// distinct banks.
constexpr int kXchStride = kHeadDim + 4;

// Row stride (floats) of a warp's token-pass exchange (8 rows of 32 partials):
// 32 + 4, so the 16-byte stores of a quarter-warp (2 rows x 4 column blocks)
// and the column reads hit distinct banks.  8 such rows fit in the warp's own
// 4 channel-exchange rows.
constexpr int kTokStride = 32 + 4;
static_assert(8 * kTokStride <= 4 * kXchStride, "token exchange inside the warp's channel rows");

// Where one tile's results go.
struct TileOut {
  uint8_t* codes;        // this side's code block (2048 * BITS bytes, 16-byte aligned)
  uint8_t* scales;       // this side's 528-byte scale record
  float* dbg;            // nullable: fp32 log-scales before rounding (256 floats)
};

// Per-CTA scratch of one tile's normalisation and quantisation.  Channels are
// kept in the permuted order j = g*16 + 2a + ri of channel 16a + g + 8ri (the
// order in which a lane of the register layout holds its 16 channels).
struct QuantScratch {
  union {
    // normalisation: channel partial sums, row (warp, c) x permuted channel;
    // during the token pass, rows 4w .. 4w+3 hold warp w's token partials
    alignas(16) float xch[16 * kXchStride];
    // quantisation (after the last pass)
    struct {
      float mt[kTile];                     // fp32(2^-Lt)
      float mc[kHeadDim];                  // fp32(2^-Lc)
      float zmin[4], zmax[4];
    } q;
  };
  alignas(16) float u[kHeadDim];         // channel weights 2^(-2 lc), permuted order
  alignas(16) float wb[4][32];           // per-warp token-weight exchange
  // Where the tile's results go, written by the caller's thread 0 before
  // quantize_tile and read only after the tile's first CTA barrier: kept here
  // rather than in registers, beside the 128 that hold R^2 during the passes.
  TileOut out;
};

// channel of permuted index j = g*16 + 2a + ri
__device__ __forceinline__ int perm_channel(int j) { return 16 * ((j >> 1) & 7) + (j >> 4) + 8 * (j & 1); }

// Tensor memory can hold a tile's rotated R (fp32, 128 lanes x 128 columns =
// 64 KB) from the rotation until quantisation, so R is computed once.
constexpr int kTmemCols = 128;

// byte offset of (row t, 16-byte chunk c16 in 0..15) inside one stage
__device__ __forceinline__ uint32_t xoff(int t, int c16) {
  return (c16 >> 3) * kBox + t * 128 + (((c16 & 7) ^ (t & 7)) << 4);
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// The weight 2^(-2 l) of a log-scale l = log2_scale(sum): 128 / sum, with the
// same floor.  Used inside the passes, where only the weights are needed; the
// stored log-scales come from log2_scale of the last pass's sums.
__device__ __forceinline__ float weight_of_sum(float sum_sq) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(fmaxf(sum_sq, 4.547473508864641e-13f)));
  return 128.f * r;
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

// The codes of a pair from their magic-add floats (1.5 * 2^23 + rne(y)): the
// magic constant's low 16 bits are 0 and rne(y) lies in [0, 2^BITS - 1], so
// the low 16 bits of each float are its code and one byte permute gives
// code.x | code.y << 16, ready to be shifted into its field of a packed word
// (the fields do not overlap, so adding them is or-ing them).  y is
// (Z - zero) / step for the tile's own min and max; its rounding error stays
// far below 1/2 unless the tile's whole range is below fp32 resolution of its
// offset (|zero / step| >= 2^23), where no fp32 grid can represent the tile.
__device__ __forceinline__ uint32_t pair_codes(float2 r) {
  return __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);
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

// Stages 2-5 for the fp16 tile staged at shared address xs (xoff layout), by
// all 128 threads of the CTA, with `iters` normalisation iterations; results go
// where sm.out says.  STASH: keep R in tensor memory at tmem (this CTA's
// allocation) between the rotation and quantisation; otherwise the rotation is
// run a second time from the staged tile (same arithmetic).
template <int SIDE, int BITS, bool STASH>
__device__ __forceinline__ void quantize_tile(int iters, QuantScratch& sm, uint32_t xs, uint32_t tmem) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const TileOut& o = sm.out;
  const int g = lane >> 2, c = lane & 3;

  // ---- 2. rotate
  float A[128];
  rotate_v(xs, warp, lane, A);
  // stash R in this warp's 32 TMEM lanes (lane field: bits 31..16, column: 15..0)
  const uint32_t tr = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  if (STASH) {
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_st32(tr + 32 * q, A + 32 * q);
    tmem_wait_st();
  }
#pragma unroll
  for (int i = 0; i < 128; i += 2) {
    const float2 s2 = __fmul2_rn(f2(A[i], A[i + 1]), f2(A[i], A[i + 1]));
    A[i] = s2.x;
    A[i + 1] = s2.y;
  }

  // ---- 3. normalise
  constexpr int NT = 8;   // tokens per thread
  float wt[NT];                           // token weights 2^(-2 lt)
#pragma unroll
  for (int i = 0; i < NT; ++i) wt[i] = 1.f;
  float lt_sum = 1.f, lc_sum = 1.f;   // this thread's token / channel sums of the last pass

  for (int it = 0; it < iters; ++it) {
    // channel pass: partial sums over this thread's 8 tokens for its 16
    // channels, to row (warp, c) of the exchange in the permuted order (four
    // 16-byte stores); thread j then sums permuted channel j over the 16 rows
    {
      float* row = sm.xch + (warp * 4 + c) * kXchStride + g * 16;
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        // permuted positions 4*k4 .. 4*k4+3 (a = 2*k4 + (m >> 1), ri = m & 1):
        // four independent chains, interleaved token group by token group
        float2 acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
        for (int ntl = 0; ntl < 4; ++ntl)
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int i = (ntl * 8 + 2 * k4 + (m >> 1)) * 4 + 2 * (m & 1);
            acc[m] = __ffma2_rn(f2(A[i], A[i + 1]), f2(wt[ntl * 2], wt[ntl * 2 + 1]), acc[m]);
          }
        *reinterpret_cast<float4*>(row + 4 * k4) =
            make_float4(acc[0].x + acc[0].y, acc[1].x + acc[1].y, acc[2].x + acc[2].y, acc[3].x + acc[3].y);
      }
    }
    __syncthreads();
    {
      float2 t[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) t[r] = f2(sm.xch[(2 * r) * kXchStride + tid], sm.xch[(2 * r + 1) * kXchStride + tid]);
#pragma unroll
      for (int r = 8; r < 16; r += 2)
        t[(r >> 1) & 3] = __fadd2_rn(t[(r >> 1) & 3], f2(sm.xch[r * kXchStride + tid], sm.xch[(r + 1) * kXchStride + tid]));
      const float2 t01 = __fadd2_rn(t[0], t[1]), t23 = __fadd2_rn(t[2], t[3]);
      const float2 tt = __fadd2_rn(t01, t23);
      lc_sum = tt.x + tt.y;
      sm.u[tid] = weight_of_sum(lc_sum);
    }
    __syncthreads();

    // token pass: one accumulator per token pair, the 16 channel weights read
    // in two halves of 8
    {
      float2 acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};   // index ntl
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float uu[8];   // permuted positions 8*hf .. 8*hf+7 of this lane's 16: a = 4*hf + (k >> 1), ri = k & 1
#pragma unroll
        for (int k4 = 0; k4 < 2; ++k4) {
          const float4 x = *reinterpret_cast<const float4*>(&sm.u[g * 16 + 8 * hf + 4 * k4]);
          uu[4 * k4] = x.x; uu[4 * k4 + 1] = x.y; uu[4 * k4 + 2] = x.z; uu[4 * k4 + 3] = x.w;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
          for (int ntl = 0; ntl < 4; ++ntl) {
            const int a = 4 * hf + (k >> 1), ri = k & 1;
            const int i = (ntl * 8 + a) * 4 + 2 * ri;
            acc[ntl] = __ffma2_rn(f2(A[i], A[i + 1]), f2(uu[k], uu[k]), acc[ntl]);
          }
      }
      const float s[8] = {acc[0].x, acc[0].y, acc[1].x, acc[1].y, acc[2].x, acc[2].y, acc[3].x, acc[3].y};   // index ntl*2 + rj
      // the 8 lanes g = 0..7 of one c hold partials of the same 8 tokens: row
      // g, columns c*8 .. c*8+7 of this warp's own exchange rows (free until
      // its next channel pass); lane (g, c) then sums column c*8 + g, i.e.
      // token (ntl, rj) = (g >> 1, g & 1) of its c
      float* tx = sm.xch + warp * 4 * kXchStride;
      *reinterpret_cast<float4*>(tx + g * kTokStride + c * 8) = make_float4(s[0], s[1], s[2], s[3]);
      *reinterpret_cast<float4*>(tx + g * kTokStride + c * 8 + 4) = make_float4(s[4], s[5], s[6], s[7]);
      __syncwarp();
      const float* col = tx + c * 8 + g;
      float2 t0 = f2(col[0], col[kTokStride]), t1 = f2(col[2 * kTokStride], col[3 * kTokStride]);
      t0 = __fadd2_rn(t0, f2(col[4 * kTokStride], col[5 * kTokStride]));
      t1 = __fadd2_rn(t1, f2(col[6 * kTokStride], col[7 * kTokStride]));
      const float2 tt = __fadd2_rn(t0, t1);
      lt_sum = tt.x + tt.y;
      sm.wb[warp][c * 8 + g] = weight_of_sum(lt_sum);
      __syncwarp();
      const float4 w0 = *reinterpret_cast<const float4*>(&sm.wb[warp][c * 8]);
      const float4 w1 = *reinterpret_cast<const float4*>(&sm.wb[warp][c * 8 + 4]);
      wt[0] = w0.x; wt[1] = w0.y; wt[2] = w0.z; wt[3] = w0.w;
      wt[4] = w1.x; wt[5] = w1.y; wt[6] = w1.z; wt[7] = w1.w;
      __syncwarp();
    }
  }

  // the last token pass's exchange rows overlap the quantisation scratch
  __syncthreads();

  // ---- stored fp16 log-scales and their fp32 multipliers
  const int t_own = 8 * (4 * warp + (lane >> 3)) + 2 * c + ((lane >> 2) & 1);
  const int c_own = perm_channel(tid);
  const float lt_own = log2_scale(lt_sum), lc_own = log2_scale(lc_sum);
  const __half Lt16 = __float2half_rn(lt_own);
  const __half Lc16 = __float2half_rn(lc_own);
  sm.q.mt[t_own] = __double2float_rn(exp2(-static_cast<double>(__half2float(Lt16))));
  sm.q.mc[c_own] = __double2float_rn(exp2(-static_cast<double>(__half2float(Lc16))));
  // the scale record's log-scales, straight from the threads that own them
  // (a warp's token scales fill one 64-byte run)
  reinterpret_cast<__half*>(o.scales)[t_own] = Lt16;
  reinterpret_cast<__half*>(o.scales + 256)[c_own] = Lc16;
  if (o.dbg != nullptr) {
    o.dbg[t_own] = lt_own;
    o.dbg[128 + c_own] = lc_own;
  }
  __syncthreads();

  // ---- 4. quantise: R again (from tensor memory, or recomputed), Z, zero/step, codes
  float Z[128];
  if (STASH) {
#pragma unroll
    for (int q = 0; q < 4; ++q) tmem_ld32(tr + 32 * q, Z + 32 * q);
    tmem_wait_ld();
  } else {
    rotate_v(xs, warp, lane, Z);
  }
  float zlo = 3.402823466e38f, zhi = -3.402823466e38f;
  float2 mtv[4];
#pragma unroll
  for (int ntl = 0; ntl < 4; ++ntl) mtv[ntl] = *reinterpret_cast<const float2*>(&sm.q.mt[8 * (4 * warp + ntl) + 2 * c]);
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      const float mcv = sm.q.mc[16 * a + g + 8 * ri];
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
  const float zl = warp_min(zlo);
  const float zh = warp_max(zhi);
  if (lane == 0) {
    sm.q.zmin[warp] = zl;
    sm.q.zmax[warp] = zh;
  }
  __syncthreads();
  const float zero = fminf(fminf(sm.q.zmin[0], sm.q.zmin[1]), fminf(sm.q.zmin[2], sm.q.zmin[3]));
  const float zmx = fmaxf(fmaxf(sm.q.zmax[0], sm.q.zmax[1]), fmaxf(sm.q.zmax[2], sm.q.zmax[3]));
  constexpr int LB = (1 << BITS) - 1;
  float step = __fdiv_rn(__fsub_rn(zmx, zero), static_cast<float>(LB));
  if (step == 0.f) step = 1.f;
  const float inv = __fdiv_rn(1.f, step);
  const float nzi = -zero * inv;

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
      // index of the (h = 0) element, h = 1 is idx + 1; bl = (ntl>>1)*8 + a,
      // j = ri + 2*(ntl&1), h = rj
      const int ntl = 2 * (bl >> 3) + (j >> 1), a = bl & 7, ri = j & 1;
      const int idx = (ntl * 8 + a) * 4 + 2 * ri;
      const float2 y = __ffma2_rn(f2(Z[idx], Z[idx + 1]), f2(inv, inv), f2(nzi, nzi));
      const float2 r = __fadd2_rn(y, f2(kMagic, kMagic));
      // 0 <= y <= 2^b - 1 up to rounding, so rne(y) sits in the low BITS bits of r
      if (SIDE == 0) {
        // K codes held in the V layout: this lane has (channel g, tokens 2c, 2c+1)
        // of an 8x8 block; the K fragment wants (token g, channels 2c, 2c+1),
        // in K register j' = (token half) + 2 (channel half) = (j >> 1) + 2 (j & 1).
        // The codes go to their K-word bit fields here and each word is
        // transposed once below.
        const int rk = 4 * bl + (j >> 1) + 2 * (j & 1);
        words[rk / PER] += pair_codes(r) << (BITS * (rk % PER));
      } else {
        const int rho = 4 * bl + j;
        words[rho / PER] += pair_codes(r) << (BITS * (rho % PER));
      }
    }

  if (SIDE == 0) {
    // The transpose of an 8x8 block of 16-bit elements moves every element by
    // the same lane permutation, whatever block it belongs to, so one
    // transpose per word carries all the code fields packed into it (up to 8
    // blocks' worth) to their K-fragment lanes and halves.
#pragma unroll
    for (int i = 0; i < NW; ++i) words[i] = movmatrix_t(words[i]);
  }

  // ---- 5. store codes (16-byte chunks, lane-interleaved) and the scale record
  uint8_t* dst = o.codes;
#pragma unroll
  for (int cc = 0; cc < BITS; ++cc) {
    const uint4 v4 = make_uint4(words[4 * cc], words[4 * cc + 1], words[4 * cc + 2], words[4 * cc + 3]);
    *reinterpret_cast<uint4*>(dst + ((warp * BITS + cc) * 32 + lane) * 16) = v4;
  }
  if (tid == 0) *reinterpret_cast<float4*>(o.scales + 512) = make_float4(zero, step, 0.f, 0.f);
}

}  // namespace qt
}  // namespace kvarn
