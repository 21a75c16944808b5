// decode.cu -- KVarN paged decode attention on the packed cache (sm_100a).
//
// Scales are folded in on read ([lehuy] "KVarN: Backend lượng tử hóa KV-cache
// …", section Cơ chế hoạt động stage 4; [hypho] "KV-cache 量化终于能跑生产了？
// KVarN …", section 它怎么做到的：四步流水线 step 4).  For sequence b, KV head
// h and the G = Hq/Hkv query heads that read it, tile i with stored codes c,
// log-scales Lt/Lc and grid zero/step contributes
//   score_t = sm_scale/128 * 2^Lt_k[t] * (zero_k * sum_d q'_d + step_k * q'.c_t),
//             q'_d = (q H)_d * 2^Lc_k[d]                       (key side)
//   acc_d  += 2^Lc_v[d] * (zero_v * sum_t p'_t + step_v * sum_t p'_t c_td),
//             p'_t = p_t * 2^Lt_v[t]                            (value side)
// and the output is (acc H / 128 + tail part) / l.
//
// Work split (stream-K): every (sequence, KV head) pair contributes its full
// tiles plus one tail unit; the units, in (sequence, head, tile) order, are
// cut into equal contiguous ranges, one per CTA of a grid of two CTAs per SM.
// A CTA decodes each run of one pair's tiles in its range with all 4 warps
// (units round-robin over the warps, each warp running its own online
// softmax, merged into one partial record per query head) and attends a
// tail unit in its range exactly in the unrotated domain.  A second,
// dependent grid (two CTAs per pair, a programmatic dependent launch) merges
// each pair's records and applies H / 128 once the decode grid has
// completed.  Each warp streams its tiles through a private 2-stage
// shared-memory ring filled by bulk copies (cp.async.bulk on the TMA engine).
// Codes are laid out in the mma fragment order, so a lane's 16-byte shared
// loads are its operands; each masked code pair is already an f16x2 of exact
// subnormals.  Both
// contractions run on the tensor cores (mma.m16n8k16, fp32 accumulate): K
// side rows = tokens, N = the 8 query heads; V side rows = channels, N =
// heads, with the softmax weights moved from accumulator to operand layout
// by movmatrix.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "kvarn_internal.h"
#include "quant_tile.cuh"

namespace kvarn {
namespace {

#ifndef KVARN_D_U_SMALL
#define KVARN_D_U_SMALL 1      // work units per tile when kb + vb <= 6
#endif
#ifndef KVARN_D_MIN_CTAS
#define KVARN_D_MIN_CTAS 2
#endif

constexpr int kDWarps = 4;
constexpr int kDThreads = 32 * kDWarps;
constexpr int kDStages = 2;
constexpr int kMaxG = 8;

// A warp's work unit is 128/U tokens of one tile; U grows with the code size
// so that 4 warps x 2 stages stay near 110 KB (two CTAs per SM).
template <int KB, int VB>
struct DecodeTraits {
  static constexpr int kCodeK = 2048 * KB;
  static constexpr int kCodeV = 2048 * VB;
  static constexpr int kCode = kCodeK + kCodeV;
  static constexpr int U = (KB + VB) <= 6 ? KVARN_D_U_SMALL : ((KB + VB) <= 12 ? 2 : 4);
  static constexpr int MT = 8 / U;                    // 16-token blocks per unit
  static constexpr int kUnitK = kCodeK / U;
  static constexpr int kUnitV = kCodeV / U;
  static constexpr int kStage = kUnitK + kUnitV + 2 * kScaleRec;
  static constexpr int kBarOff = kDWarps * kDStages * kStage;
  static constexpr int kQrotOff = kBarOff + 128;
  static constexpr int kScrOff = kQrotOff + kMaxG * kHeadDim * 4;
  static constexpr int kInvSigOff = kScrOff + kDWarps * kHeadDim * 4;
  // the per-warp token-scale scratch (1 KB) sits inside the q H buffer, which
  // is free once every warp holds q H in registers
  static constexpr int kSmem = kInvSigOff + 64;
  static_assert(kStage % 16 == 0, "stage must stay 16-byte aligned");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kDWarps * kDStages * 8 <= 128, "barrier area");
  // the append path stages a 32 KB fp16 tile and the quantiser scratch below the barriers
  static_assert(kBarOff >= 2 * qt::kBox + static_cast<int>(sizeof(qt::QuantScratch)), "append staging");
  static_assert(kBarOff >= 8 * 8 * 1024, "tail staging: 8 units of 8 KB");
};

// Where a code of `slot` sits in its fp16 half-word for the mma: bit
// kBase + kSRow * (slot & 1).  slot & 1 is the fragment row half (channel or
// token 8..15 of the 16-block) for every width, so the offset factors into a
// per-row-half power of two with no column-half part.  The positions keep each
// code in the top bits of the 10-bit mantissa: a subnormal A operand with
// leading zero mantissa bits costs the tensor core's fp32 accumulation that
// many bits (it truncates below an alignment point set by the exponent field),
// and the V-side products, all of one sign, would then sum a coherent bias.
template <int BITS> struct CodeShift {
  static constexpr int kBase = BITS == 2 ? 6 : 2;
  static constexpr int kSRow = BITS == 2 ? 2 : (BITS == 4 ? 4 : 0);
};

// f16x2 of the two codes in `slot` of a fragment-order word (low half-word:
// even column, high half-word: odd column).  The word is shifted so the code
// lands at its CodeShift position, then masked: with the exponent field zero,
// each half IS the exact subnormal code * 2^(s - 24).  Slots that share a
// shift share the shifted word (two distinct shifts per word for 4- and 8-bit
// codes, four for 2-bit), so a code pair costs one AND plus a shared shift.
template <int BITS>
__device__ __forceinline__ uint32_t dequant_slot(uint32_t w, int slot) {
  const int s = CodeShift<BITS>::kBase + CodeShift<BITS>::kSRow * (slot & 1);
  const int sh = s - BITS * slot;
  const uint32_t x = sh >= 0 ? (w << sh) : (w >> -sh);
  const uint32_t m1 = ((1u << BITS) - 1u) << s;
  return x & (m1 | (m1 << 16));
}

// Power-of-two boost of the softmax weights fed to the V-side mma (P' <= 2^12,
// far inside fp16's range, with small weights kept out of the subnormals).
constexpr int kPBoost = 12;

__device__ __forceinline__ float hf(const __half* p, int i) { return __half2float(p[i]); }

// ------------------------------------------------------------------ tail CTA

// Quantise one side (K: 0, V: 1) of the full fp16 tail tile of (b, h) --
// rows 0..126 from the tail buffer, row 127 = the appended token -- into block
// block_table[b][L / 128], by the whole CTA, with the rotation recomputed (no
// tensor memory).  Kept out of line: it runs once per 128 steps of a sequence,
// and inlined its code pushed the split loop out of the instruction cache
// (no_instruction stalls 0.2 -> 1.75 per issue, decode 60 -> 66 us under ncu).
template <int KB, int VB>
__device__ __noinline__ void quantize_full_tail(const DecodeArgs& p, uint8_t* smem, int b, int h, int L, int side) {
  using namespace qt;
  const int tid = threadIdx.x;
  const int32_t blk = p.block_table[(int64_t)b * p.max_blocks + (L >> 7)];
  if (blk < 0 || blk >= p.num_blocks) {
    if (tid == 0) report_status(p.status, KVARN_DEV_BAD_BLOCK);
    return;
  }
  QuantScratch& sq = *reinterpret_cast<QuantScratch*>(smem + 2 * kBox);
  const uint32_t xs = smem_u32(smem);
  const __half* src = p.tail + (((int64_t)b * 2 + side) * p.Hkv + h) * (int64_t)(kTile * kHeadDim);
  const __half* nrow = (side == 0 ? p.k_new : p.v_new) + ((int64_t)b * p.Hkv + h) * kHeadDim;
  // stage row t = tid into the swizzled layout the rotation reads; all 16
  // chunks of a row are in flight at once
  const uint4* row = reinterpret_cast<const uint4*>(tid == kTile - 1 ? nrow : src + (int64_t)tid * kHeadDim);
#pragma unroll
  for (int c16 = 0; c16 < 16; ++c16) cp_async16(xs + xoff(tid, c16), row + c16, 16);
  cp_async_wait_all();
  __syncthreads();
  if (tid == 0) {   // read inside quantize_tile after its first barrier
    sq.out.codes = p.packed_w + ((int64_t)blk * p.Hkv + h) * (int64_t)(2048 * (KB + VB)) + (side == 0 ? 0 : 2048 * KB);
    sq.out.scales = p.scales_w + (((int64_t)blk * p.Hkv + h) * 2 + side) * (int64_t)kScaleRec;
    sq.out.dbg = nullptr;
  }
  if (side == 0) quantize_tile<0, KB, false>(p.iters, sq, xs, 0u);
  else quantize_tile<1, VB, false>(p.iters, sq, xs, 0u);
  // order the generic-proxy accesses to the staged tile and the scratch before
  // any later tile copy (async proxy) into the same shared memory
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  __syncthreads();   // the staged tile and the scratch are free again
}

// Column slot c (0..7) of column group grp of pair (b, h): the columns of a
// pair are its (query, head) combinations n = i * G + g, 8 per group.  Gives
// the row of that query head in q / out ([B][qlen][Hq][128]) and the query
// index; false (and column 0's row, a valid address) past G * qlen.
__device__ __forceinline__ bool col_row(const DecodeArgs& p, int b, int h, int grp, int c, int64_t* row, int* qi) {
  const int n = grp * kMaxG + c;
  const bool live = c < kMaxG && n < p.G * p.qlen;
  const int nn = live ? n : 0;
  const int i = nn / p.G, g = nn - (nn / p.G) * p.G;
  *row = ((int64_t)(b * p.qlen + i) * p.Hq + h * p.G + g) * kHeadDim;
  *qi = i;
  return live;
}

// Tail attention (a9) on the tensor cores.  The tail rows (fp16, unrotated)
// are staged in 16-row units: K then V, each two 64-channel halves of
// 16 rows x 128 bytes, 16-byte chunks XOR-swizzled by row so ldmatrix reads
// are conflict-free; rows at or past the tail length are zero.
constexpr int kTU = 16;                  // tail tokens per mma unit
constexpr int kTHalf = kTU * 128;        // one 64-channel half of a unit side (2 KB)
constexpr int kTUnitBytes = 4 * kTHalf;  // K halves, then V halves (8 KB)

__device__ __forceinline__ uint32_t toff(int r, int c16) {
  return (c16 >> 3) * kTHalf + r * 128 + (((c16 & 7) ^ (r & 7)) << 4);
}

// The tail of (b, h): seq_len % 128 rows, plus the step's own token when
// appending (taken from k_new / v_new, and also written to the tail buffer).
// Writes one partial record per query head (original domain) to the tail
// slots.
template <int KB, int VB>
__device__ void decode_tail(const DecodeArgs& p, uint8_t* smem, int b, int h, int grp, int L) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, c = lane & 3;
  const int tl = (L & 127) + p.append;
  if (tl == 0 || !debug_ok(tl <= kTile, p.status)) return;
  const int pw = (b * p.Hkv + h) * p.ngrp + grp;   // work pair: (sequence, KV head, column group)
  const int nun = (tl + kTU - 1) / kTU;
  const __half* kt = p.tail + (((int64_t)b * 2 + 0) * p.Hkv + h) * (int64_t)(kTile * kHeadDim);
  const __half* vt = p.tail + (((int64_t)b * 2 + 1) * p.Hkv + h) * (int64_t)(kTile * kHeadDim);
  // row tl - 1: the appended token, or the tail buffer's own row (never a null pointer)
  const __half* klast = p.append ? p.k_new + ((int64_t)b * p.Hkv + h) * kHeadDim : kt + (int64_t)(tl - 1) * kHeadDim;
  const __half* vlast = p.append ? p.v_new + ((int64_t)b * p.Hkv + h) * kHeadDim : vt + (int64_t)(tl - 1) * kHeadDim;

  // ---- stage rows [0, 16 * nun) with asynchronous 16-byte copies, all in
  // flight at once; rows at or past tl are zero-filled (no bytes read)
  for (int idx = tid; idx < nun * kTU * 16; idx += kDThreads) {
    const int t = idx >> 4, c16 = idx & 15;
    const bool live = t < tl;
    const __half* kr = !live ? kt : (t == tl - 1 ? klast : kt + (int64_t)t * kHeadDim);
    const __half* vr = !live ? vt : (t == tl - 1 ? vlast : vt + (int64_t)t * kHeadDim);
    const uint32_t ub = smem_u32(smem + (t >> 4) * kTUnitBytes) + toff(t & 15, c16);
    cp_async16(ub, reinterpret_cast<const uint4*>(kr) + c16, live ? 16 : 0);
    cp_async16(ub + 2 * kTHalf, reinterpret_cast<const uint4*>(vr) + c16, live ? 16 : 0);
  }
  cp_async_wait_all();
  // q fragments (B operand of q.K): column g8 at channels 16kt + 2c .. +1 and +8;
  // columns past G * qlen are 0
  uint32_t qb0[8], qb1[8];
  {
    int64_t row;
    int qi;
    const bool live = col_row(p, b, h, grp, g8, &row, &qi);
    const __half* qp = p.q + row;
#pragma unroll
    for (int kt8 = 0; kt8 < 8; ++kt8) {
      qb0[kt8] = live ? __ldg(reinterpret_cast<const unsigned int*>(qp + 16 * kt8 + 2 * c)) : 0u;
      qb1[kt8] = live ? __ldg(reinterpret_cast<const unsigned int*>(qp + 16 * kt8 + 2 * c + 8)) : 0u;
    }
  }
  // causal limit (last tail row attended) of this lane's columns 2c, 2c + 1:
  // query i sits at tail row tl - qlen + i (every row for plain decode)
  int lim[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    int64_t row;
    int qi;
    (void)col_row(p, b, h, grp, 2 * c + j, &row, &qi);
    lim[j] = tl - p.qlen + qi;
  }
  __syncthreads();

  // ---- per warp: units warp, warp + 4 with an online softmax (log2 units)
  const float sl = p.sm_scale * kLog2e;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[i][r] = 0.f;
  float mrun[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
  const int mi = lane >> 3;
  for (int un = warp; un < nun; un += kDWarps) {
    const int valid_rows = min(kTU, tl - un * kTU);
    const uint32_t kb = smem_u32(smem + un * kTUnitBytes), vb = kb + 2 * kTHalf;
    float S[4] = {0.f, 0.f, 0.f, 0.f};
    const int arow = (lane & 7) + 8 * (mi & 1);
#pragma unroll
    for (int kt8 = 0; kt8 < 8; ++kt8) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(kb + toff(arow, 2 * kt8 + (mi >> 1)), a0, a1, a2, a3);
      mma_f16(S, a0, a1, a2, a3, qb0[kt8], qb1[kt8]);
    }
    // rows g8 and g8 + 8 (tokens), heads 2c and 2c + 1; tokens past the tail masked
    const int r0 = un * kTU + g8, r1 = r0 + 8;   // tail rows; causal limits per column
    const bool v0 = g8 < valid_rows, v1 = g8 + 8 < valid_rows;
    S[0] = v0 && r0 <= lim[0] ? S[0] * sl : -INFINITY;
    S[1] = v0 && r0 <= lim[1] ? S[1] * sl : -INFINITY;
    S[2] = v1 && r1 <= lim[0] ? S[2] * sl : -INFINITY;
    S[3] = v1 && r1 <= lim[1] ? S[3] * sl : -INFINITY;
    float mx0 = fmaxf(S[0], S[2]), mx1 = fmaxf(S[1], S[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(mrun[0], mx0), mn1 = fmaxf(mrun[1], mx1);
    // a column with no attended row yet keeps max -inf: exponents are then
    // taken against 0 so that every weight is 0 instead of NaN
    const float e0 = mn0 == -INFINITY ? 0.f : mn0, e1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2_fast(mrun[0] - e0), al1 = ex2_fast(mrun[1] - e1);
    mrun[0] = mn0;
    mrun[1] = mn1;
    const float p0 = ex2_fast(S[0] - e0), p1 = ex2_fast(S[1] - e1);
    const float p2 = ex2_fast(S[2] - e0), p3 = ex2_fast(S[3] - e1);
    lsum[0] = lsum[0] * al0 + (p0 + p2);
    lsum[1] = lsum[1] * al1 + (p1 + p3);
    const uint32_t bv0 = movmatrix_t(pack_f2h2(p0, p1));
    const uint32_t bv1 = movmatrix_t(pack_f2h2(p2, p3));
    // P.V: A = V^T (rows channels, k = the unit's 16 tokens) via ldmatrix.trans
    const int vrow = (lane & 7) + 8 * (mi >> 1);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_t(vb + toff(vrow, 2 * mt + (mi & 1)), a0, a1, a2, a3);
      float o[4] = {0.f, 0.f, 0.f, 0.f};
      mma_f16(o, a0, a1, a2, a3, bv0, bv1);
      acc[mt][0] = fmaf(acc[mt][0], al0, o[0]);
      acc[mt][1] = fmaf(acc[mt][1], al1, o[1]);
      acc[mt][2] = fmaf(acc[mt][2], al0, o[2]);
      acc[mt][3] = fmaf(acc[mt][3], al1, o[3]);
    }
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], o);
    lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], o);
  }
  __syncthreads();   // the staged units are dead; the merge area reuses them

  // ---- merge the four warps, write the tail record per head
  float* mS = reinterpret_cast<float*>(smem);            // [4][8]
  float* lS = mS + kDWarps * kMaxG;                      // [4][8]
  float* aS = lS + kDWarps * kMaxG;                      // [4][8][128]
  if (g8 == 0) {
    mS[warp * kMaxG + 2 * c] = mrun[0];
    mS[warp * kMaxG + 2 * c + 1] = mrun[1];
    lS[warp * kMaxG + 2 * c] = lsum[0];
    lS[warp * kMaxG + 2 * c + 1] = lsum[1];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      const int d = 16 * mt + g8 + 8 * ri;
      aS[(warp * kMaxG + 2 * c) * kHeadDim + d] = acc[mt][2 * ri];
      aS[(warp * kMaxG + 2 * c + 1) * kHeadDim + d] = acc[mt][2 * ri + 1];
    }
  __syncthreads();
  const int d = tid;
  for (int g = 0; g < p.C; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) M = fmaxf(M, mS[w * kMaxG + g]);
    float l = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) {
      const float mw = mS[w * kMaxG + g];
      const float f = mw == -INFINITY ? 0.f : ex2_fast(mw - M);
      l = fmaf(f, lS[w * kMaxG + g], l);
      a = fmaf(f, aS[(w * kMaxG + g) * kHeadDim + d], a);
    }
    float* rec = p.ws_tail + ((int64_t)pw * p.C + g) * kPartialFloats;
    if (d == 0) {
      rec[0] = M;
      rec[1] = l;
      rec[2] = 0.f;
      rec[3] = 0.f;
    }
    rec[4 + d] = a;
  }
  // the staged rows are dead: order these generic-proxy accesses before any
  // later tile copy (async proxy) into the same shared memory
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (p.append) {
    const int r = L & 127;
    __half* kw = p.tail_w + (((int64_t)b * 2 + 0) * p.Hkv + h) * (int64_t)(kTile * kHeadDim) + (int64_t)r * kHeadDim;
    __half* vw = p.tail_w + (((int64_t)b * 2 + 1) * p.Hkv + h) * (int64_t)(kTile * kHeadDim) + (int64_t)r * kHeadDim;
    kw[d] = klast[d];
    vw[d] = vlast[d];
  }
}

// ------------------------------------------------------------------ main kernel

// Copy unit `unit` of this warp (physical block blk) into stage k % 2;
// returns false (and completes the stage's phase empty) for a bad block id.
template <int KB, int VB>
__device__ __forceinline__ bool issue_unit(const DecodeArgs& p, uint8_t* stage_base, uint64_t* my_bars, int k,
                                           int unit, int32_t blk, int h, int lane) {
  using T = DecodeTraits<KB, VB>;
  const int part = unit % T::U;
  const bool ok = blk >= 0 && blk < p.num_blocks;
  if (lane == 0) {
    uint8_t* dst = stage_base + (k & 1) * T::kStage;
    uint64_t* bar = &my_bars[k & 1];
#if KVARN_TEST_STALL_FIRST_UNIT
    // test build only: the first unit of warp 0 of CTA 0 expects 16 bytes that
    // are never sent and no copy is issued, so its bounded wait runs out
    if (blockIdx.x == 0 && threadIdx.x == 0 && k == 0) {
      mbar_arrive_expect_tx(bar, 16);
      return ok;
    }
#endif
    if (ok) {
      const uint8_t* cb = p.packed + ((int64_t)blk * p.Hkv + h) * T::kCode;
      mbar_arrive_expect_tx(bar, T::kStage);
      const uint64_t pol = l2_evict_first_policy();   // the codes are read once per call
      bulk_g2s_hint(dst, cb + part * T::kUnitK, T::kUnitK, bar, pol);
      bulk_g2s_hint(dst + T::kUnitK, cb + T::kCodeK + part * T::kUnitV, T::kUnitV, bar, pol);
      bulk_g2s(dst + T::kUnitK + T::kUnitV, p.scales + ((int64_t)blk * p.Hkv + h) * (2 * kScaleRec), 2 * kScaleRec,
               bar);
    } else {
      report_status(p.status, KVARN_DEV_BAD_BLOCK);
      mbar_arrive_expect_tx(bar, 0);   // completes the phase with no bytes
    }
  }
  return ok;
}

// The tile loop of one warp: work units u0, u0 + ustep, ... (n_mine of them;
// unit = (tile, part), tiles counted from t_begin) of sequence b, KV head h,
// streamed through this warp's private 2-stage ring and folded into the warp's
// online-softmax state (acc in the rotated domain, running max and sum per
// query-head column).  kbase: how many units this warp's ring has carried since
// its barriers were initialised (unit k uses stage (kbase + k) % 2 and waits for
// phase parity ((kbase + k) / 2) % 2).  Returns the unit whose copy timed out,
// or -1.
template <int KB, int VB>
__device__ __forceinline__ int run_units(const DecodeArgs& p, uint8_t* stage_base, uint64_t* my_bars, float* scr,
                                         float* tokbuf, int b, int h, int t_begin, int kbase, int u0, int ustep,
                                         int n_mine,
                                         const float (&qr)[32], float coef0, float coef1, int mask_tile,
                                         const int (&climit)[2], float (&acc)[8][4], float (&mrun)[2],
                                         float (&lsum)[2]) {
  using T = DecodeTraits<KB, VB>;
  constexpr int U = T::U, MT = T::MT;
  const int lane = threadIdx.x & 31, g8 = lane >> 2, c = lane & 3;
  const int32_t* btab = p.block_table + (int64_t)b * p.max_blocks;
  // block id of tile t of the sequence (debug builds: an index past the row reads as a bad block)
  auto block_of = [&](int t) -> int32_t { return debug_ok(t >= 0 && t < p.max_blocks, p.status) ? btab[t] : -1; };
  // ok0 / ok1: the unit now in flight in stage 0 / 1 has a valid block
  bool ok0 = false, ok1 = false;
  if (n_mine > 0) {
    const bool o = issue_unit<KB, VB>(p, stage_base, my_bars, kbase, u0, block_of(t_begin + u0 / U), h, lane);
    if (kbase & 1) ok1 = o; else ok0 = o;
  }
  if (n_mine > 1) {
    const bool o = issue_unit<KB, VB>(p, stage_base, my_bars, kbase + 1, u0 + ustep,
                                      block_of(t_begin + (u0 + ustep) / U), h, lane);
    if (kbase & 1) ok0 = o; else ok1 = o;
  }
  int k_fail = -1;

  for (int k = 0; k < n_mine; ++k) {
    const int kg = kbase + k;
    const int stg = kg & 1;
    // block id of unit k + 2, loaded now so it is in hand when that copy is issued
    const int32_t blk_next = k + 2 < n_mine ? block_of(t_begin + (u0 + (k + 2) * ustep) / U) : 0;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&my_bars[stg], (kg >> 1) & 1))) {
      if (lane == 0) report_status(p.status, KVARN_DEV_TIMEOUT);
      k_fail = k;
      break;
    }
    const bool tile_ok = stg == 0 ? ok0 : ok1;
    const int part = (u0 + k * ustep) % U;
    const uint8_t* st = stage_base + stg * T::kStage;
    if (tile_ok) {
      const uint8_t* rk = st + T::kUnitK + T::kUnitV;   // K scale record, V record follows
      const __half* ltk = reinterpret_cast<const __half*>(rk);
      const __half* lck = ltk + 128;
      const float zk = *reinterpret_cast<const float*>(rk + 512);
      const float sk = *reinterpret_cast<const float*>(rk + 516);
      const __half* ltv = reinterpret_cast<const __half*>(rk + kScaleRec);
      const __half* lcv = ltv + 128;
      const float zv = *reinterpret_cast<const float*>(rk + kScaleRec + 512);
      const float sv = *reinterpret_cast<const float*>(rk + kScaleRec + 516);
      const int t0 = part * (16 * MT);   // first token of this unit within the tile
      // token scales once per token (MT / 2 tokens per lane): 2^Lt_k, and the V
      // scales relative to the unit's largest, times 2^kPBoost (the weights
      // p * tv fed to the V-side mma then stay in fp16's normal range down to
      // p * tv ~ 2^-26 of the unit maximum; the factor is undone in the fold);
      // read back below in the score layout
      float lvm;
      {
        constexpr int TPL = MT / 2;
        float lk[TPL], lv[TPL];
#pragma unroll
        for (int i = 0; i < TPL; ++i) {
          lk[i] = hf(ltk, t0 + TPL * lane + i);
          lv[i] = hf(ltv, t0 + TPL * lane + i);
        }
        float m = lv[0];
#pragma unroll
        for (int i = 1; i < TPL; ++i) m = fmaxf(m, lv[i]);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        lvm = ceilf(m);
#pragma unroll
        for (int i = 0; i < TPL; ++i) {
          const int tr = TPL * lane + i;   // token tr sits at lane g8 = tr % 8, slot (tr / 16, tr / 8 % 2)
          const int idx = (tr & 7) * 16 + (tr >> 4) * 2 + ((tr >> 3) & 1);
          tokbuf[idx] = ex2_fast(lk[i]);
          tokbuf[128 + idx] = ex2_fast(lv[i] - lvm + static_cast<float>(kPBoost));
        }
        __syncwarp();
      }

      // a6: channel scales with a power-of-two prescale so q' <= 1 in magnitude
      float lcl[4];
      {
        const float2 l01 = __half22float2(*reinterpret_cast<const __half2*>(lck + 4 * lane));
        const float2 l23 = __half22float2(*reinterpret_cast<const __half2*>(lck + 4 * lane + 2));
        lcl[0] = l01.x; lcl[1] = l01.y; lcl[2] = l23.x; lcl[3] = l23.y;
      }
      const float E = ceilf(warp_max(fmaxf(fmaxf(lcl[0], lcl[1]), fmaxf(lcl[2], lcl[3]))));
      *reinterpret_cast<float4*>(&scr[4 * lane]) =
          make_float4(ex2_fast(lcl[0] - E), ex2_fast(lcl[1] - E), ex2_fast(lcl[2] - E), ex2_fast(lcl[3] - E));
      __syncwarp();
      // q' as an fp16 hi + lo pair (about 22 significant bits): scores can reach
      // |s| ~ 10 nats, where plain fp16 q' would cost ~1e-2 in the output
      uint32_t qb0[8], qb1[8], ql0[8], ql1[8];
      float qsum = 0.f;
#pragma unroll
      for (int kt = 0; kt < 8; ++kt) {
        const float2 s01 = *reinterpret_cast<const float2*>(&scr[16 * kt + 2 * c]);
        const float2 s89 = *reinterpret_cast<const float2*>(&scr[16 * kt + 2 * c + 8]);
        const float x0 = qr[4 * kt] * s01.x, x1 = qr[4 * kt + 1] * s01.y;
        const float x8 = qr[4 * kt + 2] * s89.x, x9 = qr[4 * kt + 3] * s89.y;
        const __half2 h01 = __floats2half2_rn(x0, x1);
        const __half2 h89 = __floats2half2_rn(x8, x9);
        const float2 f01 = __half22float2(h01), f89 = __half22float2(h89);
        const __half2 l01 = __floats2half2_rn(x0 - f01.x, x1 - f01.y);
        const __half2 l89 = __floats2half2_rn(x8 - f89.x, x9 - f89.y);
        // sum of q' for the zero-point term, from the fp32 values: hi + lo
        // carries them to about 2^-22, so the mma's q' and this sum differ by
        // a score offset far below the fp16 output rounding
        qsum += (x0 + x1) + (x8 + x9);
        qb0[kt] = h2_as_u32(h01);
        qb1[kt] = h2_as_u32(h89);
        ql0[kt] = h2_as_u32(l01);
        ql1[kt] = h2_as_u32(l89);
      }
      __syncwarp();   // the K channel scales in scr are dead
      // V channel scales 2^Lc_v once per channel (4 per lane) into scr, read
      // back in the accumulator layout (channel 16mt + g8 + 8ri at g8 * 16 + 2mt + ri)
      {
        const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(lcv + 4 * lane));
        const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(lcv + 4 * lane + 2));
        const float vv[4] = {v01.x, v01.y, v23.x, v23.y};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int d = 4 * lane + i;
          scr[(d & 7) * 16 + (d >> 4) * 2 + ((d >> 3) & 1)] = ex2_fast(vv[i]);
        }
      }
      qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
      qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
      const float qs0 = __shfl_sync(0xffffffffu, qsum, (2 * c) * 4);
      const float qs1 = __shfl_sync(0xffffffffu, qsum, (2 * c + 1) * 4);
      const float pw = ldexpf(1.f, static_cast<int>(E));
      const float cf0 = coef0 * pw, cf1 = coef1 * pw;
      const float za0 = zk * qs0, za1 = zk * qs1;

      // a7: K-side contraction on the tensor cores (rows = this unit's tokens)
      float S[MT][4];
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int r = 0; r < 4; ++r) S[i][r] = 0.f;
      {
        constexpr int PK = 16 / KB;
        uint32_t afr[4];
#pragma unroll
        for (int q = 0; q < 4 * KB / U; ++q) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(st + ((q * 32 + lane) << 4));
          const uint32_t wds[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w = wds[i];
#pragma unroll
            for (int sl = 0; sl < PK; ++sl) {
              const int rho = (4 * q + i) * PK + sl;
              afr[rho & 3] = dequant_slot<KB>(w, sl);
              if ((rho & 3) == 3) {
                const int blk = rho >> 2;   // (token block in unit) * 8 + channel block
                mma_f16(S[blk >> 3], afr[0], afr[1], afr[2], afr[3], qb0[blk & 7], qb1[blk & 7]);
                mma_f16(S[blk >> 3], afr[0], afr[1], afr[2], afr[3], ql0[blk & 7], ql1[blk & 7]);
              }
            }
          }
        }
      }

      // scores (log2 units) with the token scales, online softmax (a8)
      // the step with the codes' 2^(s - 24) placement undone, per row half
      constexpr float kRowK0 = 16777216.f / static_cast<float>(1 << CodeShift<KB>::kBase);
      constexpr float kRowK1 = kRowK0 / static_cast<float>(1 << CodeShift<KB>::kSRow);
      float tv[MT][2], tkv[MT][2];
#pragma unroll
      for (int k4 = 0; k4 < MT / 2; ++k4) {
        const float4 a = *reinterpret_cast<const float4*>(&tokbuf[g8 * 16 + 4 * k4]);
        const float4 b = *reinterpret_cast<const float4*>(&tokbuf[128 + g8 * 16 + 4 * k4]);
        tkv[2 * k4][0] = a.x; tkv[2 * k4][1] = a.y; tkv[2 * k4 + 1][0] = a.z; tkv[2 * k4 + 1][1] = a.w;
        tv[2 * k4][0] = b.x; tv[2 * k4][1] = b.y; tv[2 * k4 + 1][0] = b.z; tv[2 * k4 + 1][1] = b.w;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          const float tk = tkv[mt][ri];
          const float skr = sk * (ri ? kRowK1 : kRowK0);
          S[mt][2 * ri] = fmaf(skr, S[mt][2 * ri], za0) * (cf0 * tk);
          S[mt][2 * ri + 1] = fmaf(skr, S[mt][2 * ri + 1], za1) * (cf1 * tk);
          mx0 = fmaxf(mx0, S[mt][2 * ri]);
          mx1 = fmaxf(mx1, S[mt][2 * ri + 1]);
        }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (t_begin + (u0 + k * ustep) / U == mask_tile) {   // warp-uniform: the tile holding query positions
        mx0 = -INFINITY;
        mx1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int ri = 0; ri < 2; ++ri) {
            const int t = t0 + 16 * mt + g8 + 8 * ri;
            if (t > climit[0]) S[mt][2 * ri] = -INFINITY;
            if (t > climit[1]) S[mt][2 * ri + 1] = -INFINITY;
            mx0 = fmaxf(mx0, S[mt][2 * ri]);
            mx1 = fmaxf(mx1, S[mt][2 * ri + 1]);
          }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
      }
      const float mn0 = fmaxf(mrun[0], mx0), mn1 = fmaxf(mrun[1], mx1);
      // a column that has attended no token yet (masked) keeps max -inf: its
      // exponents are taken against 0, so its weights are 0 instead of NaN
      const float e0 = mn0 == -INFINITY ? 0.f : mn0, e1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = ex2_fast(mrun[0] - e0), al1 = ex2_fast(mrun[1] - e1);
      mrun[0] = mn0;
      mrun[1] = mn1;
      float ls0 = 0.f, ls1 = 0.f, ps0 = 0.f, ps1 = 0.f;
      uint32_t bv0[MT], bv1[MT];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t pk[2];
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          const float p0 = ex2_fast(S[mt][2 * ri] - e0);
          const float p1 = ex2_fast(S[mt][2 * ri + 1] - e1);
          ls0 += p0;
          ls1 += p1;
          const __half2 hp = __floats2half2_rn(p0 * tv[mt][ri], p1 * tv[mt][ri]);
          // the zero-point term must use exactly the weights the mma sees: after the
          // inverse Hadamard a common error across channels lands on one output channel
          const float2 fp = __half22float2(hp);
          ps0 += fp.x;
          ps1 += fp.y;
          pk[ri] = h2_as_u32(hp);
        }
        bv0[mt] = movmatrix_t(pk[0]);
        bv1[mt] = movmatrix_t(pk[1]);
      }
      lsum[0] = lsum[0] * al0 + ls0;
      lsum[1] = lsum[1] * al1 + ls1;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        ps0 += __shfl_xor_sync(0xffffffffu, ps0, o);
        ps1 += __shfl_xor_sync(0xffffffffu, ps1, o);
      }

      // V-side contraction on the tensor cores (rows = channels, k = this unit's tokens)
      float O[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int r = 0; r < 4; ++r) O[i][r] = 0.f;
      {
        constexpr int PV = 16 / VB;
        uint32_t afr[4];
        const uint8_t* vc = st + T::kUnitK;
#pragma unroll
        for (int q = 0; q < 4 * VB / U; ++q) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(vc + ((q * 32 + lane) << 4));
          const uint32_t wds[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t w = wds[i];
#pragma unroll
            for (int sl = 0; sl < PV; ++sl) {
              const int rho = (4 * q + i) * PV + sl;
              afr[rho & 3] = dequant_slot<VB>(w, sl);
              if ((rho & 3) == 3) {
                const int blk = rho >> 2;   // (token block in unit) * 8 + channel block
                mma_f16(O[blk & 7], afr[0], afr[1], afr[2], afr[3], bv0[blk >> 3], bv1[blk >> 3]);
              }
            }
          }
        }
      }

      // fold the V grid and channel scales into the running accumulator
      const float tvf = ex2_fast(lvm - static_cast<float>(kPBoost));
      const float zp0 = zv * tvf * ps0, zp1 = zv * tvf * ps1;
      const float sv0 = sv * tvf * (16777216.f / static_cast<float>(1 << CodeShift<VB>::kBase));
      const float sv1 = sv0 * (1.f / static_cast<float>(1 << CodeShift<VB>::kSRow));
      __syncwarp();   // the V channel scales are in scr
      float vcsv[16];
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        const float4 x = *reinterpret_cast<const float4*>(&scr[g8 * 16 + 4 * k4]);
        vcsv[4 * k4] = x.x; vcsv[4 * k4 + 1] = x.y; vcsv[4 * k4 + 2] = x.z; vcsv[4 * k4 + 3] = x.w;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int ri = 0; ri < 2; ++ri) {
          const float vcs = vcsv[2 * mt + ri];
          const float svr = ri ? sv1 : sv0;   // step with the codes' placement undone, per row half
          acc[mt][2 * ri] = fmaf(acc[mt][2 * ri], al0, vcs * fmaf(svr, O[mt][2 * ri], zp0));
          acc[mt][2 * ri + 1] = fmaf(acc[mt][2 * ri + 1], al1, vcs * fmaf(svr, O[mt][2 * ri + 1], zp1));
        }
    }
    // the stage's generic reads are ordered before the async-proxy refill
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    __syncwarp();
    if (k + 2 < n_mine) {
      const bool okn = issue_unit<KB, VB>(p, stage_base, my_bars, kg + 2, u0 + (k + 2) * ustep, blk_next, h, lane);
      if (stg == 0) ok0 = okn; else ok1 = okn;
    }
  }

  if (k_fail >= 0) {
    // let the copies still in flight land before the shared memory is released
    const int kf = kbase + k_fail;
    (void)mbar_wait_bounded(&my_bars[kf & 1], (kf >> 1) & 1);
    if (k_fail + 1 < n_mine) (void)mbar_wait_bounded(&my_bars[(kf + 1) & 1], ((kf + 1) >> 1) & 1);
  }

  return k_fail;
}

// One segment: full tiles [t_begin, t_end) of sequence b (length L), KV head
// h, by the whole CTA; writes one partial record per query head at
// recs + g * 132.  With several queries per sequence the last full tile can
// hold query positions: there each (query, head) column masks the tokens
// after its own query.
// Work units (tile, part) go round-robin over the warps starting at warp
// `woff`, so a CTA that runs several segments keeps its warps level.  `rearm`:
// the barriers were used by an earlier segment and are invalidated first.
// Returns false if a copy timed out (the status is set).
template <int KB, int VB>
__device__ __forceinline__ bool decode_segment(const DecodeArgs& p, uint8_t* smem, int b, int h, int grp, int L,
                                               int t_begin, int t_end, int woff, bool rearm, float* recs) {
  using T = DecodeTraits<KB, VB>;
  constexpr int U = T::U;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T::kBarOff);
  float* qrot = reinterpret_cast<float*>(smem + T::kQrotOff);
  float* invsig = reinterpret_cast<float*>(smem + T::kInvSigOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (t_begin >= t_end) return true;

  if (tid == 0) {
    for (int i = 0; i < kDWarps * kDStages; ++i) {
      if (rearm) mbar_inval(&bars[i]);
      mbar_init(&bars[i], 1);
    }
    fence_barrier_init();
  }

  // ---- q H for the group's (query, head) columns, scaled by a power of two so |q H| <= 1 (a6)
  {
    const int g = tid >> 4, part = tid & 15;
    float x[8];
    int64_t qrow;
    int qi;
    if (col_row(p, b, h, grp, g, &qrow, &qi)) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.q + qrow + part * 8));
      const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(hp[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
    }
#pragma unroll
    for (int hl = 1; hl < 8; hl <<= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if ((i & hl) == 0) {
          const float a = x[i], c = x[i + hl];
          x[i] = a + c;
          x[i + hl] = a - c;
        }
#pragma unroll
    for (int m = 1; m < 16; m <<= 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float y = __shfl_xor_sync(0xffffffffu, x[i], m);
        x[i] = up ? (y - x[i]) : (x[i] + y);
      }
    }
    float mx = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(x[i]));
#pragma unroll
    for (int m = 1; m < 16; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    int e = 0;
    if (mx > 0.f) frexpf(mx, &e);
    const float sig = ldexpf(1.f, -e);
#pragma unroll
    for (int i = 0; i < 8; ++i) qrot[g * 128 + part * 8 + i] = x[i] * sig;
    if (part == 0) invsig[g] = ldexpf(1.f, e);
  }
  __syncthreads();

  // ---- per-warp state
  const int g8 = lane >> 2, c = lane & 3;
  float qr[32];   // q H of head g8 at channels 16kt + 2c + {0,1,8,9}
#pragma unroll
  for (int kt = 0; kt < 8; ++kt) {
    const float2 lo = *reinterpret_cast<const float2*>(&qrot[g8 * 128 + 16 * kt + 2 * c]);
    const float2 hi = *reinterpret_cast<const float2*>(&qrot[g8 * 128 + 16 * kt + 2 * c + 8]);
    qr[4 * kt] = lo.x;
    qr[4 * kt + 1] = lo.y;
    qr[4 * kt + 2] = hi.x;
    qr[4 * kt + 3] = hi.y;
  }
  // causal limits (last token index attended inside the last full tile) of
  // this lane's columns 2c, 2c + 1: query i sits at position L - qlen + i
  const int mask_tile = p.qlen > 1 ? (L >> 7) - 1 : -1;
  int climit[2] = {kTile - 1, kTile - 1};
  if (mask_tile >= 0) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      int64_t row;
      int qi;
      if (col_row(p, b, h, grp, 2 * c + j, &row, &qi)) climit[j] = L - p.qlen + qi - kTile * mask_tile;
    }
  }
  __syncthreads();   // every warp holds its q H: the q H buffer now serves as per-warp token-scale scratch
  float* tokbuf = qrot + warp * 256;   // [2 (K, V)][8 (g8)][16 (mt, ri)]
  const float coef0 = p.sm_scale * kLog2e * (1.f / 128.f) * invsig[2 * c];
  const float coef1 = p.sm_scale * kLog2e * (1.f / 128.f) * invsig[2 * c + 1];
  float* scr = reinterpret_cast<float*>(smem + T::kScrOff) + warp * kHeadDim;

  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[i][r] = 0.f;
  float mrun[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};

  // work units of this segment: (tile, part), part in [0, U); warp takes every 4th from u0
  const int n_units = (t_end - t_begin) * U;
  const int u0 = (warp - woff + kDWarps) % kDWarps;
  const int n_mine = u0 < n_units ? (n_units - u0 + kDWarps - 1) / kDWarps : 0;
  uint8_t* stage_base = smem + warp * kDStages * T::kStage;
  uint64_t* my_bars = bars + warp * kDStages;

  const int k_fail = run_units<KB, VB>(p, stage_base, my_bars, scr, tokbuf, b, h, t_begin, 0, u0, kDWarps, n_mine, qr,
                                       coef0, coef1, mask_tile, climit, acc, mrun, lsum);

  // ---- merge the four warps and write the partial (m, l, acc) per head
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], o);
    lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], o);
  }
  const bool failed = __syncthreads_or(k_fail >= 0) != 0;   // all warps are done with their stages
  float* mS = reinterpret_cast<float*>(smem);            // [4][8]
  float* lS = mS + kDWarps * kMaxG;                      // [4][8]
  float* aS = lS + kDWarps * kMaxG;                      // [4][8][128]
  if (g8 == 0) {
    mS[warp * kMaxG + 2 * c] = mrun[0];
    mS[warp * kMaxG + 2 * c + 1] = mrun[1];
    lS[warp * kMaxG + 2 * c] = lsum[0];
    lS[warp * kMaxG + 2 * c + 1] = lsum[1];
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int ri = 0; ri < 2; ++ri) {
      const int d = 16 * mt + g8 + 8 * ri;
      aS[(warp * kMaxG + 2 * c) * kHeadDim + d] = acc[mt][2 * ri];
      aS[(warp * kMaxG + 2 * c + 1) * kHeadDim + d] = acc[mt][2 * ri + 1];
    }
  __syncthreads();
  const int d = tid;
  for (int g = 0; g < p.C; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) M = fmaxf(M, mS[w * kMaxG + g]);
    float l = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) {
      const float mw = mS[w * kMaxG + g];
      const float f = mw == -INFINITY ? 0.f : ex2_fast(mw - M);
      l = fmaf(f, lS[w * kMaxG + g], l);
      a = fmaf(f, aS[(w * kMaxG + g) * kHeadDim + d], a);
    }
    float* rec = recs + (int64_t)g * kPartialFloats;
    if (d == 0) {
      rec[0] = M;
      rec[1] = l;
      rec[2] = 0.f;
      rec[3] = 0.f;
    }
    rec[4 + d] = a;
  }
  // the merge area is dead: order its generic-proxy accesses before the next
  // segment's tile copies (async proxy) into the same shared memory
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  __syncthreads();   // the merge area and the q buffers are free for the next segment
  return !failed;
}

// ------------------------------------------------------------------ stream-K geometry

// Work units of each KV head of sequence b: one per full tile, plus
// kTailUnits for the fp16 tail (which also carries an empty or invalid
// sequence, so every pair is owned).  The tail, and usually the merge of the
// pair, fall to the CTA owning the pair's last unit; weighting them as
// several tiles keeps that CTA's range shorter (14 measured best of 4-18).  A pair with no tail rows
// (seq_len a multiple of 128, nothing appended) weighs kTailUnitsEmpty: the
// merge and a segment restart only.
// A tail that an appended token fills is also quantised, K and V as two more
// work items of kFillUnits each after the tail (rotation recomputed), so that
// up to three CTAs share a fill.  Each item falls to the CTA holding its last unit.
constexpr int kTailUnits = 14;
constexpr int kTailUnitsEmpty = 3;
constexpr int kFillUnits = 16;

// With qlen > 1 the sequence must hold its qlen query tokens (L >= qlen); as
// qlen <= 128, query positions reach back at most into the last full tile.
__device__ __forceinline__ bool seq_valid(const DecodeArgs& p, int L) {
  return L >= 0 && L + p.append <= kTile * p.max_blocks && (p.qlen == 1 || L >= p.qlen);
}
__device__ __forceinline__ int pair_tiles(int L, bool valid) { return valid ? (L >> 7) : 0; }
__device__ __forceinline__ int tail_units(const DecodeArgs& p, int L, bool valid) {
  return valid && (L & 127) + p.append == 0 ? kTailUnitsEmpty : kTailUnits;
}
__device__ __forceinline__ int pair_units(const DecodeArgs& p, int L, bool valid) {
  const bool fills = valid && p.append && (L & 127) == kTile - 1;
  return pair_tiles(L, valid) + tail_units(p, L, valid) + (fills ? 2 * kFillUnits : 0);
}

// CTA i of P owns units [W*i/P, W*(i+1)/P); owner(u) inverts that.
__device__ __forceinline__ long long sk_begin(long long W, int P, int i) { return W * i / P; }
__device__ __forceinline__ int sk_owner(long long W, int P, long long u) {
  return static_cast<int>(((u + 1) * P - 1) / W);
}

// Warp 0: total units W, and the sequence whose units hold this CTA's first
// unit with that sequence's first unit.
__device__ void sk_locate(const DecodeArgs& p, int cta, int P, long long* W_out, int* b_out, long long* ps_out) {
  const int lane = threadIdx.x & 31;
  long long mine = 0;
  for (int b = lane; b < p.B; b += 32) {
    const int L = p.seq_lens[b];
    mine += static_cast<long long>(pair_units(p, L, seq_valid(p, L))) * p.Hkv * p.ngrp;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  const long long W = mine;
  const long long u0 = sk_begin(W, P, cta);
  long long base = 0;
  int fb = 0;
  long long fps = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    long long v = 0;
    if (b < p.B) {
      const int L = p.seq_lens[b];
      v = static_cast<long long>(pair_units(p, L, seq_valid(p, L))) * p.Hkv * p.ngrp;
    }
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const long long first = base + incl - v;
    const unsigned hit = __ballot_sync(0xffffffffu, b < p.B && u0 >= first && u0 < first + v);
    if (hit != 0u) {
      const int l = __ffs(hit) - 1;
      fb = b0 + l;
      fps = __shfl_sync(0xffffffffu, first, l);
      break;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  *W_out = W;
  *b_out = fb;
  *ps_out = fps;
}

// ------------------------------------------------------------------ combine (a10)

// Merge the partials of pair (b, h) for its G query heads:
// o = (acc H / 128 + tail) / l.  Tile records come from every CTA whose range
// meets the pair's full tiles [pst, pst + nt) (record slot pair + CTA), the
// tail record from its own slot.  One warp per head; lane owns channels
// 4*lane .. 4*lane + 3.  Records written by other CTAs are read with
// ld.global.cg (L2), never through L1.
template <int NC, int CH>
__device__ void combine_columns(const DecodeArgs& p, int b, int h, int grp, int L, bool valid, long long pst, int nt,
                                long long W, int P, int col0, int col1) {
  const int lane = threadIdx.x & 31;
  const int pair = (b * p.Hkv + h) * p.ngrp + grp;   // work pair: (sequence, KV head, column group)
  // CTAs whose ranges meet the tiles: owner(pst) .. owner(pst + nt - 1).  With
  // W >= P every CTA range is non-empty, so each of them wrote a record.
  const int i_lo = nt > 0 ? sk_owner(W, P, pst) : 0;
  const int n_rec = nt > 0 ? sk_owner(W, P, pst + nt - 1) - i_lo + 1 : 0;
  // debug builds: the records read below are slots pair + i_lo .. pair + i_lo + n_rec - 1 of the workspace
  if (!debug_ok(i_lo >= 0 && n_rec >= 0 && i_lo + n_rec <= P && P <= kDecodeMaxCtas, p.status)) return;
  const bool dense = W >= P;
  const bool has_tail = (L & 127) + p.append != 0;
  // a warp merges NC column slots (col0, then col1) together, so one round of
  // L2 loads serves them all; records are read CH at a time
  int gh[NC];
  bool hl[NC];
  int64_t orow[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    int qi;
    gh[k] = k == 0 ? col0 : col1;
    hl[k] = col_row(p, b, h, grp, gh[k], &orow[k], &qi);
  }
  if (!hl[0]) return;
  if (!valid || L + p.append == 0) {
#pragma unroll
    for (int k = 0; k < NC; ++k)
      if (hl[k]) {
        __half* o = p.out + orow[k] + 4 * lane;
        *reinterpret_cast<uint2*>(o) = make_uint2(0u, 0u);
      }
    return;
  }
  float M[NC], l[NC], a[NC][4];
  float mt[NC], lt[NC];
  float4 vt[NC];
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    M[k] = -INFINITY;
    l[k] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) a[k][i] = 0.f;
    const float* trec = p.ws_tail + ((int64_t)pair * p.C + (hl[k] ? gh[k] : 0)) * kPartialFloats;
    const bool t = has_tail && hl[k];
    mt[k] = t ? __ldcg(trec) : -INFINITY;
    lt[k] = t ? __ldcg(trec + 1) : 0.f;
    vt[k] = t ? __ldcg(reinterpret_cast<const float4*>(trec + 4 + 4 * lane)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int k0 = 0; k0 < n_rec; k0 += CH) {
    float mr[NC][CH], lr[NC][CH];
    float4 vr[NC][CH];
#pragma unroll
    for (int q = 0; q < CH; ++q) {
      const int i = i_lo + k0 + q;
      bool live = k0 + q < n_rec;
      if (live && !dense) live = max(sk_begin(W, P, i), pst) < min(sk_begin(W, P, i + 1), pst + nt);
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        const bool lk = live && hl[k];
        const float* r = p.ws + ((int64_t)(pair + (lk ? i : i_lo)) * p.C + (hl[k] ? gh[k] : 0)) * kPartialFloats;
        mr[k][q] = lk ? __ldcg(r) : -INFINITY;
        lr[k][q] = lk ? __ldcg(r + 1) : 0.f;
        vr[k][q] = lk ? __ldcg(reinterpret_cast<const float4*>(r + 4 + 4 * lane)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    // the round's records at once: their max, then the weights 2^(m - max)
    // (independent) and the weighted sums in four interleaved partials, so no
    // step waits on the previous record; rounds combine online
#pragma unroll
    for (int k = 0; k < NC; ++k) {
      float Mr = -INFINITY;
#pragma unroll
      for (int q = 0; q < CH; ++q) Mr = fmaxf(Mr, mr[k][q]);
      if (Mr == -INFINITY) continue;   // no live record in this round
      float lp[4] = {0.f, 0.f, 0.f, 0.f};
      float4 ap[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) ap[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < CH; ++q) {
        const float f = mr[k][q] == -INFINITY ? 0.f : ex2_fast(mr[k][q] - Mr);
        lp[q & 3] = fmaf(f, lr[k][q], lp[q & 3]);
        ap[q & 3].x = fmaf(f, vr[k][q].x, ap[q & 3].x);
        ap[q & 3].y = fmaf(f, vr[k][q].y, ap[q & 3].y);
        ap[q & 3].z = fmaf(f, vr[k][q].z, ap[q & 3].z);
        ap[q & 3].w = fmaf(f, vr[k][q].w, ap[q & 3].w);
      }
      const float Mn = fmaxf(M[k], Mr);
      const float fo = ex2_fast(M[k] - Mn), fr = ex2_fast(Mr - Mn);
      l[k] = fmaf(l[k], fo, ((lp[0] + lp[1]) + (lp[2] + lp[3])) * fr);
      a[k][0] = fmaf(a[k][0], fo, ((ap[0].x + ap[1].x) + (ap[2].x + ap[3].x)) * fr);
      a[k][1] = fmaf(a[k][1], fo, ((ap[0].y + ap[1].y) + (ap[2].y + ap[3].y)) * fr);
      a[k][2] = fmaf(a[k][2], fo, ((ap[0].z + ap[1].z) + (ap[2].z + ap[3].z)) * fr);
      a[k][3] = fmaf(a[k][3], fo, ((ap[0].w + ap[1].w) + (ap[2].w + ap[3].w)) * fr);
      M[k] = Mn;
    }
  }
#pragma unroll
  for (int k = 0; k < NC; ++k) {
    if (!hl[k]) continue;
    float* ak = a[k];
    {   // acc H / 128
      const float b0 = ak[0] + ak[1], b1 = ak[0] - ak[1], b2 = ak[2] + ak[3], b3 = ak[2] - ak[3];
      ak[0] = b0 + b2; ak[1] = b1 + b3; ak[2] = b0 - b2; ak[3] = b1 - b3;
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        const bool up = (lane & m) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float y = __shfl_xor_sync(0xffffffffu, ak[i], m);
          ak[i] = up ? (y - ak[i]) : (ak[i] + y);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) ak[i] *= (1.f / 128.f);
    }
    if (has_tail) {   // the tail, in the original domain
      const float Mn = fmaxf(M[k], mt[k]);
      const float fo = ex2_fast(M[k] - Mn), fr = ex2_fast(mt[k] - Mn);
      l[k] = fmaf(l[k], fo, lt[k] * fr);
      ak[0] = fmaf(ak[0], fo, vt[k].x * fr);
      ak[1] = fmaf(ak[1], fo, vt[k].y * fr);
      ak[2] = fmaf(ak[2], fo, vt[k].z * fr);
      ak[3] = fmaf(ak[3], fo, vt[k].w * fr);
    }
    const float il = 1.f / l[k];
    const __half2 o01 = __floats2half2_rn(ak[0] * il, ak[1] * il);
    const __half2 o23 = __floats2half2_rn(ak[2] * il, ak[3] * il);
    __half* o = p.out + orow[k] + 4 * lane;
    *reinterpret_cast<uint2*>(o) = make_uint2(h2_as_u32(o01), h2_as_u32(o23));
  }
}

// Half a pair's columns by one CTA: warp w merges column 4 * half + w alone,
// reading up to 16 records per round of L2 loads.
__device__ __forceinline__ void combine_half(const DecodeArgs& p, int b, int h, int grp, int half, int L,
                                             bool valid, long long pst, int nt, long long W, int P) {
  const int warp = threadIdx.x >> 5;
  combine_columns<1, 16>(p, b, h, grp, L, valid, pst, nt, W, P, kDWarps * half + warp, kMaxG);
}

// ------------------------------------------------------------------ main kernel

// Stream-K: CTA `cta` of P walks its unit range [W*cta/P, W*(cta+1)/P) pair by
// pair.  For each pair it meets it decodes the run of full tiles in its range
// (one partial record per query head, slot pair + cta) and attends the tail if
// the pair's tail unit is in its range.  The pairs are merged by merge_kernel,
// behind this grid.  No CTA waits on another.
template <int KB, int VB>
__global__ void __launch_bounds__(kDThreads, KVARN_D_MIN_CTAS) decode_kernel(const __grid_constant__ DecodeArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  // walker state (thread 0) and the current segment, in shared memory so that
  // almost nothing of the walk is live in registers across a segment
  __shared__ long long sh_W, sh_u, sh_ps;
  __shared__ int sh_b, sg_b, sg_h, sg_L, sg_ta, sg_te, sg_tail;
  const int tid = threadIdx.x, cta = blockIdx.x, P = gridDim.x;
  // This grid is a programmatic dependent launch: it waits for the previous
  // kernel in the stream before its first global-memory access.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  if (tid < 32) {
    long long W, ps;
    int b0;
    sk_locate(p, cta, P, &W, &b0, &ps);
    if (tid == 0) {
      sh_W = W;
      sh_u = sk_begin(W, P, cta);
      sh_b = b0;
      sh_ps = ps;
    }
  }
  int woff = 0;
  bool rearm = false, ok = true;
  for (;;) {
    __syncthreads();
    if (tid == 0) {   // the next segment: one pair's part of this CTA's range
      const long long W = sh_W, u = sh_u, u_end = sk_begin(W, P, cta + 1);
      if (u >= u_end) {
        sg_b = -1;
      } else {
        int b = sh_b;
        long long ps = sh_ps;
        int L = p.seq_lens[b];
        int nu = pair_units(p, L, seq_valid(p, L));
        if (u >= ps + static_cast<long long>(nu) * p.Hkv * p.ngrp) {   // next sequence (each has >= Hkv units)
          ps += static_cast<long long>(nu) * p.Hkv * p.ngrp;
          ++b;
          L = p.seq_lens[b];
          nu = pair_units(p, L, seq_valid(p, L));
          sh_b = b;
          sh_ps = ps;
        }
        const int h = static_cast<int>((u - ps) / nu);   // sub-pair: KV head x column group
        const long long pst = ps + static_cast<long long>(h) * nu;
        const long long e = min(u_end, pst + nu);
        sg_b = b;
        sg_h = h;
        sg_L = L;
        sg_ta = static_cast<int>(u - pst);
        sg_te = static_cast<int>(min(e - pst, static_cast<long long>(pair_tiles(L, seq_valid(p, L)))));
        // last units of the work items after the tiles: tail attention, then
        // (a filling append) quantise K, quantise V
        const int tu = tail_units(p, L, seq_valid(p, L));
        const long long m_att = pst + pair_tiles(L, seq_valid(p, L)) + tu - 1;
        const int items = nu - pair_tiles(L, seq_valid(p, L)) > tu ? 3 : 1;
        int flags = 0;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const long long m = m_att + static_cast<long long>(k) * kFillUnits;
          if (k < items && m >= u && m < e) flags |= 1 << k;
        }
        sg_tail = flags;
        sh_u = e;
      }
    }
    __syncthreads();
    const int b = sg_b;
    if (b < 0) break;
    // sub-pair sp of sequence b = (KV head h, column group grp); work pair index
    const int sp = sg_h, L = sg_L, t_a = sg_ta, t_e = sg_te;
    const int h = sp / p.ngrp, grp = sp - (sp / p.ngrp) * p.ngrp;
    const int pair = b * p.Hkv * p.ngrp + sp;
    // debug builds: the pair's record slot (pair + cta) lies in the workspace
    // (uniform across the CTA: every input is in shared memory or the launch)
    if (!debug_ok(b < p.B && sp < p.Hkv * p.ngrp && cta < kDecodeMaxCtas, p.status)) {
      ok = false;
      continue;
    }
    if (ok && t_a < t_e) {
      ok = decode_segment<KB, VB>(p, smem, b, h, grp, L, t_a, t_e, woff, rearm,
                                  p.ws + static_cast<int64_t>(pair + cta) * p.C * kPartialFloats);
      rearm = true;
      woff = (woff + (t_e - t_a) * DecodeTraits<KB, VB>::U) % kDWarps;
    }
    const int items = sg_tail;
    if (items & 1) {   // the pair's tail
      if (!seq_valid(p, L)) {
        if (tid == 0 && sp == 0) report_status(p.status, KVARN_DEV_BAD_SEQ_LEN);
      } else {
        decode_tail<KB, VB>(p, smem, b, h, grp, L);
      }
      __syncthreads();   // shared memory is free again
    }
#pragma unroll 1
    for (int side = 0; side < 2; ++side)
      if (items & (2 << side)) quantize_full_tail<KB, VB>(p, smem, b, h, L, side);
  }
  // the merge grid behind this one may launch once every CTA of this grid has
  // reached here (it waits for this grid's completion before reading any
  // record).  Triggering at the start instead let merge CTAs sit resident
  // beside running decode CTAs, which cost the quantise + decode step 7 us.
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// The merge (a10): two CTAs per work pair (sequence, KV head, column group),
// one per half of its columns, launched behind the decode grid as a
// programmatic dependent launch.  Its CTAs may become resident once every
// decode CTA has finished its range (the decode's trigger), before the decode
// grid has fully drained; each locates its pair's units from seq_lens (an
// input of the decode call, written before the decode grid started), then
// waits in griddepcontrol.wait, which returns once the decode grid has
// completed and its writes are visible, and merges the pair's records.
// P: the decode grid's CTA count (it fixes which CTAs wrote records for the
// pair).
__global__ void __launch_bounds__(kDThreads) merge_kernel(const __grid_constant__ DecodeArgs p, int P) {
  __shared__ long long sh_W, sh_pst;
  const int pair = blockIdx.x >> 1, half = blockIdx.x & 1;   // two CTAs per pair: column halves
  const int per_seq = p.Hkv * p.ngrp;
  const int b = pair / per_seq, sp = pair - (pair / per_seq) * per_seq;
  const int h = sp / p.ngrp, grp = sp - (sp / p.ngrp) * p.ngrp;
  const int L = p.seq_lens[b];
  const bool valid = seq_valid(p, L);
  if (threadIdx.x < 32) {   // total units W and the first unit of sequence b, by one warp
    const int lane = threadIdx.x;
    long long all = 0, before = 0;
    for (int s = lane; s < p.B; s += 32) {
      const int Ls = p.seq_lens[s];
      const long long u = static_cast<long long>(pair_units(p, Ls, seq_valid(p, Ls))) * per_seq;
      all += u;
      if (s < b) before += u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      all += __shfl_xor_sync(0xffffffffu, all, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    if (lane == 0) {
      sh_W = all;
      sh_pst = before + static_cast<long long>(sp) * pair_units(p, L, valid);
    }
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;\n" ::: "memory");   // the decode grid's records are complete
  combine_half(p, b, h, grp, half, L, valid, sh_pst, pair_tiles(L, valid), sh_W, P);
}


template <int KB, int VB>
cudaError_t launch_d(const DecodeArgs& p, cudaStream_t stream) {
  using T = DecodeTraits<KB, VB>;
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  static int ctas[64] = {};
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;   // one configured bit per ordinal
  const uint64_t bit = 1ull << dev;
  if ((configured.load(std::memory_order_acquire) & bit) == 0) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, T::kSmem);
    if (e != cudaSuccess) return e;
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int n = KVARN_D_MIN_CTAS * sms;
    ctas[dev] = n < 1 ? 1 : (n > kDecodeMaxCtas ? kDecodeMaxCtas : n);
    configured.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaError_t e = launch_pdl(decode_kernel<KB, VB>, dim3(ctas[dev]), dim3(kDThreads), static_cast<size_t>(T::kSmem),
                             stream, p);
  if (e != cudaSuccess) return e;
  const int pairs = p.B * p.Hkv * p.ngrp;
  if (pairs == 0) return cudaSuccess;
  return launch_pdl(merge_kernel, dim3(static_cast<unsigned>(2 * pairs)), dim3(kDThreads), 0, stream, p, ctas[dev]);
}

}  // namespace

// ------------------------------------------------------------------ fixed scratch
// Device-resident scratch for kvarn_decode_attention_noalloc: the stream-K
// partial records live in this file-scope array instead of a caller-supplied
// workspace.  Every GPU that loads the library holds these
// bytes until exit.  Its device address is looked up once per device ordinal
// and cached for the life of the process: after a reset of the device's
// primary context (cudaDeviceReset) the cached address is stale.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

cudaError_t noalloc_scratch(void** ptr, size_t* bytes) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    // once per device, with that device current: the symbol's device address
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  *bytes = kNoAllocScratchBytes;
  return cudaSuccess;
}

// Split-K geometry of the uncompressed baselines (baseline.cu).
void decode_geometry(int B, int Hkv, int max_blocks, int ctas_per_sm, int* tiles_per_split, int* num_splits) {
  // Tiles per split T (a multiple of the 4 warps) chosen to minimise
  // waves x (T / 4 tiles per warp + one tile of fixed cost), with
  // ctas_per_sm resident CTAs per SM on a 148-SM part; ties go to the larger T.
  const long pairs = B * Hkv > 0 ? static_cast<long>(B) * Hkv : 1;
  const long slots = static_cast<long>(ctas_per_sm > 0 ? ctas_per_sm : 1) * 148;
  int best_t = kDWarps;
  double best = 1e300;
  for (int T = kDWarps; T <= 64; T += kDWarps) {
    const long ns = (max_blocks + T - 1) / T;
    const long waves = (pairs * ns + slots - 1) / slots;
    const double cost = static_cast<double>(waves) * (T / static_cast<double>(kDWarps) + 1.0);
    if (cost <= best) {
      best = cost;
      best_t = T;
    }
    if (ns == 1) break;
  }
  int ns = (max_blocks + best_t - 1) / best_t;
  if (ns < 1) ns = 1;
  *tiles_per_split = best_t;
  *num_splits = ns;
}

size_t decode_workspace(int B, int Hq, int Hkv, int qlen) {
  if (Hkv <= 0 || qlen <= 0) return 0;
  const size_t cols = static_cast<size_t>(Hq / Hkv) * qlen;              // columns per (sequence, KV head)
  const size_t ngrp = (cols + kMaxG - 1) / kMaxG;
  const size_t C = cols < kMaxG ? cols : kMaxG;                           // records per column group
  const size_t pairs = static_cast<size_t>(B) * Hkv * ngrp;
  const size_t records = (pairs + kDecodeMaxCtas) * C + pairs * C;       // tile records, then tail records
  // then one reserved int32 word per work pair (kept so the size formula is stable)
  const size_t reserved = (pairs * sizeof(int32_t) + 15) & ~static_cast<size_t>(15);
  return records * kPartialFloats * sizeof(float) + reserved;
}

cudaError_t launch_decode(const DecodeArgs& p, cudaStream_t stream) {
#define KVARN_D_CASE(KB, VB) \
  if (p.kb == KB && p.vb == VB) return launch_d<KB, VB>(p, stream);
  KVARN_D_CASE(4, 2)
  KVARN_D_CASE(2, 2)
  KVARN_D_CASE(4, 4)
  KVARN_D_CASE(8, 8)
  KVARN_D_CASE(2, 4)
  KVARN_D_CASE(4, 8)
  KVARN_D_CASE(8, 4)
  KVARN_D_CASE(8, 2)
  KVARN_D_CASE(2, 8)
#undef KVARN_D_CASE
  return cudaErrorInvalidValue;
}

}  // namespace kvarn
