// kvarn_internal.h -- launch descriptors shared by the host layer and the kernels.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kvarn.h"

namespace kvarn {

struct QuantArgs {
  const __half* k;
  const __half* v;
  const int64_t* slot_mapping;
  int64_t num_groups;   // num_tokens / 128
  int hkv;
  int64_t num_blocks;
  uint8_t* packed;
  uint8_t* scales;
  int iters;
  int kb, vb;
  float* dbg;           // nullable: fp32 log-scales before rounding
  int32_t* status;      // nullable
};

// One split-K partial record: m, l, two pad words, acc[128]  (528 bytes).
constexpr int kPartialFloats = 132;

struct DecodeArgs {
  const __half* q;
  const uint8_t* packed;
  const uint8_t* scales;
  const __half* tail;
  const int32_t* block_table;
  const int32_t* seq_lens;
  __half* out;
  float* ws;            // tile partial records [(B * Hkv * ngrp + kDecodeMaxCtas) * C]
  float* ws_tail;       // tail partial records [B * Hkv * G]
  int* counters;        // B * Hkv reserved words of the workspace (unused by the decode)
  int B, Hq, Hkv, G, max_blocks;
  int64_t num_blocks;
  int kb, vb;
  float sm_scale;
  int32_t* status;
  // decode step with append (append = 1): seq_lens are the lengths before the
  // step; each (seq, KV head) first takes k_new / v_new ([B][Hkv][128]) as its
  // token at position seq_len, written to the fp16 tail; a tail that this
  // fills (128 tokens) is quantised into block block_table[seq][seq_len / 128]
  // multi-query (qlen > 1): q and out are [B][qlen][Hq][128]; query i of
  // sequence b sits at position seq_len - qlen + i and attends keys up to it.
  // A (sequence, KV head) pair's G * qlen columns (query, head) are processed
  // in ngrp groups of up to 8; C = min(8, G * qlen) records per group.
  int qlen, ngrp, C;
  int append;
  const __half* k_new;
  const __half* v_new;
  __half* tail_w;       // the same buffers as tail / packed / scales, written
  uint8_t* packed_w;
  uint8_t* scales_w;
  int iters;
};

// Stream-K decode: the work of all (sequence, KV head) pairs -- each pair's
// full tiles and one tail unit -- is cut into equal contiguous ranges, one per
// CTA of a grid of two CTAs per SM, at most kDecodeMaxCtas.  The workspace is a
// function of the dims only (never of seq_lens or the device).
constexpr int kDecodeMaxCtas = 320;
size_t decode_workspace(int B, int Hq, int Hkv, int qlen);

// Split-K geometry of the uncompressed baselines: a pure function of the dims.
// Split geometry of the uncompressed baselines, for ctas_per_sm resident CTAs
// per SM (kBaselineCtasPerSm[fp8]: the fp16 kernel's staging ring takes 128 KB
// of shared memory, the e4m3 one 32 KB).
void decode_geometry(int B, int Hkv, int max_blocks, int ctas_per_sm, int* tiles_per_split, int* num_splits);
constexpr int kBaselineCtasPerSm[2] = {2, 4};

cudaError_t launch_quantize(const QuantArgs& p, cudaStream_t stream);

// Fixed device scratch of kvarn_decode_attention_noalloc (KVARN_NOALLOC_SCRATCH_BYTES).
constexpr size_t kNoAllocScratchBytes = KVARN_NOALLOC_SCRATCH_BYTES;
// Device address and size of that scratch on the current device; the first
// call on a device looks the address up (cudaGetSymbolAddress) and caches it.
cudaError_t noalloc_scratch(void** ptr, size_t* bytes);
cudaError_t launch_decode(const DecodeArgs& p, cudaStream_t stream);

struct BaselineArgs {
  const __half* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  __half* out;
  float* ws;            // partial records, then the per-(seq, KV head) counters
  int* counters;
  int B, Hq, Hkv, G, max_blocks;
  int64_t num_blocks;
  int tiles_per_split, num_splits;
  float sm_scale, k_scale, v_scale;
  int fp8;               // 0 = fp16 cache, 1 = e4m3 cache
  int32_t* status;
};

cudaError_t launch_baseline(const BaselineArgs& p, cudaStream_t stream);

}  // namespace kvarn
