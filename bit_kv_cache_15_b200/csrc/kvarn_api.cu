// kvarn_api.cu -- the extern "C" boundary of libkvarn.so.
//
// Every entry point validates its arguments on the host, then enqueues the
// kernels on the caller's stream and returns; nothing here allocates,
// synchronises or keeps state.  The user-facing configuration string and
// block size follow [hypho] "KV-cache 量化终于能跑生产了？KVarN …", section
// 工程实践：一行配置启用 (kv_cache_dtype="kvarn_k4v2_g128", block_size=128)
// and [lehuy] "KVarN: Backend lượng tử hóa KV-cache …", section Dễ dàng tích
// hợp và sử dụng (block_size 128 is the KVarN tile size).
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../include/kvarn.h"
#include "kvarn_internal.h"

// NVTX ranges around every call that enqueues GPU work, so a timeline tool
// shows which library call launched which kernels (header-only NVTX 3: with
// no tool attached a range costs a null check).  -DKVARN_NVTX=0 removes them.
#ifndef KVARN_NVTX
#define KVARN_NVTX 1
#endif
#if KVARN_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace {

struct NvtxRange {
#if KVARN_NVTX
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
#else
  explicit NvtxRange(const char*) {}
#endif
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

bool bits_ok(int b) { return b == 2 || b == 4 || b == 8; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float effective_sm_scale(const kvarn_config* cfg) {
  return cfg->sm_scale > 0.f ? cfg->sm_scale : 1.0f / std::sqrt(static_cast<float>(KVARN_HEAD_DIM));
}

kvarn_status check_dims(const kvarn_decode_dims* dims, int max_group) {
  if (dims == nullptr) return KVARN_ERR_INVALID_ARGUMENT;
  if (dims->num_seqs < 0 || dims->num_q_heads <= 0 || dims->num_kv_heads <= 0 ||
      dims->max_blocks_per_seq <= 0 || dims->num_blocks < 0)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (dims->num_q_heads % dims->num_kv_heads != 0) return KVARN_ERR_INVALID_ARGUMENT;
  if (dims->num_q_heads / dims->num_kv_heads > max_group) return KVARN_ERR_UNSUPPORTED;
  if (dims->num_kv_heads > 65535 || dims->num_seqs > 65535) return KVARN_ERR_UNSUPPORTED;
  return KVARN_OK;
}

kvarn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVARN_OK : KVARN_ERR_CUDA; }

size_t partial_bytes(int B, int Hq, int Hkv, int max_blocks) {
  // room for the splits of either baseline's geometry
  int ns_max = 0;
  for (int fp8 = 0; fp8 < 2; ++fp8) {
    int T = 0, ns = 0;
    kvarn::decode_geometry(B, Hkv, max_blocks, kvarn::kBaselineCtasPerSm[fp8], &T, &ns);
    ns_max = ns > ns_max ? ns : ns_max;
  }
  return static_cast<size_t>(B) * Hq * (ns_max + 1) * kvarn::kPartialFloats * sizeof(float);
}

// Uncompressed baselines: split-K partial records followed by B * Hkv int32
// arrival counters (rounded to 16 bytes).
size_t workspace_for(int B, int Hq, int Hkv, int max_blocks) {
  const size_t counters = (static_cast<size_t>(B) * Hkv * sizeof(int32_t) + 15) & ~static_cast<size_t>(15);
  return partial_bytes(B, Hq, Hkv, max_blocks) + counters;
}

kvarn_status quantize_impl(const void* k, const void* v, const int64_t* slot_mapping, int64_t num_tokens,
                           int32_t num_kv_heads, int64_t num_blocks, void* packed_cache, void* scales,
                           const kvarn_config* cfg, float* dbg, int32_t* dev_status, void* stream) {
  kvarn_status st = kvarn_config_validate(cfg);
  if (st != KVARN_OK) return st;
  if (num_tokens < 0 || num_tokens % KVARN_TILE_TOKENS != 0 || num_kv_heads <= 0 || num_blocks < 0)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (num_tokens == 0) return KVARN_OK;
  if (k == nullptr || v == nullptr || slot_mapping == nullptr || packed_cache == nullptr || scales == nullptr)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (!aligned16(k) || !aligned16(v) || !aligned16(packed_cache) || !aligned16(scales))
    return KVARN_ERR_INVALID_ARGUMENT;
  if (num_kv_heads > 65535 || num_tokens / KVARN_TILE_TOKENS > 0x7fffffffLL) return KVARN_ERR_UNSUPPORTED;
  kvarn::QuantArgs p;
  p.k = static_cast<const __half*>(k);
  p.v = static_cast<const __half*>(v);
  p.slot_mapping = slot_mapping;
  p.num_groups = num_tokens / KVARN_TILE_TOKENS;
  p.hkv = num_kv_heads;
  p.num_blocks = num_blocks;
  p.packed = static_cast<uint8_t*>(packed_cache);
  p.scales = static_cast<uint8_t*>(scales);
  p.iters = cfg->sinkhorn_iters;
  p.kb = cfg->k_bits;
  p.vb = cfg->v_bits;
  p.dbg = dbg;
  p.status = dev_status;
  return from_cuda(kvarn::launch_quantize(p, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

kvarn_status kvarn_config_validate(const kvarn_config* cfg) {
  if (cfg == nullptr) return KVARN_ERR_INVALID_ARGUMENT;
  if (cfg->version != KVARN_ABI_VERSION) return KVARN_ERR_UNSUPPORTED;
  if (!bits_ok(cfg->k_bits) || !bits_ok(cfg->v_bits)) return KVARN_ERR_UNSUPPORTED;
  if (cfg->tile_tokens != KVARN_TILE_TOKENS || cfg->head_dim != KVARN_HEAD_DIM) return KVARN_ERR_UNSUPPORTED;
  if (cfg->layout != 0 || cfg->flags != 0) return KVARN_ERR_UNSUPPORTED;
  if (cfg->sinkhorn_iters < 1 || cfg->sinkhorn_iters > 1000) return KVARN_ERR_INVALID_ARGUMENT;
  if (!(cfg->sm_scale >= 0.f) || std::isinf(cfg->sm_scale)) return KVARN_ERR_INVALID_ARGUMENT;
  return KVARN_OK;
}

kvarn_status kvarn_config_from_string(const char* s, kvarn_config* out) {
  if (s == nullptr || out == nullptr) return KVARN_ERR_INVALID_ARGUMENT;
  int kb = 0, vb = 0, g = 0, n = 0;
  if (std::sscanf(s, "kvarn_k%dv%d_g%d%n", &kb, &vb, &g, &n) != 3 || s[n] != '\0')
    return KVARN_ERR_INVALID_ARGUMENT;
  if (!bits_ok(kb) || !bits_ok(vb) || g != KVARN_TILE_TOKENS) return KVARN_ERR_UNSUPPORTED;
  std::memset(out, 0, sizeof(*out));
  out->version = KVARN_ABI_VERSION;
  out->k_bits = kb;
  out->v_bits = vb;
  out->tile_tokens = KVARN_TILE_TOKENS;
  out->head_dim = KVARN_HEAD_DIM;
  out->sinkhorn_iters = 8;
  out->layout = 0;
  out->flags = 0;
  out->sm_scale = 0.f;
  return KVARN_OK;
}

size_t kvarn_cache_bytes_per_block(const kvarn_config* cfg, int32_t num_kv_heads) {
  if (kvarn_config_validate(cfg) != KVARN_OK || num_kv_heads <= 0) return 0;
  return static_cast<size_t>(num_kv_heads) * 2048u * static_cast<size_t>(cfg->k_bits + cfg->v_bits);
}

size_t kvarn_scale_bytes_per_block(int32_t num_kv_heads) {
  if (num_kv_heads <= 0) return 0;
  return static_cast<size_t>(num_kv_heads) * 2u * KVARN_SCALE_RECORD_BYTES;
}

size_t kvarn_decode_workspace_bytes(const kvarn_config* cfg, const kvarn_decode_dims* dims) {
  if (kvarn_config_validate(cfg) != KVARN_OK || check_dims(dims, 8) != KVARN_OK) return 0;
  return kvarn::decode_workspace(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, 1);
}

kvarn_status kvarn_quantize_tiles(const void* k, const void* v, const int64_t* slot_mapping, int64_t num_tokens,
                                  int32_t num_kv_heads, int64_t num_blocks, void* packed_cache, void* scales,
                                  const kvarn_config* cfg, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_quantize_tiles");
  return quantize_impl(k, v, slot_mapping, num_tokens, num_kv_heads, num_blocks, packed_cache, scales, cfg,
                       nullptr, dev_status, stream);
}

kvarn_status kvarn_quantize_tiles_debug(const void* k, const void* v, const int64_t* slot_mapping,
                                        int64_t num_tokens, int32_t num_kv_heads, int64_t num_blocks,
                                        void* packed_cache, void* scales, const kvarn_config* cfg,
                                        float* debug_logscales, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_quantize_tiles_debug");
  if (debug_logscales == nullptr && num_tokens > 0) return KVARN_ERR_INVALID_ARGUMENT;
  return quantize_impl(k, v, slot_mapping, num_tokens, num_kv_heads, num_blocks, packed_cache, scales, cfg,
                       debug_logscales, dev_status, stream);
}

static kvarn_status decode_impl(const void* q, const void* k_new, const void* v_new, const void* packed_cache,
                                const void* scales, const void* fp16_tail, const int32_t* block_table,
                                const int32_t* seq_lens, void* out, const kvarn_decode_dims* dims,
                                const kvarn_config* cfg, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                void* stream, int append, int32_t q_len) {
  kvarn_status st = kvarn_config_validate(cfg);
  if (st != KVARN_OK) return st;
  st = check_dims(dims, 8);
  if (st != KVARN_OK) return st;
  if (dims->num_seqs == 0) return KVARN_OK;
  if (q == nullptr || packed_cache == nullptr || scales == nullptr || fp16_tail == nullptr ||
      block_table == nullptr || seq_lens == nullptr || out == nullptr || workspace == nullptr)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(packed_cache) || !aligned16(scales) || !aligned16(fp16_tail) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(out) & 7u) != 0)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (append && (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new)))
    return KVARN_ERR_INVALID_ARGUMENT;
  if (q_len < 1 || q_len > KVARN_MAX_Q_LEN || (append && q_len != 1)) return KVARN_ERR_INVALID_ARGUMENT;
  const size_t need = kvarn::decode_workspace(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, q_len);
  if (workspace_bytes < need) return KVARN_ERR_WORKSPACE_TOO_SMALL;
  kvarn::DecodeArgs p;
  p.q = static_cast<const __half*>(q);
  p.packed = static_cast<const uint8_t*>(packed_cache);
  p.scales = static_cast<const uint8_t*>(scales);
  p.tail = static_cast<const __half*>(fp16_tail);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__half*>(out);
  {   // tile records, tail records, reserved words; per (sequence, KV head) the
      // G * q_len (query, head) columns form groups of up to 8
    const int cols = (dims->num_q_heads / dims->num_kv_heads) * q_len;
    p.qlen = q_len;
    p.ngrp = (cols + 7) / 8;
    p.C = cols < 8 ? cols : 8;
    const size_t pairs = static_cast<size_t>(dims->num_seqs) * dims->num_kv_heads * p.ngrp;
    float* ws = static_cast<float*>(workspace);
    p.ws = ws;
    p.ws_tail = ws + (pairs + kvarn::kDecodeMaxCtas) * p.C * kvarn::kPartialFloats;
    p.counters = reinterpret_cast<int*>(p.ws_tail + pairs * p.C * kvarn::kPartialFloats);
  }
  p.B = dims->num_seqs;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.G = dims->num_q_heads / dims->num_kv_heads;
  p.max_blocks = dims->max_blocks_per_seq;
  p.num_blocks = dims->num_blocks;
  p.kb = cfg->k_bits;
  p.vb = cfg->v_bits;
  p.sm_scale = effective_sm_scale(cfg);
  p.status = dev_status;
  p.append = append;
  p.k_new = static_cast<const __half*>(k_new);
  p.v_new = static_cast<const __half*>(v_new);
  p.tail_w = append ? static_cast<__half*>(const_cast<void*>(fp16_tail)) : nullptr;
  p.packed_w = append ? static_cast<uint8_t*>(const_cast<void*>(packed_cache)) : nullptr;
  p.scales_w = append ? static_cast<uint8_t*>(const_cast<void*>(scales)) : nullptr;
  p.iters = cfg->sinkhorn_iters;
  return from_cuda(kvarn::launch_decode(p, static_cast<cudaStream_t>(stream)));
}

kvarn_status kvarn_decode_attention(const void* q, const void* packed_cache, const void* scales,
                                    const void* fp16_tail, const int32_t* block_table, const int32_t* seq_lens,
                                    void* out, const kvarn_decode_dims* dims, const kvarn_config* cfg,
                                    void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention");
  return decode_impl(q, nullptr, nullptr, packed_cache, scales, fp16_tail, block_table, seq_lens, out, dims, cfg,
                     workspace, workspace_bytes, dev_status, stream, 0, 1);
}

size_t kvarn_decode_multiquery_workspace_bytes(const kvarn_config* cfg, const kvarn_decode_dims* dims,
                                               int32_t q_len) {
  if (kvarn_config_validate(cfg) != KVARN_OK || check_dims(dims, 8) != KVARN_OK) return 0;
  if (q_len < 1 || q_len > KVARN_MAX_Q_LEN) return 0;
  return kvarn::decode_workspace(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, q_len);
}

kvarn_status kvarn_decode_attention_multiquery(const void* q, int32_t q_len, const void* packed_cache,
                                               const void* scales, const void* fp16_tail, const int32_t* block_table,
                                               const int32_t* seq_lens, void* out, const kvarn_decode_dims* dims,
                                               const kvarn_config* cfg, void* workspace, size_t workspace_bytes,
                                               int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention_multiquery");
  return decode_impl(q, nullptr, nullptr, packed_cache, scales, fp16_tail, block_table, seq_lens, out, dims, cfg,
                     workspace, workspace_bytes, dev_status, stream, 0, q_len);
}

kvarn_status kvarn_decode_attention_append(const void* q, const void* k_new, const void* v_new, void* packed_cache,
                                           void* scales, void* fp16_tail, const int32_t* block_table,
                                           const int32_t* seq_lens, void* out, const kvarn_decode_dims* dims,
                                           const kvarn_config* cfg, void* workspace, size_t workspace_bytes,
                                           int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention_append");
  return decode_impl(q, k_new, v_new, packed_cache, scales, fp16_tail, block_table, seq_lens, out, dims, cfg,
                     workspace, workspace_bytes, dev_status, stream, 1, 1);
}

kvarn_status kvarn_decode_attention_noalloc(const void* q, const void* packed_cache, const void* scales,
                                            const void* fp16_tail, const int32_t* block_table,
                                            const int32_t* seq_lens, void* out, const kvarn_decode_dims* dims,
                                            const kvarn_config* cfg, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention_noalloc");
  // Same path as kvarn_decode_attention, with the library's fixed device
  // scratch standing in for the caller's workspace.
  kvarn_status st = kvarn_config_validate(cfg);
  if (st != KVARN_OK) return st;
  st = check_dims(dims, 8);
  if (st != KVARN_OK) return st;
  if (dims->num_seqs == 0) return KVARN_OK;
  const size_t need = kvarn::decode_workspace(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, 1);
  if (need > kvarn::kNoAllocScratchBytes) return KVARN_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (kvarn::noalloc_scratch(&scratch, &scratch_bytes) != cudaSuccess) return KVARN_ERR_CUDA;
  return kvarn_decode_attention(q, packed_cache, scales, fp16_tail, block_table, seq_lens, out, dims, cfg, scratch,
                                scratch_bytes, dev_status, stream);
}

size_t kvarn_baseline_workspace_bytes(const kvarn_decode_dims* dims) {
  if (check_dims(dims, 8) != KVARN_OK) return 0;
  return workspace_for(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, dims->max_blocks_per_seq);
}

static kvarn_status baseline_impl(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                                  const int32_t* seq_lens, void* out, const kvarn_decode_dims* dims, float sm_scale,
                                  float k_scale, float v_scale, int fp8, void* workspace, size_t workspace_bytes,
                                  int32_t* dev_status, void* stream) {
  kvarn_status st = check_dims(dims, 8);
  if (st != KVARN_OK) return st;
  if (dims->num_seqs == 0) return KVARN_OK;
  if (q == nullptr || k_cache == nullptr || v_cache == nullptr || block_table == nullptr || seq_lens == nullptr ||
      out == nullptr || workspace == nullptr)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(out) & 7u) != 0)
    return KVARN_ERR_INVALID_ARGUMENT;
  if (!(sm_scale >= 0.f) || std::isinf(sm_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
    return KVARN_ERR_INVALID_ARGUMENT;
  const size_t need = workspace_for(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads, dims->max_blocks_per_seq);
  if (workspace_bytes < need) return KVARN_ERR_WORKSPACE_TOO_SMALL;
  kvarn::BaselineArgs p;
  p.q = static_cast<const __half*>(q);
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__half*>(out);
  p.ws = static_cast<float*>(workspace);
  p.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) +
                                      partial_bytes(dims->num_seqs, dims->num_q_heads, dims->num_kv_heads,
                                                    dims->max_blocks_per_seq));
  p.B = dims->num_seqs;
  p.Hq = dims->num_q_heads;
  p.Hkv = dims->num_kv_heads;
  p.G = dims->num_q_heads / dims->num_kv_heads;
  p.max_blocks = dims->max_blocks_per_seq;
  p.num_blocks = dims->num_blocks;
  kvarn::decode_geometry(p.B, p.Hkv, p.max_blocks, kvarn::kBaselineCtasPerSm[fp8 ? 1 : 0], &p.tiles_per_split,
                         &p.num_splits);
  p.sm_scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(KVARN_HEAD_DIM));
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.fp8 = fp8;
  p.status = dev_status;
  return from_cuda(kvarn::launch_baseline(p, static_cast<cudaStream_t>(stream)));
}

kvarn_status kvarn_decode_attention_fp16(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens, void* out,
                                         const kvarn_decode_dims* dims, float sm_scale, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention_fp16");
  return baseline_impl(q, k_cache, v_cache, block_table, seq_lens, out, dims, sm_scale, 1.f, 1.f, 0, workspace,
                       workspace_bytes, dev_status, stream);
}

kvarn_status kvarn_decode_attention_fp8(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_table, const int32_t* seq_lens, void* out,
                                        const kvarn_decode_dims* dims, float sm_scale, float k_scale, float v_scale,
                                        void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream) {
  const NvtxRange nvtx_range("kvarn_decode_attention_fp8");
  return baseline_impl(q, k_cache, v_cache, block_table, seq_lens, out, dims, sm_scale, k_scale, v_scale, 1,
                       workspace, workspace_bytes, dev_status, stream);
}

const char* kvarn_status_string(kvarn_status s) {
  switch (s) {
    case KVARN_OK: return "KVARN_OK";
    case KVARN_ERR_INVALID_ARGUMENT: return "KVARN_ERR_INVALID_ARGUMENT";
    case KVARN_ERR_UNSUPPORTED: return "KVARN_ERR_UNSUPPORTED";
    case KVARN_ERR_CUDA: return "KVARN_ERR_CUDA";
    case KVARN_ERR_WORKSPACE_TOO_SMALL: return "KVARN_ERR_WORKSPACE_TOO_SMALL";
  }
  return "KVARN_ERR_UNKNOWN";
}

int32_t kvarn_abi_version(void) { return KVARN_ABI_VERSION; }

}  // extern "C"
