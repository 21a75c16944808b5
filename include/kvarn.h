/*
 * kvarn.h -- C ABI of the KVarN hot path on NVIDIA B200 (sm_100a).
 *
 * KVarN (variance-normalised KV cache) quantises each 128-token x 128-channel
 * fp16 K or V tile in four stages -- the raw tile, a Hadamard rotation along
 * channels, alternating row/column RMS normalisation in log space
 * (Sinkhorn-like), asymmetric low-bit round-to-nearest -- and folds the scales
 * back in when attention reads the cache.
 *   [hypho] "KV-cache 量化终于能跑生产了？KVarN 用方差归一化打破 vLLM 的吞吐量魔咒"
 *           (blog.hypho.cn), section "它怎么做到的：四步流水线" steps 1-4, and
 *           "工程实践：一行配置启用" (kv_cache_dtype="kvarn_k4v2_g128",
 *           block_size=128, no calibration data).
 *   [lehuy] "KVarN: Backend lượng tử hóa KV-cache gốc của Huawei giúp vLLM tăng
 *           hiệu suất vượt trội" (lehuy.net), section "Cơ chế hoạt động: Chuẩn
 *           hóa phương sai" (stages 1-4; scale factors merged when read) and
 *           "Dễ dàng tích hợp và sử dụng" (block_size 128 is the tile size).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers the caller allocated; the library
 *    allocates no memory and keeps no state between calls.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.  Calls are reentrant.
 *  - The kernels are programmatic dependent launches: a kernel's CTAs may
 *    become resident before the previous kernel in the stream has finished
 *    and do their on-chip set-up, but each waits for that kernel's completion
 *    (griddepcontrol.wait) before its first global-memory access, so stream
 *    order holds against any earlier work.  They work inside CUDA graph
 *    capture as well.
 *  - Each kernel's launch set-up (its shared-memory attribute and grid size)
 *    is done once per device ordinal (ordinals 0-63; others get
 *    KVARN_ERR_CUDA) and kept for the process; a reset of the device's primary
 *    context (cudaDeviceReset) is not supported while the library is in use.
 *  - Argument and shape errors are found on the host and returned before any
 *    launch.  A launch failure returns KVARN_ERR_CUDA.
 *  - Data-dependent faults found on the device (a slot or block id out of
 *    range, a wait that timed out) are written to *dev_status (a device int32
 *    the caller zeroes; NULL = not reported) as one of the KVARN_DEV_* codes,
 *    first error wins; the offending work item is skipped.  Kernels never trap.
 *  - NaN/Inf inputs are the caller's error; results are then unspecified.
 *  - No C++ exception crosses this interface.
 * All multi-byte values are little-endian.  Pointers to packed caches, scales
 * and workspaces must be 16-byte aligned.
 */
#ifndef KVARN_H_
#define KVARN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KVARN_API __attribute__((visibility("default")))
#else
#define KVARN_API
#endif

#define KVARN_ABI_VERSION 1
#define KVARN_TILE_TOKENS 128
#define KVARN_HEAD_DIM 128
#define KVARN_MAX_Q_LEN 128   /* queries per sequence of kvarn_decode_attention_multiquery */
/* bytes of one scale record (per block, KV head and K-or-V):
 * fp16 lt[128] | fp16 lc[128] | fp32 zero | fp32 step | 8 B pad */
#define KVARN_SCALE_RECORD_BYTES 528

typedef enum {
  KVARN_OK = 0,
  KVARN_ERR_INVALID_ARGUMENT = 1,  /* null pointer, bad count, misaligned pointer */
  KVARN_ERR_UNSUPPORTED = 2,       /* bits not in {2,4,8}, head_dim/tile != 128, Hq/Hkv > 8 */
  KVARN_ERR_CUDA = 3,              /* a CUDA launch or query failed */
  KVARN_ERR_WORKSPACE_TOO_SMALL = 4
} kvarn_status;

/* device-side status codes written to *dev_status */
#define KVARN_DEV_OK 0
#define KVARN_DEV_BAD_SLOT 1       /* slot_mapping entry misaligned or beyond the pool */
#define KVARN_DEV_BAD_BLOCK 2      /* block_table entry beyond the pool */
#define KVARN_DEV_BAD_SEQ_LEN 3    /* seq_len < 0 or > 128 * max_blocks_per_seq */
#define KVARN_DEV_TIMEOUT 4        /* a bounded wait on an asynchronous copy gave up */
#define KVARN_DEV_INTERNAL 5       /* debug builds (KVARN_DEBUG=1) only: one of the kernels' own
                                      index checks failed, i.e. a library defect; the access it
                                      guards was skipped, so the outputs of that call are invalid */

typedef struct {
  int32_t version;         /* KVARN_ABI_VERSION */
  int32_t k_bits;          /* 2, 4 or 8 */
  int32_t v_bits;          /* 2, 4 or 8 */
  int32_t tile_tokens;     /* 128 (the only supported tile) */
  int32_t head_dim;        /* 128 (the only supported head size) */
  int32_t sinkhorn_iters;  /* normalisation iterations, >= 1 (default 8) */
  int32_t layout;          /* 0 = mma-fragment code order (the only one) */
  int32_t flags;           /* reserved, 0 */
  float sm_scale;          /* softmax scale; 0 means 1/sqrt(head_dim) */
} kvarn_config;

typedef struct {
  int32_t num_seqs;            /* B */
  int32_t num_q_heads;         /* Hq, a multiple of Hkv with Hq / Hkv <= 8 */
  int32_t num_kv_heads;        /* Hkv */
  int32_t max_blocks_per_seq;  /* row length of block_table */
  int64_t num_blocks;          /* blocks in the paged pool */
} kvarn_decode_dims;

/* Parse "kvarn_k{kb}v{vb}_g128" ([hypho] 工程实践：一行配置启用) into *out with
 * the defaults (8 iterations, sm_scale 0).  Returns INVALID_ARGUMENT if the
 * string does not parse, UNSUPPORTED for bits outside {2,4,8} or g != 128. */
KVARN_API kvarn_status kvarn_config_from_string(const char* s, kvarn_config* out);

/* Check a configuration (what every call checks first). */
KVARN_API kvarn_status kvarn_config_validate(const kvarn_config* cfg);

/* Bytes of packed codes per paged block: num_kv_heads * 2048 * (k_bits + v_bits).
 * Returns 0 for an invalid configuration. */
KVARN_API size_t kvarn_cache_bytes_per_block(const kvarn_config* cfg, int32_t num_kv_heads);

/* Bytes of scales per paged block: num_kv_heads * 2 * 528. */
KVARN_API size_t kvarn_scale_bytes_per_block(int32_t num_kv_heads);

/* Bytes of decode workspace needed for these dims: 528-byte partial records
 * ((B*Hkv + 320) * G for runs of full tiles, B*Hkv*G for the fp16 tails;
 * 320 bounds the decode grid) followed by one reserved int32 word per
 * (sequence, KV head).  Depends only on cfg and dims (not on seq_lens,
 * max_blocks or the device).  Its contents need no initialisation: every
 * record a call reads is written earlier in the same call (the decode grid
 * writes the partial records, the merge grid launched behind it reads them). */
KVARN_API size_t kvarn_decode_workspace_bytes(const kvarn_config* cfg, const kvarn_decode_dims* dims);

/* Quantise-on-write of whole 128-token tiles ([hypho] 四步流水线 steps 1-4;
 * [lehuy] Cơ chế hoạt động stages 1-4).
 *
 *  k, v          fp16 [num_tokens][num_kv_heads][128], row-major, contiguous.
 *  slot_mapping  int64 [num_tokens]; token group g = rows [128g, 128g+128)
 *                goes to paged block slot_mapping[128g] / 128, which must be
 *                a multiple of 128 and < 128 * num_blocks (the other 127
 *                entries of the group are assumed to follow it).
 *  num_tokens    a multiple of 128 (0 allowed: nothing is launched).
 *  packed_cache  uint8 [num_blocks][num_kv_heads][2048*(k_bits+v_bits)].
 *  scales        uint8 [num_blocks][num_kv_heads][2][528].
 * Each (group, head, K|V) tile: R = X H (Sylvester Hadamard, unnormalised);
 * sinkhorn_iters passes of channel then token RMS normalisation in base-2 log
 * space; log-scales stored fp16; Z = (R*2^-Lt)*2^-Lc in fp32; one zero/step
 * per tile from min/max; codes = clamp(rne((Z-zero)/step)), the quotient taken
 * in fp32 as Z*(1/step) - zero*(1/step), packed in the mma-fragment order.  Groups whose slot is invalid are skipped and reported
 * as KVARN_DEV_BAD_SLOT. */
KVARN_API kvarn_status kvarn_quantize_tiles(const void* k, const void* v, const int64_t* slot_mapping,
                                  int64_t num_tokens, int32_t num_kv_heads, int64_t num_blocks,
                                  void* packed_cache, void* scales, const kvarn_config* cfg,
                                  int32_t* dev_status, void* stream);

/* Same as kvarn_quantize_tiles, and also writes each tile's fp32 log-scales
 * before fp16 rounding to debug_logscales: float [num_tokens/128][num_kv_heads]
 * [2 (K,V)][256] = lt[128] then lc[128].  For parity testing. */
KVARN_API kvarn_status kvarn_quantize_tiles_debug(const void* k, const void* v, const int64_t* slot_mapping,
                                        int64_t num_tokens, int32_t num_kv_heads, int64_t num_blocks,
                                        void* packed_cache, void* scales, const kvarn_config* cfg,
                                        float* debug_logscales, int32_t* dev_status, void* stream);

/* Paged decode attention on the packed cache, scales folded on read
 * ([lehuy] Cơ chế hoạt động stage 4; [hypho] 四步流水线 step 4).
 *
 *  q            fp16 [B][Hq][128].
 *  packed_cache, scales  as written by kvarn_quantize_tiles.
 *  fp16_tail    fp16 [B][2 (K,V)][Hkv][128][128]: rows [0, seq_len % 128) of
 *               sequence b hold its partial last tile, unquantised.
 *  block_table  int32 [B][max_blocks_per_seq]; entry i < seq_len/128 is the
 *               paged block of full tile i.
 *  seq_lens     int32 [B]: full tiles * 128 + tail tokens (read on the device
 *               only; the host never synchronises).
 *  out          fp16 [B][Hq][128]; sequence b, q head j attends with KV head
 *               j / (Hq/Hkv).  A zero-length sequence gets 0.
 *  workspace    device scratch of at least kvarn_decode_workspace_bytes();
 *               calls that share a workspace must not overlap on the GPU.
 * Key side: q H is multiplied by the per-channel scales, the per-token scales
 * multiply the scores; value side: the per-token scales multiply the softmax
 * weights, the per-channel scales and H/128 apply to the output. */
KVARN_API kvarn_status kvarn_decode_attention(const void* q, const void* packed_cache, const void* scales,
                                    const void* fp16_tail, const int32_t* block_table,
                                    const int32_t* seq_lens, void* out,
                                    const kvarn_decode_dims* dims, const kvarn_config* cfg,
                                    void* workspace, size_t workspace_bytes,
                                    int32_t* dev_status, void* stream);

/* One decode step that first appends each sequence's new token: the step
 * before the path in a serving loop (the cache grows by one token per
 * sequence per step).  The pages keep the newest tokens of a sequence
 * unquantised until a whole 128-token tile exists and then quantise that tile
 * ([lehuy] Cơ chế hoạt động: fixed 128-token tiles; [hypho] 需要关注的几个问题
 * item 3: block size 128); this call does both in the decode kernel.
 *
 *  k_new, v_new  fp16 [B][Hkv][128]: the step's token of sequence b.
 *  seq_lens      int32 [B]: lengths BEFORE the step (L).  The call does not
 *                change them: the caller adds 1 afterwards.
 *  fp16_tail, packed_cache, scales   read and written (see below).
 *  Other arguments as kvarn_decode_attention; workspace size is the same.
 * For each sequence b and KV head h:
 *  - the output attends L + 1 tokens: the full tiles i < L/128 from the
 *    packed cache and rows [0, L % 128] of the fp16 tail, where row L % 128
 *    is the new token (read from k_new / v_new);
 *  - the new token is written to row L % 128 of the fp16 tail;
 *  - if L % 128 == 127 (the tail is now a full tile), the tail tile is
 *    quantised exactly as kvarn_quantize_tiles would (same config and
 *    iterations) into block block_table[b][L / 128] (codes and scale records
 *    of head h).  That block must not be read by any sequence in the same
 *    call.  After the caller sets seq_len = L + 1, the next call reads that
 *    tile from the packed cache and the tail is empty.
 * Requires L + 1 <= 128 * max_blocks_per_seq (else KVARN_DEV_BAD_SEQ_LEN,
 * output 0, nothing written for b); a block id outside [0, num_blocks) for
 * the filled tile is reported as KVARN_DEV_BAD_BLOCK and nothing is quantised. */
KVARN_API kvarn_status kvarn_decode_attention_append(const void* q, const void* k_new, const void* v_new,
                                                     void* packed_cache, void* scales, void* fp16_tail,
                                                     const int32_t* block_table, const int32_t* seq_lens, void* out,
                                                     const kvarn_decode_dims* dims, const kvarn_config* cfg,
                                                     void* workspace, size_t workspace_bytes,
                                                     int32_t* dev_status, void* stream);

/* Multi-query attention over the packed cache: q_len query tokens per
 * sequence, each attending causally -- the shape of a speculative-decoding
 * verify step or a chunk of chunked prefill.  The pages quote first-token
 * latency (openai-hub.com/news/593, "华为云开源 KVarN：vLLM 原生 KV 缓存量化
 * 后端", section 对开发者意味着什么: 180 -> 120 ms) but give no kernel for
 * it; this is the decode path with (query, head) columns in place of heads.
 *
 *  q      fp16 [B][q_len][Hq][128]: query i of sequence b sits at position
 *         seq_len - q_len + i and attends keys [0, seq_len - q_len + i].
 *  out    fp16 [B][q_len][Hq][128].
 *  The q_len tokens' own K/V must already be in the cache -- in the fp16 tail
 *  or, once a tile of 128 has filled, in the packed tile (which is then read
 *  with a per-query causal mask); seq_len counts them.
 *  Other arguments as kvarn_decode_attention.
 *  workspace  at least kvarn_decode_multiquery_workspace_bytes(cfg, dims, q_len).
 * Requires 1 <= q_len <= KVARN_MAX_Q_LEN and seq_len >= q_len; as q_len <= 128,
 * the queries reach back at most into the last full tile.  With q_len > 1 a
 * sequence with seq_len < q_len is reported as KVARN_DEV_BAD_SEQ_LEN and its
 * outputs are 0.  q_len = 1 is exactly kvarn_decode_attention (an empty
 * sequence gives 0 and no status). */
KVARN_API size_t kvarn_decode_multiquery_workspace_bytes(const kvarn_config* cfg, const kvarn_decode_dims* dims,
                                                         int32_t q_len);

KVARN_API kvarn_status kvarn_decode_attention_multiquery(const void* q, int32_t q_len, const void* packed_cache,
                                                         const void* scales, const void* fp16_tail,
                                                         const int32_t* block_table, const int32_t* seq_lens,
                                                         void* out, const kvarn_decode_dims* dims,
                                                         const kvarn_config* cfg, void* workspace,
                                                         size_t workspace_bytes, int32_t* dev_status, void* stream);

/* Size of the fixed device scratch used by kvarn_decode_attention_noalloc. */
#define KVARN_NOALLOC_SCRATCH_BYTES (8u << 20)

/* kvarn_decode_attention without a workspace argument: the call allocates
 * nothing.  (The pages have no counterpart; this is a convenience of this
 * library.)  It is meant for callers that cannot allocate device memory
 * themselves -- for instance code running inside another framework's step
 * that owns all allocations, or a host thread that must not call cudaMalloc
 * because that can synchronise the device.  The partial-record scratch is instead a
 * file-scope __device__ array of KVARN_NOALLOC_SCRATCH_BYTES (8 MiB) that
 * every GPU loading this library keeps until the process exits.
 *  - Same arguments and results as kvarn_decode_attention, minus workspace.
 *  - If the problem needs more scratch than that (kvarn_decode_workspace_bytes
 *    > KVARN_NOALLOC_SCRATCH_BYTES) the call returns
 *    KVARN_ERR_WORKSPACE_TOO_SMALL and launches nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it for the
 *    life of the process; make that first call before any stream capture
 *    begins.  The cache is keyed by device ordinal: after the device's
 *    primary context is reset (cudaDeviceReset) the cached address is stale,
 *    so do not use this entry point across such a reset.
 *  - All calls on a device share the one array and it keeps the previous
 *    call's contents; no word of it needs a starting value, because the
 *    partial records a call reads are written earlier in the same call.
 *    Calls whose kernels overlap on the GPU (different streams, no ordering)
 *    race on the array; order them on one stream or by events.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine. */
KVARN_API kvarn_status kvarn_decode_attention_noalloc(const void* q, const void* packed_cache, const void* scales,
                                                      const void* fp16_tail, const int32_t* block_table,
                                                      const int32_t* seq_lens, void* out,
                                                      const kvarn_decode_dims* dims, const kvarn_config* cfg,
                                                      int32_t* dev_status, void* stream);

/* Measurement baselines: the same paged decode over UNCOMPRESSED caches.
 *  k_cache, v_cache  [num_blocks][Hkv][128 tokens][128] fp16 (or fp8 e4m3 for
 *                    the _fp8 variant, values = e4m3 * k_scale / v_scale);
 *                    token i of sequence b sits in block block_table[b][i/128],
 *                    row i % 128 (the last block may be partial; no tail).
 *  sm_scale          0 means 1/sqrt(128).
 *  workspace         at least kvarn_baseline_workspace_bytes(dims). */
KVARN_API size_t kvarn_baseline_workspace_bytes(const kvarn_decode_dims* dims);

KVARN_API kvarn_status kvarn_decode_attention_fp16(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         void* out, const kvarn_decode_dims* dims, float sm_scale,
                                         void* workspace, size_t workspace_bytes,
                                         int32_t* dev_status, void* stream);

KVARN_API kvarn_status kvarn_decode_attention_fp8(const void* q, const void* k_cache, const void* v_cache,
                                        const int32_t* block_table, const int32_t* seq_lens,
                                        void* out, const kvarn_decode_dims* dims, float sm_scale,
                                        float k_scale, float v_scale,
                                        void* workspace, size_t workspace_bytes,
                                        int32_t* dev_status, void* stream);

/* Human-readable name of a status code (static storage). */
KVARN_API const char* kvarn_status_string(kvarn_status s);

/* KVARN_ABI_VERSION of the loaded library. */
KVARN_API int32_t kvarn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVARN_H_ */
