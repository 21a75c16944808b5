"""Python binding of libkvarn.so (ctypes).  Argument marshalling only.

Every function takes torch tensors that already live on the GPU, checks
their dtype/shape/contiguity, and passes raw device pointers plus the
current CUDA stream to the C ABI declared in include/kvarn.h.  All
arithmetic runs in the library's kernels; there is no CPU fallback, and
importing this module fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvarn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_kv_cache_15_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

TILE = 128
HEAD_DIM = 128
SCALE_RECORD_BYTES = 528

OK = 0
STATUS_NAMES = {0: "KVARN_OK", 1: "KVARN_ERR_INVALID_ARGUMENT", 2: "KVARN_ERR_UNSUPPORTED",
                3: "KVARN_ERR_CUDA", 4: "KVARN_ERR_WORKSPACE_TOO_SMALL"}
DEV_STATUS_NAMES = {0: "ok", 1: "bad slot", 2: "bad block", 3: "bad seq_len", 4: "timeout"}


class Config(ctypes.Structure):
    _fields_ = [("version", ctypes.c_int32), ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32),
                ("tile_tokens", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("sinkhorn_iters", ctypes.c_int32), ("layout", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("sm_scale", ctypes.c_float)]


class DecodeDims(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("num_blocks", ctypes.c_int64)]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_st = ctypes.c_int

_SIGS = {
    "kvarn_config_from_string": (_st, [ctypes.c_char_p, ctypes.POINTER(Config)]),
    "kvarn_config_validate": (_st, [ctypes.POINTER(Config)]),
    "kvarn_cache_bytes_per_block": (_sz, [ctypes.POINTER(Config), _i32]),
    "kvarn_scale_bytes_per_block": (_sz, [_i32]),
    "kvarn_decode_workspace_bytes": (_sz, [ctypes.POINTER(Config), ctypes.POINTER(DecodeDims)]),
    "kvarn_quantize_tiles": (_st, [_vp, _vp, _vp, _i64, _i32, _i64, _vp, _vp, ctypes.POINTER(Config), _vp, _vp]),
    "kvarn_quantize_tiles_debug": (_st, [_vp, _vp, _vp, _i64, _i32, _i64, _vp, _vp, ctypes.POINTER(Config),
                                         _vp, _vp, _vp]),
    "kvarn_decode_attention": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                     ctypes.POINTER(Config), _vp, _sz, _vp, _vp]),
    "kvarn_decode_attention_noalloc": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                             ctypes.POINTER(Config), _vp, _vp]),
    "kvarn_decode_attention_append": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                            ctypes.POINTER(Config), _vp, _sz, _vp, _vp]),
    "kvarn_decode_multiquery_workspace_bytes": (_sz, [ctypes.POINTER(Config), ctypes.POINTER(DecodeDims), _i32]),
    "kvarn_decode_attention_multiquery": (_st, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                                ctypes.POINTER(Config), _vp, _sz, _vp, _vp]),
    "kvarn_baseline_workspace_bytes": (_sz, [ctypes.POINTER(DecodeDims)]),
    "kvarn_decode_attention_fp16": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                          ctypes.c_float, _vp, _sz, _vp, _vp]),
    "kvarn_decode_attention_fp8": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DecodeDims),
                                         ctypes.c_float, ctypes.c_float, ctypes.c_float, _vp, _sz, _vp, _vp]),
    "kvarn_status_string": (ctypes.c_char_p, [_st]),
    "kvarn_abi_version": (_i32, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

lib = _lib


class KvarnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != OK:
        raise KvarnError(fn, status)


def config(s: str = "kvarn_k4v2_g128", sinkhorn_iters: int = 8, sm_scale: float = 0.0) -> Config:
    cfg = Config()
    _check("kvarn_config_from_string", _lib.kvarn_config_from_string(s.encode(), ctypes.byref(cfg)))
    cfg.sinkhorn_iters = sinkhorn_iters
    cfg.sm_scale = sm_scale
    _check("kvarn_config_validate", _lib.kvarn_config_validate(ctypes.byref(cfg)))
    return cfg


def dims(num_seqs: int, num_q_heads: int, num_kv_heads: int, max_blocks_per_seq: int,
         num_blocks: int) -> DecodeDims:
    return DecodeDims(num_seqs, num_q_heads, num_kv_heads, max_blocks_per_seq, num_blocks)


def cache_bytes_per_block(cfg: Config, num_kv_heads: int) -> int:
    return int(_lib.kvarn_cache_bytes_per_block(ctypes.byref(cfg), num_kv_heads))


def scale_bytes_per_block(num_kv_heads: int) -> int:
    return int(_lib.kvarn_scale_bytes_per_block(num_kv_heads))


def decode_workspace_bytes(cfg: Config, d: DecodeDims) -> int:
    return int(_lib.kvarn_decode_workspace_bytes(ctypes.byref(cfg), ctypes.byref(d)))


def baseline_workspace_bytes(d: DecodeDims) -> int:
    return int(_lib.kvarn_baseline_workspace_bytes(ctypes.byref(d)))


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t: torch.Tensor, name: str, dtype, cuda: bool = True) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def alloc_cache(cfg: Config, num_blocks: int, num_kv_heads: int, device="cuda"):
    """Zeroed packed cache [num_blocks][Hkv][2048(kb+vb)] and scales [num_blocks][Hkv][2][528] (uint8)."""
    cb = cache_bytes_per_block(cfg, num_kv_heads) // num_kv_heads
    packed = torch.zeros((num_blocks, num_kv_heads, cb), dtype=torch.uint8, device=device)
    scales = torch.zeros((num_blocks, num_kv_heads, 2, SCALE_RECORD_BYTES), dtype=torch.uint8, device=device)
    return packed, scales


def quantize_tiles(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, packed_cache: torch.Tensor,
                   scales: torch.Tensor, cfg: Config, dev_status: torch.Tensor | None = None,
                   debug_logscales: torch.Tensor | None = None, stream=None) -> None:
    """Quantise k, v ([n][Hkv][128] fp16, n % 128 == 0) into the paged cache."""
    _need(k, "k", torch.float16)
    _need(v, "v", torch.float16)
    _need(slot_mapping, "slot_mapping", torch.int64)
    _need(packed_cache, "packed_cache", torch.uint8)
    _need(scales, "scales", torch.uint8)
    if k.shape != v.shape or k.dim() != 3 or k.shape[2] != HEAD_DIM:
        raise ValueError("k, v must be [num_tokens][num_kv_heads][128]")
    n, hkv = int(k.shape[0]), int(k.shape[1])
    if slot_mapping.numel() != n:
        raise ValueError("slot_mapping must have one entry per token")
    nb = int(packed_cache.shape[0])
    if debug_logscales is None:
        st = _lib.kvarn_quantize_tiles(_ptr(k), _ptr(v), _ptr(slot_mapping), n, hkv, nb, _ptr(packed_cache),
                                       _ptr(scales), ctypes.byref(cfg), _ptr(dev_status), _stream(stream))
        _check("kvarn_quantize_tiles", st)
    else:
        _need(debug_logscales, "debug_logscales", torch.float32)
        st = _lib.kvarn_quantize_tiles_debug(_ptr(k), _ptr(v), _ptr(slot_mapping), n, hkv, nb,
                                             _ptr(packed_cache), _ptr(scales), ctypes.byref(cfg),
                                             _ptr(debug_logscales), _ptr(dev_status), _stream(stream))
        _check("kvarn_quantize_tiles_debug", st)


def decode_attention(q: torch.Tensor, packed_cache: torch.Tensor, scales: torch.Tensor, fp16_tail: torch.Tensor,
                     block_table: torch.Tensor, seq_lens: torch.Tensor, cfg: Config, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Paged decode attention on the packed cache; returns out [B][Hq][128] fp16."""
    _need(q, "q", torch.float16)
    _need(packed_cache, "packed_cache", torch.uint8)
    _need(scales, "scales", torch.uint8)
    _need(fp16_tail, "fp16_tail", torch.float16)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hq, _ = q.shape
    Hkv = int(packed_cache.shape[1])
    d = dims(B, Hq, Hkv, int(block_table.shape[1]), int(packed_cache.shape[0]))
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:   # zeroed: the trailing arrival counters must start at zero
        workspace = torch.zeros(decode_workspace_bytes(cfg, d), dtype=torch.uint8, device=q.device)
    st = _lib.kvarn_decode_attention(_ptr(q), _ptr(packed_cache), _ptr(scales), _ptr(fp16_tail), _ptr(block_table),
                                     _ptr(seq_lens), _ptr(out), ctypes.byref(d), ctypes.byref(cfg),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _ptr(dev_status), _stream(stream))
    _check("kvarn_decode_attention", st)
    return out


def decode_attention_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, packed_cache: torch.Tensor,
                            scales: torch.Tensor, fp16_tail: torch.Tensor, block_table: torch.Tensor,
                            seq_lens: torch.Tensor, cfg: Config, out: torch.Tensor | None = None,
                            workspace: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                            stream=None) -> torch.Tensor:
    """One decode step with append (kvarn_decode_attention_append in
    include/kvarn.h): k_new / v_new [B][Hkv][128] fp16 are the step's tokens,
    seq_lens the lengths before the step (left unchanged: add 1 afterwards).
    Writes the tail, quantises tails that fill, returns out [B][Hq][128]."""
    _need(q, "q", torch.float16)
    _need(k_new, "k_new", torch.float16)
    _need(v_new, "v_new", torch.float16)
    _need(packed_cache, "packed_cache", torch.uint8)
    _need(scales, "scales", torch.uint8)
    _need(fp16_tail, "fp16_tail", torch.float16)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hq, _ = q.shape
    Hkv = int(packed_cache.shape[1])
    if tuple(k_new.shape) != (B, Hkv, 128) or tuple(v_new.shape) != (B, Hkv, 128):
        raise ValueError("k_new / v_new must be [B][Hkv][128]")
    d = dims(B, Hq, Hkv, int(block_table.shape[1]), int(packed_cache.shape[0]))
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.zeros(decode_workspace_bytes(cfg, d), dtype=torch.uint8, device=q.device)
    st = _lib.kvarn_decode_attention_append(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(packed_cache), _ptr(scales),
                                            _ptr(fp16_tail), _ptr(block_table), _ptr(seq_lens), _ptr(out),
                                            ctypes.byref(d), ctypes.byref(cfg), _ptr(workspace),
                                            workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                            _stream(stream))
    _check("kvarn_decode_attention_append", st)
    return out


def decode_multiquery_workspace_bytes(cfg: Config, d: DecodeDims, q_len: int) -> int:
    return int(_lib.kvarn_decode_multiquery_workspace_bytes(ctypes.byref(cfg), ctypes.byref(d), int(q_len)))


def decode_attention_multiquery(q: torch.Tensor, packed_cache: torch.Tensor, scales: torch.Tensor,
                                fp16_tail: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor,
                                cfg: Config, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                                dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Multi-query attention over the packed cache (kvarn_decode_attention_multiquery
    in include/kvarn.h): q [B][q_len][Hq][128] fp16, query i of sequence b at
    position seq_len - q_len + i, attending causally.  Returns out like q."""
    _need(q, "q", torch.float16)
    _need(packed_cache, "packed_cache", torch.uint8)
    _need(scales, "scales", torch.uint8)
    _need(fp16_tail, "fp16_tail", torch.float16)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    if q.dim() != 4:
        raise ValueError("q must be [B][q_len][Hq][128]")
    B, q_len, Hq, _ = q.shape
    Hkv = int(packed_cache.shape[1])
    d = dims(B, Hq, Hkv, int(block_table.shape[1]), int(packed_cache.shape[0]))
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.zeros(decode_multiquery_workspace_bytes(cfg, d, q_len), dtype=torch.uint8, device=q.device)
    st = _lib.kvarn_decode_attention_multiquery(_ptr(q), int(q_len), _ptr(packed_cache), _ptr(scales),
                                                _ptr(fp16_tail), _ptr(block_table), _ptr(seq_lens), _ptr(out),
                                                ctypes.byref(d), ctypes.byref(cfg), _ptr(workspace),
                                                workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                                _stream(stream))
    _check("kvarn_decode_attention_multiquery", st)
    return out


def decode_attention_noalloc(q: torch.Tensor, packed_cache: torch.Tensor, scales: torch.Tensor,
                             fp16_tail: torch.Tensor, block_table: torch.Tensor, seq_lens: torch.Tensor, cfg: Config,
                             out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                             stream=None) -> torch.Tensor:
    """decode_attention with the library's fixed device scratch instead of a
    workspace tensor (see kvarn_decode_attention_noalloc in include/kvarn.h)."""
    _need(q, "q", torch.float16)
    _need(packed_cache, "packed_cache", torch.uint8)
    _need(scales, "scales", torch.uint8)
    _need(fp16_tail, "fp16_tail", torch.float16)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32)
    B, Hq, _ = q.shape
    d = dims(B, Hq, int(packed_cache.shape[1]), int(block_table.shape[1]), int(packed_cache.shape[0]))
    if out is None:
        out = torch.empty_like(q)
    st = _lib.kvarn_decode_attention_noalloc(_ptr(q), _ptr(packed_cache), _ptr(scales), _ptr(fp16_tail),
                                             _ptr(block_table), _ptr(seq_lens), _ptr(out), ctypes.byref(d),
                                             ctypes.byref(cfg), _ptr(dev_status), _stream(stream))
    _check("kvarn_decode_attention_noalloc", st)
    return out


def decode_attention_fp16(q, k_cache, v_cache, block_table, seq_lens, out=None, workspace=None, sm_scale=0.0,
                          dev_status=None, stream=None):
    """Baseline: paged decode over an uncompressed fp16 cache [num_blocks][Hkv][128][128]."""
    _need(q, "q", torch.float16)
    _need(k_cache, "k_cache", torch.float16)
    _need(v_cache, "v_cache", torch.float16)
    B, Hq, _ = q.shape
    d = dims(B, Hq, int(k_cache.shape[1]), int(block_table.shape[1]), int(k_cache.shape[0]))
    out = torch.empty_like(q) if out is None else out
    if workspace is None:
        workspace = torch.zeros(baseline_workspace_bytes(d), dtype=torch.uint8, device=q.device)
    st = _lib.kvarn_decode_attention_fp16(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                          _ptr(out), ctypes.byref(d), sm_scale, _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                          _stream(stream))
    _check("kvarn_decode_attention_fp16", st)
    return out


def decode_attention_fp8(q, k_cache, v_cache, block_table, seq_lens, k_scale, v_scale, out=None, workspace=None,
                         sm_scale=0.0, dev_status=None, stream=None):
    """Baseline: paged decode over an e4m3 cache (uint8 [num_blocks][Hkv][128][128])."""
    _need(q, "q", torch.float16)
    _need(k_cache, "k_cache", torch.uint8)
    _need(v_cache, "v_cache", torch.uint8)
    B, Hq, _ = q.shape
    d = dims(B, Hq, int(k_cache.shape[1]), int(block_table.shape[1]), int(k_cache.shape[0]))
    out = torch.empty_like(q) if out is None else out
    if workspace is None:
        workspace = torch.zeros(baseline_workspace_bytes(d), dtype=torch.uint8, device=q.device)
    st = _lib.kvarn_decode_attention_fp8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(seq_lens),
                                         _ptr(out), ctypes.byref(d), sm_scale, k_scale, v_scale, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                         _stream(stream))
    _check("kvarn_decode_attention_fp8", st)
    return out
