"""The C-ABI library on the host: it loads, exports every function that
include/kvarn.h declares, and rejects bad arguments before any launch.
No call here reaches the GPU (argument errors return first)."""
import ctypes
import os
import re

import pytest

from bit_kv_cache_15_b200 import build

build.build()
from bit_kv_cache_15_b200 import kvarn as K  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "kvarn.h")

FAKE = 0x100000  # an aligned, never dereferenced address for host-side checks


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvarn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "kvarn_quantize_tiles" in names and "kvarn_decode_attention" in names
    for n in names:
        assert hasattr(K.lib, n), n
        assert n in K._SIGS, f"binding misses {n}"


@pytest.mark.parametrize("path", [build.DEBUG_LIB, build.STALL_LIB])
def test_test_builds_load_and_export_the_same_symbols(path):
    """The debug build (device-side index checks) and the stall-test build
    load on the host and export the same C ABI as the release library."""
    lib = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(lib, n), (path, n)
    assert lib.kvarn_abi_version() == K.lib.kvarn_abi_version()


def test_abi_version_and_status_strings():
    assert K.lib.kvarn_abi_version() == 1
    assert K.lib.kvarn_status_string(0) == b"KVARN_OK"
    assert K.lib.kvarn_status_string(4) == b"KVARN_ERR_WORKSPACE_TOO_SMALL"


def test_config_string_parsing():
    cfg = K.config("kvarn_k4v2_g128")
    assert (cfg.k_bits, cfg.v_bits, cfg.tile_tokens, cfg.head_dim, cfg.sinkhorn_iters) == (4, 2, 128, 128, 8)
    bad = K.Config()
    assert K.lib.kvarn_config_from_string(b"kvarn_k3v2_g128", ctypes.byref(bad)) == 2
    assert K.lib.kvarn_config_from_string(b"kvarn_k4v2_g64", ctypes.byref(bad)) == 2
    assert K.lib.kvarn_config_from_string(b"fp8", ctypes.byref(bad)) == 1
    assert K.lib.kvarn_config_from_string(b"kvarn_k4v2_g128x", ctypes.byref(bad)) == 1
    for kb in (2, 4, 8):
        for vb in (2, 4, 8):
            c = K.config(f"kvarn_k{kb}v{vb}_g128")
            assert K.cache_bytes_per_block(c, 8) == 8 * 2048 * (kb + vb)


def test_sizes():
    cfg = K.config()
    assert K.cache_bytes_per_block(cfg, 8) == 8 * 12288
    assert K.scale_bytes_per_block(8) == 8 * 1056
    d = K.dims(8, 64, 8, 129, 1024)
    ws = K.decode_workspace_bytes(cfg, d)
    # partial records (528 B per seq x q head x split, plus the tail slot) then 8 x 8 int32 counters
    assert ws % 16 == 0 and (ws - 8 * 8 * 4) % 528 == 0 and ws >= 8 * 64 * 2 * 528 + 8 * 8 * 4
    assert K.decode_workspace_bytes(cfg, K.dims(8, 72, 8, 129, 1024)) == 0   # G = 9 unsupported


def _q(n, cfg, hkv=2, nb=4, k=FAKE, v=FAKE, slot=FAKE, packed=FAKE, scales=FAKE):
    return K.lib.kvarn_quantize_tiles(k, v, slot, n, hkv, nb, packed, scales, ctypes.byref(cfg), None, None)


def test_quantize_argument_checks():
    cfg = K.config()
    assert _q(0, cfg) == 0                       # nothing to do, no launch
    assert _q(100, cfg) == 1                     # not a multiple of 128
    assert _q(-128, cfg) == 1
    assert _q(128, cfg, k=None) == 1
    assert _q(128, cfg, packed=FAKE + 8) == 1    # misaligned
    assert _q(128, cfg, hkv=0) == 1
    cfg.sinkhorn_iters = 0
    assert _q(128, cfg) == 1
    cfg = K.config()
    cfg.k_bits = 3
    assert _q(128, cfg) == 2
    cfg = K.config()
    cfg.version = 7
    assert _q(128, cfg) == 2


def test_decode_argument_checks():
    cfg = K.config()
    d = K.dims(2, 8, 2, 4, 16)
    need = K.decode_workspace_bytes(cfg, d)

    def call(dd, ws_bytes=need, q=FAKE, out=FAKE):
        return K.lib.kvarn_decode_attention(q, FAKE, FAKE, FAKE, FAKE, FAKE, out, ctypes.byref(dd), ctypes.byref(cfg),
                                            FAKE, ws_bytes, None, None)

    assert call(d, need - 1) == 4
    assert call(d, q=None) == 1
    assert call(d, out=FAKE + 2) == 1
    assert call(K.dims(2, 7, 2, 4, 16)) == 1          # Hq not a multiple of Hkv
    assert call(K.dims(2, 32, 2, 4, 16)) == 2         # G = 16 unsupported
    assert call(K.dims(0, 8, 2, 4, 16)) == 0          # empty batch: nothing to do
    assert call(K.dims(2, 8, 2, 0, 16)) == 1


def test_baseline_argument_checks():
    d = K.dims(2, 8, 2, 4, 16)
    need = K.baseline_workspace_bytes(d)
    r = K.lib.kvarn_decode_attention_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), 0.0, 0.0, 1.0, FAKE,
                                         need, None, None)
    assert r == 1                                      # k_scale must be > 0
    r = K.lib.kvarn_decode_attention_fp16(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.byref(d), 0.0, FAKE,
                                          need - 1, None, None)
    assert r == 4


def _baseline_splits(B, hkv, max_blocks, ctas_per_sm):
    """The uncompressed baselines' split geometry restated: tiles per split T
    (a multiple of 4) minimising waves x (T / 4 + 1) over ctas_per_sm x 148
    slots, ties to the larger T; returns the number of splits."""
    pairs, slots = max(1, B * hkv), ctas_per_sm * 148
    best_t, best = 4, float("inf")
    for t in range(4, 65, 4):
        ns = -(-max_blocks // t)
        cost = -(-(pairs * ns) // slots) * (t / 4 + 1)
        if cost <= best:
            best, best_t = cost, t
        if ns == 1:
            break
    return max(1, -(-max_blocks // best_t))


@pytest.mark.parametrize("B,hq,hkv,mb", [(8, 64, 8, 129), (16, 32, 8, 33), (4, 64, 8, 1025), (1, 8, 1, 1),
                                         (2, 8, 2, 4), (64, 16, 2, 300)])
def test_baseline_workspace_fits_both_geometries(B, hq, hkv, mb):
    """The workspace holds the split records of the fp16 geometry (2 CTAs per
    SM planned) and of the fp8 one (4), whichever is larger, then the B x Hkv
    int32 arrival counters rounded to 16 bytes."""
    ns = max(_baseline_splits(B, hkv, mb, 2), _baseline_splits(B, hkv, mb, 4))
    counters = (B * hkv * 4 + 15) // 16 * 16
    assert K.baseline_workspace_bytes(K.dims(B, hq, hkv, mb, 1024)) == B * hq * (ns + 1) * 528 + counters


def test_binding_fails_loudly_without_library(tmp_path):
    """The binding refuses to import when libkvarn.so is absent (no fallback)."""
    import subprocess
    import sys
    import shutil
    pkg = tmp_path / "bit_kv_cache_15_b200"
    shutil.copytree(os.path.dirname(K.__file__), pkg, ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import bit_kv_cache_15_b200.kvarn"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libkvarn.so is missing" in r.stderr


def test_decode_append_argument_checks():
    cfg = K.config()
    d = K.dims(2, 8, 2, 4, 16)
    need = K.decode_workspace_bytes(cfg, d)

    def call(k_new=FAKE, v_new=FAKE, ws_bytes=need, dd=d):
        return K.lib.kvarn_decode_attention_append(FAKE, k_new, v_new, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                   ctypes.byref(dd), ctypes.byref(cfg), FAKE, ws_bytes, None, None)

    assert call(k_new=None) == 1
    assert call(v_new=FAKE + 4) == 1                   # misaligned
    assert call(ws_bytes=need - 1) == 4
    assert call(dd=K.dims(0, 8, 2, 4, 16)) == 0         # empty batch: nothing to do


def test_multiquery_argument_checks():
    cfg = K.config()
    d = K.dims(2, 8, 2, 4, 16)
    need = K.decode_multiquery_workspace_bytes(cfg, d, 4)
    assert need > K.decode_workspace_bytes(cfg, d)           # 16 columns per KV head: two groups
    assert K.decode_multiquery_workspace_bytes(cfg, d, 1) == K.decode_workspace_bytes(cfg, d)
    assert K.decode_multiquery_workspace_bytes(cfg, d, 0) == 0

    def call(q_len, ws_bytes=need):
        return K.lib.kvarn_decode_attention_multiquery(FAKE, q_len, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                       ctypes.byref(d), ctypes.byref(cfg), FAKE, ws_bytes, None, None)

    assert call(0) == 1
    assert call(129) == 1
    assert call(4, need - 1) == 4
