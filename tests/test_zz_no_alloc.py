"""The allocation-free decode entry point (kvarn_decode_attention_noalloc).

It is for callers that cannot allocate device memory themselves; the
partial-record scratch of its stream-K decode is a fixed device array inside
the library.  Here it is
called straight through the C ABI and its output is checked against the
workspace-taking kvarn_decode_attention on the same inputs, within the
decode tolerance the parity tests use, on two calls in a row (the second
call finds the first call's leftovers in the shared array).  This file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_kv_cache_15_b200 import inputs

pytestmark = pytest.mark.gpu

DECODE_TOL = 2e-3


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_15_b200 import build
    build.build()
    from bit_kv_cache_15_b200 import kvarn
    return kvarn


def _bound(ref16):
    r = np.abs(ref16.astype(np.float16))
    return np.maximum(DECODE_TOL, np.spacing(r).astype(np.float64))


def _problem(K, lens, hq, hkv, seed):
    w = inputs.make_decode_workload("noalloc", lens, hq, hkv, seed=seed)
    cfg = K.config("kvarn_k4v2_g128")
    packed, scales = K.alloc_cache(cfg, w.num_blocks, hkv)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    K.quantize_tiles(dev(w.k_full), dev(w.v_full), dev(w.slot_mapping), packed, scales, cfg)
    return cfg, w, packed, scales, dev(w.q), dev(w.tail), dev(w.block_table), dev(w.seq_lens)


def _noalloc_via_cabi(K, cfg, q, packed, scales, tail, bt, sl, status):
    out = torch.empty_like(q)
    d = K.dims(q.shape[0], q.shape[1], packed.shape[1], bt.shape[1], packed.shape[0])
    st = K.lib.kvarn_decode_attention_noalloc(q.data_ptr(), packed.data_ptr(), scales.data_ptr(), tail.data_ptr(),
                                              bt.data_ptr(), sl.data_ptr(), out.data_ptr(), ctypes.byref(d),
                                              ctypes.byref(cfg), status.data_ptr(),
                                              torch.cuda.current_stream().cuda_stream)
    assert st == 0, K.STATUS_NAMES.get(st, st)
    return out


def test_noalloc_matches_workspace_entry_point_twice(K):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a larger problem first, then a smaller one with a different geometry
    for lens, hq, hkv, seed in (([40 * 128 + 70, 9 * 128, 300, 5], 16, 2, 901),
                                ([3 * 128 + 1, 128], 8, 1, 902)):
        cfg, w, packed, scales, q, tail, bt, sl = _problem(K, lens, hq, hkv, seed)
        ref = K.decode_attention(q, packed, scales, tail, bt, sl, cfg, dev_status=status)
        got = _noalloc_via_cabi(K, cfg, q, packed, scales, tail, bt, sl, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        r = ref.cpu().numpy()
        g = got.cpu().numpy()
        assert np.all(np.isfinite(g.astype(np.float32)))
        assert np.all(np.abs(g.astype(np.float64) - r.astype(np.float64)) <= _bound(r))


def test_noalloc_rejects_problems_beyond_its_scratch(K):
    cfg = K.config("kvarn_k4v2_g128")
    # (B*Hkv + 320)*G tile records plus B*Hkv*G tail records of 528 B (and the
    # reserved words) exceed the fixed 8 MiB array
    d = K.dims(4096, 64, 8, 64, 4096)
    assert K.decode_workspace_bytes(cfg, d) > (8 << 20)
    one = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = one.data_ptr()
    st = K.lib.kvarn_decode_attention_noalloc(p, p, p, p, p, p, p, ctypes.byref(d), ctypes.byref(cfg), None,
                                              torch.cuda.current_stream().cuda_stream)
    assert st == 4   # KVARN_ERR_WORKSPACE_TOO_SMALL, nothing launched
