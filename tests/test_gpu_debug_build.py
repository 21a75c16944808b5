"""The debug build of the library (libkvarn_debug.so, built beside libkvarn.so
with -DKVARN_DEBUG=1): the same kernels with their own index arithmetic
checked on the device -- block-table rows and record slots of the decode's
work split, the merge's record range, the tail staging, the quantiser's tile
coordinates.  A failed check would report KVARN_DEV_INTERNAL
(5) and skip the guarded access; it never traps.

On valid inputs no check may fire (the status stays 0), and every output must
be bit-identical to the release library's on the same inputs: the checks
guard accesses and change no arithmetic.  Compute-sanitizer is not available
on this GPU pool; this build is the bounds checking that stands in for it.
"""
import contextlib
import ctypes

import numpy as np
import pytest
import torch

from bit_kv_cache_15_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_15_b200 import build
    build.build()
    from bit_kv_cache_15_b200 import kvarn
    dbg = ctypes.CDLL(build.DEBUG_LIB)
    for name, (res, args) in kvarn._SIGS.items():
        f = getattr(dbg, name)
        f.restype = res
        f.argtypes = args
    kvarn.debug_handle_for_tests = dbg
    return kvarn


@contextlib.contextmanager
def library(K, which):
    """Route the binding's calls to the release or the debug library."""
    old = K._lib
    K._lib = old if which == "release" else K.debug_handle_for_tests
    try:
        yield
    finally:
        K._lib = old


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_both(K, fn):
    """fn(status) -> dict of tensors, on each library; checks the debug run's
    status and that every result is bit-identical to the release run's."""
    res = {}
    for which in ("release", "debug"):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        with library(K, which):
            out = fn(status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, (which, int(status.item()))
        res[which] = {k: v.cpu() for k, v in out.items()}
    for k in res["release"]:
        a, b = res["release"][k], res["debug"][k]
        assert a.shape == b.shape and torch.equal(a.view(torch.uint8) if a.dtype == torch.float16 else a,
                                                  b.view(torch.uint8) if b.dtype == torch.float16 else b), k
    return res


@pytest.mark.parametrize("kb,vb", [(4, 2), (8, 8)])
def test_debug_build_quantize_and_decode(K, kb, vb):
    # empty, tail only, exactly one tile, ragged, long: several CTAs per pair
    lens = [0, 77, 128, 129, 300, 30 * 128 + 5, 1000]
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("dbg", lens, 16, 2, seed=1200 + kb, pool_blocks=full + 3)
    cfg = K.config(f"kvarn_k{kb}v{vb}_g128")

    def fn(status):
        packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
        K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg,
                         dev_status=status)
        out = K.decode_attention(_dev(w.q), packed, scales, _dev(w.tail), _dev(w.block_table), _dev(w.seq_lens),
                                 cfg, dev_status=status)
        return {"packed": packed, "scales": scales, "out": out}

    run_both(K, fn)


def test_debug_build_multiquery(K):
    qlen = 4
    lens = [256 + qlen - 1, 40 * 128 + 10, 7 + qlen, 128 + 2, 5 * 128]
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("dbg_mq", lens, 16, 2, seed=1210, pool_blocks=full + 2)
    cfg = K.config()
    q = np.random.default_rng(1211).standard_normal((len(lens), qlen, 16, 128)).astype(np.float16)

    def fn(status):
        packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
        K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg,
                         dev_status=status)
        out = K.decode_attention_multiquery(_dev(q), packed, scales, _dev(w.tail), _dev(w.block_table),
                                            _dev(w.seq_lens), cfg, dev_status=status)
        return {"out": out}

    run_both(K, fn)


def test_debug_build_append_with_fills(K):
    # lengths before the step: empty, fills with no full tile, fills after full tiles, mid-tile
    lens = [0, 127, 3 * 128 + 127, 200, 9 * 128 + 127]
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("dbg_app", lens, 8, 2, seed=1220, pool_blocks=full + 8)
    k_new, v_new, bt = inputs.append_step(w, 1221)
    cfg = K.config()

    def fn(status):
        packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
        if w.k_full.shape[0]:
            K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg,
                             dev_status=status)
        tail = _dev(w.tail)
        out = K.decode_attention_append(_dev(w.q), _dev(k_new), _dev(v_new), packed, scales, tail, _dev(bt),
                                        _dev(w.seq_lens), cfg, dev_status=status)
        return {"out": out, "packed": packed, "scales": scales, "tail": tail}

    run_both(K, fn)
