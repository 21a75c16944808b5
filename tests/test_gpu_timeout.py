"""The bounded-wait status path of the decode kernel (KVARN_DEV_TIMEOUT).

A test-only build of the library (libkvarn_stalltest.so, built beside
libkvarn.so) arms the first copy stage of one warp with 16 bytes that are
never sent and issues no copy for it, and lowers the wait limit to 2^10
polls.  No copy is in flight and no access goes out of bounds: the wait
simply runs out.  The kernel must report KVARN_DEV_TIMEOUT and return, and
a normal decode afterwards must still be correct.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import kvarn_oracle as O
from bit_kv_cache_15_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_kv_cache_15_b200 import build
    build.build()
    from bit_kv_cache_15_b200 import kvarn
    stall = ctypes.CDLL(build.STALL_LIB)
    stall.kvarn_decode_attention.restype = ctypes.c_int
    stall.kvarn_decode_attention.argtypes = kvarn.lib.kvarn_decode_attention.argtypes
    return kvarn, stall


def test_decode_wait_timeout_is_reported_and_device_stays_usable(libs):
    K, stall = libs
    # more work units than decode warps (4 per CTA, 2 CTAs per SM), so that warp 0
    # of CTA 0 (whose first copy stalls) has a range
    w = inputs.make_decode_workload("timeout", [200 * 128 + 9, 180 * 128, 300], 16, 4, seed=990, pool_blocks=390)
    cfg = K.config()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, 4)
    K.quantize_tiles(dev(w.k_full), dev(w.v_full), dev(w.slot_mapping), packed, scales, cfg)
    q, tail, bt, sl = dev(w.q), dev(w.tail), dev(w.block_table), dev(w.seq_lens)
    d = K.dims(w.num_seqs, 16, 4, w.max_blocks_per_seq, w.num_blocks)
    ws = torch.zeros(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = stall.kvarn_decode_attention(q.data_ptr(), packed.data_ptr(), scales.data_ptr(), tail.data_ptr(),
                                      bt.data_ptr(), sl.data_ptr(), out.data_ptr(), ctypes.byref(d),
                                      ctypes.byref(cfg), ws.data_ptr(), ws.numel(), status.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 4            # KVARN_DEV_TIMEOUT
    # the context is intact: a normal call on the same buffers is green and correct
    status.zero_()
    got = K.decode_attention(q, packed, scales, tail, bt, sl, cfg, workspace=ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.decode(w.q, packed.cpu().numpy(), scales.cpu().numpy(), w.tail, w.block_table, w.seq_lens, 4, 4, 2)
    err = np.abs(got.cpu().numpy().astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= np.maximum(2e-3, np.spacing(np.abs(ref)).astype(np.float64)))
