"""The library's calls inside CUDA graph capture.

Every kernel is a programmatic dependent launch; captured into a graph, the
launches become graph nodes with programmatic edges.  A quantise + decode
step and a decode step with append, captured once and replayed, must give
exactly the outputs of the same calls run eagerly.  The first (eager) calls
do each kernel's one-time launch set-up, which must happen before capture.
"""
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
    return kvarn


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_quantize_and_decode_replayed_from_a_graph(K):
    lens = [5 * 128 + 33, 2 * 128, 77, 9 * 128 + 1]
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("graph", lens, 16, 2, seed=1300, pool_blocks=full)
    cfg = K.config()
    k, v, slot = _dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping)
    q, tail, bt, sl = _dev(w.q), _dev(w.tail), _dev(w.block_table), _dev(w.seq_lens)
    d = K.dims(w.num_seqs, 16, 2, w.max_blocks_per_seq, w.num_blocks)
    ws = torch.zeros(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
    out = torch.empty_like(q)
    stream = torch.cuda.Stream()

    def step():
        K.quantize_tiles(k, v, slot, packed, scales, cfg, dev_status=status, stream=stream)
        K.decode_attention(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws, dev_status=status,
                           stream=stream)

    with torch.cuda.stream(stream):
        step()                                   # eager: one-time launch set-up, reference result
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_out, ref_packed = out.clone(), packed.clone()

    packed.zero_()
    out.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    for _ in range(2):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(packed, ref_packed)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    del g


def test_append_step_replayed_from_a_graph(K):
    lens = [3 * 128 + 127, 200, 127]             # two fills and one plain append
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("graph_app", lens, 8, 2, seed=1310, pool_blocks=full + 4)
    k_new, v_new, bt_np = inputs.append_step(w, 1311)
    cfg = K.config()
    d = K.dims(w.num_seqs, 8, 2, bt_np.shape[1], w.num_blocks)
    ws = torch.zeros(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, kn, vn, bt, sl = _dev(w.q), _dev(k_new), _dev(v_new), _dev(bt_np), _dev(w.seq_lens)
    stream = torch.cuda.Stream()
    results = []
    for mode in ("eager", "graph"):
        packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
        if w.k_full.shape[0]:
            K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
        tail = _dev(w.tail)
        out = torch.empty_like(q)
        torch.cuda.synchronize()

        def call():
            K.decode_attention_append(q, kn, vn, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws,
                                      dev_status=status, stream=stream)

        if mode == "eager":
            with torch.cuda.stream(stream):
                call()
        else:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                call()
            g.replay()                           # the same step once: tail row and filled tiles rewritten
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        results.append((out.clone(), packed.clone(), scales.clone(), tail.clone()))
    for a, b in zip(results[0], results[1]):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
