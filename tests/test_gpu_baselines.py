"""GPU parity of the uncompressed fp16 / fp8 (e4m3) paged decode baselines
against the oracle's textbook softmax attention over the same cache
contents (fp64, fp16 output).  Bound: 2e-3 absolute, or one fp16 step
where the output's own spacing is larger."""
import numpy as np
import pytest
import torch

from oracle import kvarn_oracle as O
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


def _bound(ref16):
    r = np.abs(ref16.astype(np.float16))
    return np.maximum(2e-3, np.spacing(r).astype(np.float64))


def paged_uncompressed(lens, hq, hkv, seed):
    """Per-sequence fp16 K/V rows and a shuffled paged cache holding them
    ([num_blocks][Hkv][128][128]); partial last blocks are padded with noise."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    nblk = [(int(L) + 127) // 128 for L in lens]
    num_blocks = max(1, sum(nblk)) + 3
    perm = rng.permutation(num_blocks)
    max_blocks = max(1, max(nblk))
    bt = np.zeros((len(lens), max_blocks), dtype=np.int32)
    kc = rng.standard_normal((num_blocks, hkv, 128, 128)).astype(np.float16)   # noise everywhere
    vc = rng.standard_normal((num_blocks, hkv, 128, 128)).astype(np.float16)
    outl = inputs.pick_outlier_channels(rng, hkv)
    rows_k, rows_v = [], []
    nxt = 0
    for b, L in enumerate(lens):
        k = inputs.gen_k(rng, int(L), hkv, outl)
        v = inputs.gen_v(rng, int(L), hkv)
        rows_k.append(k)
        rows_v.append(v)
        for i in range(nblk[b]):
            blk = int(perm[nxt]); nxt += 1
            bt[b, i] = blk
            n = min(128, int(L) - 128 * i)
            kc[blk, :, :n] = k[128 * i:128 * i + n].transpose(1, 0, 2)
            vc[blk, :, :n] = v[128 * i:128 * i + n].transpose(1, 0, 2)
    q = rng.standard_normal((len(lens), hq, 128)).astype(np.float16)
    return q, kc, vc, bt, lens, rows_k, rows_v


@pytest.mark.parametrize("G", [1, 4, 8])
def test_fp16_baseline_parity(K, G):
    lens = [1, 77, 128, 300, 33 * 128 + 5, 0, 129]
    q, kc, vc, bt, lens, rk, rv = paged_uncompressed(lens, 2 * G, 2, seed=50 + G)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention_fp16(dev(q), dev(kc), dev(vc), dev(bt), dev(lens), dev_status=status).cpu().numpy()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.decode_uncompressed(q, rk, rv, lens, 2)
    err = np.abs(out.astype(np.float64) - ref.astype(np.float64))
    print(f"fp16 G={G}: max err {err.max():.2e}")
    assert np.all(err <= _bound(ref))
    assert np.all(out[5] == 0)


@pytest.mark.parametrize("G", [4, 8])
def test_fp8_baseline_parity(K, G):
    lens = [50, 128, 2 * 128 + 100, 21 * 128]
    q, kc, vc, bt, lens, rk, rv = paged_uncompressed(lens, 2 * G, 2, seed=70 + G)
    k_scale = float(np.abs(kc.astype(np.float32)).max()) / 448.0
    v_scale = float(np.abs(vc.astype(np.float32)).max()) / 448.0
    kq = O.float_to_e4m3(kc.astype(np.float64) / k_scale)
    vq = O.float_to_e4m3(vc.astype(np.float64) / v_scale)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention_fp8(dev(q), dev(kq), dev(vq), dev(bt), dev(lens), k_scale, v_scale,
                                 dev_status=status).cpu().numpy()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # the oracle attends over exactly the stored e4m3 values
    kd = O.e4m3_to_float(kq) * k_scale
    vd = O.e4m3_to_float(vq) * v_scale
    rows_k = [np.concatenate([kd[bt[b, i], :, :min(128, int(L) - 128 * i)].transpose(1, 0, 2)
                              for i in range((int(L) + 127) // 128)]) for b, L in enumerate(lens)]
    rows_v = [np.concatenate([vd[bt[b, i], :, :min(128, int(L) - 128 * i)].transpose(1, 0, 2)
                              for i in range((int(L) + 127) // 128)]) for b, L in enumerate(lens)]
    ref = O.decode_uncompressed(q, rows_k, rows_v, lens, 2)
    err = np.abs(out.astype(np.float64) - ref.astype(np.float64))
    print(f"fp8 G={G}: max err {err.max():.2e}")
    assert np.all(err <= _bound(ref))
