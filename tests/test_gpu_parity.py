"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Quantizer, staged as in the tolerance plan:
  1. fp32 log-scales before rounding: the scale 2^lt within 1e-5 relative,
     i.e. |lt_gpu - lt_oracle| <= log2(1 + 1e-5);
  2. stored fp16 log-scales: the fp16 rounding of some value within that
     tolerance of the oracle's fp64 value (at a rounding boundary either
     neighbour is correct);
  3. codes re-derived by the oracle (fp64 decision, its own exact rotation)
     from the GPU's stored scales, zero and step: >= 99.99 % identical, and
     every mismatch is +-1 at a rounding tie, within the error bound of the
     GPU's fp32 arithmetic;
  4. end-to-end codes >= 99.99 % identical to the oracle's own, over all
     codes and over those whose row and column scales agree, at every width
     (8-bit included); a stored scale may differ only where the oracle's value
     lies within the stage-1 tolerance of an fp16 rounding boundary.
Decode: <= 2e-3 absolute (one fp16 step where |o| >= 4 makes that step
larger) against the oracle's explicit-dequant attention over the GPU's own
packed cache (read through the oracle's own unpacker).
"""
import numpy as np
import pytest
import torch

from oracle import kvarn_oracle as O
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


def _dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def gpu_quantize(K, k, v, slot, num_blocks, cfg_str="kvarn_k4v2_g128", debug=True):
    cfg = K.config(cfg_str)
    hkv = k.shape[1]
    packed, scales = K.alloc_cache(cfg, num_blocks, hkv)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbg = torch.zeros((k.shape[0] // 128, hkv, 2, 256), dtype=torch.float32, device="cuda") if debug else None
    K.quantize_tiles(_dev(k), _dev(v), _dev(slot), packed, scales, cfg, dev_status=status, debug_logscales=dbg)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return (packed.cpu().numpy(), scales.cpu().numpy(), dbg.cpu().numpy() if debug else None)


# "scales within 1e-5 relative": the scale factor is 2^lt, so the log-scale
# may differ by log2(1 + 1e-5)
LOG_TOL = float(np.log2(1.0 + 1e-5))


def _fp16_neighbours_ok(gpu16, x64, tol=LOG_TOL):
    """gpu16 is the fp16 rounding of some value within tol of the oracle's
    fp64 x64 (either neighbour is correct at a rounding boundary); rounding
    is monotone, so that is the interval [fp16(x - tol), fp16(x + tol)]."""
    lo = (x64 - tol).astype(np.float16).astype(np.float64)
    hi = (x64 + tol).astype(np.float16).astype(np.float64)
    g = gpu16.astype(np.float64)
    return (g >= lo) & (g <= hi)


def stage3_bound(x, Lt, Lc, zero, step, y):
    """How far the kernel's fp32 value of (Z - zero) / step may lie from the
    oracle's fp64 one: the kernel's fp32 rotation (error below 2^-18 of the
    row's absolute sum), Z formed with two fp32 products of fp32 multipliers,
    the subtraction of zero and the product with the fp32 reciprocal of step."""
    mt = np.exp2(-Lt.astype(np.float64))[:, None]
    mc = np.exp2(-Lc.astype(np.float64))[None, :]
    dR = 2.0 ** -18 * np.abs(x.astype(np.float64)).sum(axis=1)[:, None]
    Z = np.float64(zero) + np.float64(step) * y
    return (dR * mt * mc + 2.0 ** -21 * (np.abs(Z) + abs(float(zero)))) / float(step) + 2.0 ** -21 * np.abs(y)


def check_tile(x, bits, codes, Lt, Lc, zero, step, cnt, lt_gpu=None, lc_gpu=None, where=()):
    """Stages 1-4 for one tile x ([128][128] fp16) against the GPU's stored
    codes / Lt / Lc / zero / step (stage 1 only with the GPU's fp32
    log-scales).  Adds counts to cnt."""
    r = O.quantize_tile(x, bits, 8)
    if lt_gpu is not None:   # stage 1
        e1 = np.max(np.abs(lt_gpu - r["lt"]))
        e2 = np.max(np.abs(lc_gpu - r["lc"]))
        cnt["worst_scale"] = max(cnt.get("worst_scale", 0.0), e1, e2)
        assert e1 <= LOG_TOL and e2 <= LOG_TOL, (where, e1, e2)
    # stage 2
    assert np.all(_fp16_neighbours_ok(Lt, r["lt"])), where
    assert np.all(_fp16_neighbours_ok(Lc, r["lc"])), where
    # stage 3: the oracle's fp64 code decision given the GPU's stored scales;
    # its own zero / step from those scales agree with the GPU's to fp32 rounding
    c_given, z2, s2, _ = O.quantize_given_scales(r["R"], Lt, Lc, bits)
    assert abs(float(z2) - float(zero)) <= 2e-6 * max(1.0, abs(float(zero))), (z2, zero)
    assert abs(float(s2) - float(step)) <= 2e-6 * float(s2), (s2, step)
    c_g, _, _, y_g = O.quantize_given_scales(r["R"], Lt, Lc, bits, zero, step)
    diff = codes != c_g
    if diff.any():
        assert np.all(np.abs(codes[diff] - c_g[diff]) == 1)
        dy = stage3_bound(x, Lt, Lc, zero, step, y_g)
        frac = np.abs(y_g - np.floor(y_g) - 0.5)
        assert np.all(frac[diff] <= dy[diff]), (where, frac[diff].max())
    # stage 4: end to end against the oracle's own codes.  A stored log-scale
    # the GPU rounded to the other fp16 neighbour (stage 2 allows it at a
    # rounding boundary) moves the codes of its whole row or column, and both
    # results are correct; the unique part is the codes whose row and column
    # scales agree.
    e2e = codes != r["codes"]
    flips_t = Lt != r["Lt"]
    flips_c = Lc != r["Lc"]
    same = (~flips_t)[:, None] & (~flips_c)[None, :]
    window_t = (r["lt"] - LOG_TOL).astype(np.float16) != (r["lt"] + LOG_TOL).astype(np.float16)
    window_c = (r["lc"] - LOG_TOL).astype(np.float16) != (r["lc"] + LOG_TOL).astype(np.float16)
    for k, v in (("mism_given", int(diff.sum())), ("mism_e2e", int(e2e.sum())), ("total", codes.size),
                 ("mism_same", int((e2e & same).sum())), ("total_same", int(same.sum())),
                 ("scale_flips", int(flips_t.sum() + flips_c.sum())), ("scales", 256),
                 ("scale_window", int(window_t.sum() + window_c.sum()))):
        cnt[k] = cnt.get(k, 0) + v


def assert_counts(cnt, kb, vb):
    """>= 99.99 % of codes bit-exact end to end, over all codes and over the
    codes whose row and column scales agree, at every width; the re-derived
    codes of stage 3 too; stored scales flip only inside the rounding-boundary
    window."""
    assert cnt["mism_given"] <= 1e-4 * cnt["total"], cnt
    assert cnt["mism_same"] <= 1e-4 * cnt["total_same"], cnt
    assert cnt["scale_flips"] <= cnt["scale_window"], cnt
    assert cnt["mism_e2e"] <= 1e-4 * cnt["total"], cnt


def check_quantize_parity(K, k, v, slot, num_blocks, kb, vb, groups=None, report=None):
    packed, scales, dbg = gpu_quantize(K, k, v, slot, num_blocks, f"kvarn_k{kb}v{vb}_g128")
    hkv = k.shape[1]
    n_groups = k.shape[0] // 128
    groups = range(n_groups) if groups is None else groups
    cnt = {}
    for g in groups:
        blk = int(slot[g * 128]) // 128
        for h in range(hkv):
            for side, src, bits in (("K", k, kb), ("V", v, vb)):
                x = np.ascontiguousarray(src[g * 128:(g + 1) * 128, h, :])
                codes, Lt, Lc, zero, step = O.read_tile(packed, scales, blk, h, side, kb, vb)
                sidx = 0 if side == "K" else 1
                check_tile(x, bits, codes, Lt, Lc, zero, step, cnt,
                           dbg[g, h, sidx, :128].astype(np.float64), dbg[g, h, sidx, 128:].astype(np.float64),
                           where=(g, h, side))
    if report is not None:
        report.update(cnt)
    assert_counts(cnt, kb, vb)
    return packed, scales


@pytest.mark.parametrize("kb,vb", [(4, 2), (2, 2), (4, 4), (8, 8)])
def test_quantize_parity_small(K, kb, vb):
    """24 token groups x 2 heads x {K,V} = 96 tiles, shuffled slots."""
    prob = inputs.quantize_batch(seed=7 + kb * 10 + vb, num_tokens=128 * 24, num_kv_heads=2, num_blocks=40)
    rep = {}
    check_quantize_parity(K, prob["k"], prob["v"], prob["slot_mapping"], prob["num_blocks"], kb, vb, report=rep)
    print(f"k{kb}v{vb}: {rep}")


def test_quantize_tiny_and_special_tiles(K):
    """The tiny workload, a zero tile and a rank-one tile."""
    w = inputs.tiny()
    check_quantize_parity(K, w.k_full, w.v_full, w.slot_mapping, w.num_blocks, 4, 2)
    z = np.zeros((128, 1, 128), np.float16)
    packed, scales, _ = gpu_quantize(K, z, z, np.arange(128, dtype=np.int64), 1)
    codes, Lt, Lc, zero, step = O.read_tile(packed, scales, 0, 0, "K", 4, 2)
    assert np.all(codes == 0) and step == 1.0 and np.all(np.isfinite(Lt.astype(np.float32)))


def test_quantize_status_on_bad_slot(K):
    cfg = K.config()
    k = torch.zeros((256, 1, 128), dtype=torch.float16, device="cuda")
    packed, scales = K.alloc_cache(cfg, 2, 1)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    slot = torch.tensor(list(range(128)) + [5 * 128 + i for i in range(128)], dtype=torch.int64, device="cuda")
    K.quantize_tiles(k, k, slot, packed, scales, cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1          # block 5 is beyond a 2-block pool
    status.zero_()
    slot[128:] = torch.arange(128, device="cuda") + 7   # misaligned start
    K.quantize_tiles(k, k, slot, packed, scales, cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1


# ------------------------------------------------------------------ decode

def run_decode(K, w, kb=4, vb=2, packed=None, scales=None):
    cfg = K.config(f"kvarn_k{kb}v{vb}_g128")
    if packed is None:
        packed, scales = K.alloc_cache(cfg, w.num_blocks, w.num_kv_heads)
        if w.k_full.shape[0]:
            K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention(_dev(w.q), packed, scales, _dev(w.tail), _dev(w.block_table), _dev(w.seq_lens), cfg,
                             dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out.cpu().numpy(), packed.cpu().numpy(), scales.cpu().numpy()


def decode_bound(ref16):
    """2e-3 absolute, or one fp16 step where the output's own spacing is
    larger (|o| >= 4): two fp16 results cannot be closer than one step
    unless they are equal."""
    r = np.abs(ref16.astype(np.float16))
    step = np.spacing(r).astype(np.float64)
    return np.maximum(DECODE_TOL, step)


def decode_errors(out, ref, pairs):
    err = np.zeros(0)
    bnd = np.zeros(0)
    mag = np.zeros(0)
    for b, j in pairs:
        e = np.abs(out[b, j].astype(np.float64) - ref[b, j].astype(np.float64))
        err = np.concatenate([err, e])
        bnd = np.concatenate([bnd, decode_bound(ref[b, j])])
        mag = np.concatenate([mag, np.abs(ref[b, j].astype(np.float64))])
    return err, bnd, mag


def check_decode(K, w, kb=4, vb=2, heads=None):
    out, packed, scales = run_decode(K, w, kb, vb)
    ref = O.decode(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, w.num_kv_heads, kb, vb, heads=heads)
    pairs = heads if heads is not None else [(b, j) for b in range(w.num_seqs) for j in range(w.num_q_heads)]
    err, bnd, mag = decode_errors(out, ref, pairs)
    small = mag < 4
    print(f"decode max err {err.max():.2e} (|o|<4: {err[small].max() if small.any() else 0:.2e}, "
          f"|o|>=4: {err[~small].max() if (~small).any() else 0:.2e}, n>=4: {(~small).sum()})")
    assert np.all(err <= bnd), float(np.max(err - bnd))
    return float(err.max()), out


@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_parity_ragged(K, G):
    """Tail-only, exactly one tile, tile + tail, many tiles (several splits), empty."""
    lens = [77, 128, 300, 40 * 128 + 5, 0, 129, 1]
    w = inputs.make_decode_workload("ragged", lens, 2 * G, 2, seed=300 + G, pool_blocks=80)
    err, out = check_decode(K, w)
    assert np.all(out[4] == 0)                      # empty sequence
    print(f"G={G} max abs err {err:.2e}")


@pytest.mark.parametrize("kb,vb", [(2, 2), (4, 4), (8, 8), (2, 4), (8, 2)])
def test_decode_parity_precisions(K, kb, vb):
    w = inputs.make_decode_workload("prec", [20 * 128 + 33, 3 * 128], 16, 2, seed=400 + kb * 10 + vb)
    err, _ = check_decode(K, w, kb, vb)
    print(f"k{kb}v{vb} max abs err {err:.2e}")


def test_decode_tiny(K):
    err, _ = check_decode(K, inputs.tiny())
    print(f"tiny max abs err {err:.2e}")


def test_decode_status_codes(K):
    w = inputs.make_decode_workload("st", [256, 300], 4, 1, seed=9, pool_blocks=4)
    cfg = K.config()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, 1)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = w.block_table.copy()
    bt[1, 1] = 99                                   # beyond the 4-block pool
    K.decode_attention(_dev(w.q), packed, scales, _dev(w.tail), _dev(bt), _dev(w.seq_lens), cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    status.zero_()
    sl = w.seq_lens.copy()
    sl[0] = 128 * w.max_blocks_per_seq + 1          # longer than the block table
    K.decode_attention(_dev(w.q), packed, scales, _dev(w.tail), _dev(w.block_table), _dev(sl), cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 3


def test_decode_quality_vs_fp16_reported(K):
    """Reported, not gated: k4v2 decode against fp16 attention on the unquantised cache."""
    w = inputs.make_decode_workload("q", [16 * 128 + 50] * 2, 16, 2, seed=11)
    out, _, _ = run_decode(K, w)
    rows_k, rows_v = [], []
    for b in range(2):
        s, e = w.token_range(b)
        tl = int(w.seq_lens[b]) % 128
        rows_k.append(np.concatenate([w.k_full[s:e], w.tail[b, 0, :, :tl].transpose(1, 0, 2)]))
        rows_v.append(np.concatenate([w.v_full[s:e], w.tail[b, 1, :, :tl].transpose(1, 0, 2)]))
    ref = O.decode_uncompressed(w.q, rows_k, rows_v, w.seq_lens, 2).astype(np.float64)
    rel = np.abs(out.astype(np.float64) - ref).mean() / np.abs(ref).mean()
    print(f"k4v2 vs fp16 attention: mean relative error {rel:.3f}")
    assert rel < 1.0


# ------------------------------------------------------------------ decode step with append

APPEND_LENS = [0, 127, 128 + 127, 300, 128, 40 * 128 + 127, 5, 2 * 128]


def run_append_case(K, lens, hq, hkv, seed, kb=4, vb=2):
    """One decode step with append on the GPU against the oracle's step over
    the GPU's own pre-step cache.  Returns the GPU and oracle results."""
    full = sum(int(L) // 128 for L in lens)
    w = inputs.make_decode_workload("append", lens, hq, hkv, seed, pool_blocks=full + 8)
    k_new, v_new, bt = inputs.append_step(w, seed + 1)
    cfg = K.config(f"kvarn_k{kb}v{vb}_g128")
    packed, scales = K.alloc_cache(cfg, w.num_blocks, hkv)
    if w.k_full.shape[0]:
        K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
    torch.cuda.synchronize()
    p0, s0 = packed.cpu().numpy(), scales.cpu().numpy()
    tail = _dev(w.tail)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention_append(_dev(w.q), _dev(k_new), _dev(v_new), packed, scales, tail, _dev(bt),
                                    _dev(w.seq_lens), cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, p2, s2, t2 = O.decode_append(w.q, k_new, v_new, p0, s0, w.tail, bt, w.seq_lens, hkv, kb, vb)
    return dict(w=w, bt=bt, k_new=k_new, v_new=v_new, cfg=cfg, out=out.cpu().numpy(), ref=ref,
                packed=packed, scales=scales, tail=tail, p0=p0, s0=s0, p2=p2, s2=s2, t2=t2)


@pytest.mark.parametrize("G", [1, 8])
def test_decode_append_parity(K, G):
    """Lengths before the step cover: empty, a tail filled with no full tile,
    a fill after full tiles, mid-tile, a tail starting, a long fill.  Output
    within the decode bound; the tail written bit-exactly; blocks other than
    the filled ones untouched; filled blocks through the quantiser's stages."""
    r = run_append_case(K, APPEND_LENS, 2 * G, 2, seed=500 + G)
    w = r["w"]
    pairs = [(b, j) for b in range(w.num_seqs) for j in range(w.num_q_heads)]
    err, bnd, _ = decode_errors(r["out"], r["ref"], pairs)
    print(f"append G={G}: decode max err {err.max():.2e}")
    assert np.all(err <= bnd)
    assert np.array_equal(r["tail"].cpu().numpy(), r["t2"])
    packed, scales = r["packed"].cpu().numpy(), r["scales"].cpu().numpy()
    filled = {int(r["bt"][b, L // 128]): b for b, L in enumerate(APPEND_LENS) if L % 128 == 127}
    others = [i for i in range(w.num_blocks) if i not in filled]
    assert np.array_equal(packed[others], r["p0"][others]) and np.array_equal(scales[others], r["s0"][others])
    cnt = {}
    for blk, b in filled.items():
        for h in range(w.num_kv_heads):
            for sidx, side, bits in ((0, "K", 4), (1, "V", 2)):
                x = np.ascontiguousarray(r["t2"][b, sidx, h])
                codes, Lt, Lc, zero, step = O.read_tile(packed, scales, blk, h, side, 4, 2)
                check_tile(x, bits, codes, Lt, Lc, zero, step, cnt, where=(b, h, side))
    assert cnt["total"] == len(filled) * w.num_kv_heads * 2 * 128 * 128
    assert_counts(cnt, 4, 2)


def test_decode_append_then_next_step(K):
    """The step after an append (seq_len + 1, plain decode) reads the filled
    tile from the packed cache: parity against the oracle on the GPU's cache."""
    r = run_append_case(K, APPEND_LENS, 8, 2, seed=520)
    w = r["w"]
    lens1 = (w.seq_lens + 1).astype(np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention(_dev(w.q), r["packed"], r["scales"], r["tail"], _dev(r["bt"]), _dev(lens1), r["cfg"],
                             dev_status=status).cpu().numpy()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.decode(w.q, r["packed"].cpu().numpy(), r["scales"].cpu().numpy(), r["tail"].cpu().numpy(), r["bt"],
                   lens1, 2, 4, 2)
    err, bnd, _ = decode_errors(out, ref, [(b, j) for b in range(w.num_seqs) for j in range(8)])
    assert np.all(err <= bnd)


def test_decode_append_status(K):
    """A step whose token would not fit the block table reports a bad length
    and leaves that sequence's output 0; a bad block id for a filled tile
    reports a bad block."""
    w = inputs.make_decode_workload("append", [128, 127], 2, 1, seed=530, pool_blocks=4, max_blocks_per_seq=2)
    k_new, v_new, bt = inputs.append_step(w, 531)
    cfg = K.config()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, 1)
    K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt1 = np.ascontiguousarray(bt[:, :1])                 # max_blocks 1: L = 128 has no room
    out = K.decode_attention_append(_dev(w.q), _dev(k_new), _dev(v_new), packed, scales, _dev(w.tail), _dev(bt1),
                                    _dev(w.seq_lens), cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 3                       # KVARN_DEV_BAD_SEQ_LEN
    assert np.all(out.cpu().numpy()[0] == 0)
    status.zero_()
    bt2 = bt.copy()
    bt2[1, 0] = w.num_blocks + 5                          # the filled tile's block is out of range
    K.decode_attention_append(_dev(w.q), _dev(k_new), _dev(v_new), packed, scales, _dev(w.tail), _dev(bt2),
                              _dev(w.seq_lens), cfg, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2                       # KVARN_DEV_BAD_BLOCK


# ------------------------------------------------------------------ full-size, sampled

def test_full_size_qwen3_32b_sampled(K):
    """The Qwen3-32B-shaped workload (B=8, 16K + ragged tail, 64/8 heads) in the
    bench's launch configuration: every tile quantised and decoded on the
    GPU.  The quantiser is checked through stages 1-4 on 256 sampled tiles
    (16 token groups x all 8 KV heads x K and V) with the contract's bounds;
    the decode on sampled outputs, including every head of one sequence."""
    w = inputs.qwen3_32b()
    cfg = K.config()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, w.num_kv_heads)
    dbg = torch.zeros((w.k_full.shape[0] // 128, 8, 2, 256), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg, dev_status=status,
                     debug_logscales=dbg)
    out, packed_h, scales_h = run_decode(K, w, packed=packed, scales=scales)
    assert int(status.item()) == 0
    dbg_h = dbg.cpu().numpy()
    rng = np.random.default_rng(5)
    n_groups = w.k_full.shape[0] // 128
    cnt = {}
    for g in rng.choice(n_groups, size=16, replace=False):
        blk = int(w.slot_mapping[g * 128]) // 128
        for h in range(8):
            for sidx, side, src, bits in ((0, "K", w.k_full, 4), (1, "V", w.v_full, 2)):
                x = np.ascontiguousarray(src[g * 128:(g + 1) * 128, h])
                codes, Lt, Lc, z, s = O.read_tile(packed_h, scales_h, blk, h, side, 4, 2)
                check_tile(x, bits, codes, Lt, Lc, z, s, cnt, dbg_h[g, h, sidx, :128].astype(np.float64),
                           dbg_h[g, h, sidx, 128:].astype(np.float64), where=(int(g), h, side))
    print(f"full size k4v2, 256 tiles: {cnt}")
    assert cnt["total"] == 256 * 128 * 128
    assert_counts(cnt, 4, 2)
    heads = [(0, 0), (3, 17), (7, 63), (5, 40)] + [(2, j) for j in range(64)]
    ref = O.decode(w.q, packed_h, scales_h, w.tail, w.block_table, w.seq_lens, 8, 4, 2, heads=heads)
    err, bnd, _ = decode_errors(out, ref, heads)
    print(f"full size decode: max err {err.max():.2e} over {len(heads)} outputs")
    assert np.all(err <= bnd)
    assert np.all(np.isfinite(out.astype(np.float32)))


def test_llama3_8b_config_decode_all_outputs(K):
    """The Llama-3-8B-shaped decode (B=16, 4096 tokens each, 32/8 heads,
    shuffled 512-block pool): every output against the oracle over the GPU's
    own cache."""
    w = inputs.llama3_8b()
    err, _ = check_decode(K, w)
    print(f"llama3_8b B16 x 4K: max abs err {err:.2e}")


def test_llama3_70b_config_decode_sampled(K):
    """The Llama-3-70B-shaped long-context decode (B=4, lengths U[1024,
    131072] from the seed, 64/8 heads): 16 sampled outputs, 4 per sequence
    over 2 KV heads each, the longest sequence included, against the oracle
    over the GPU's own cache."""
    w = inputs.llama3_70b()
    assert int(w.seq_lens.max()) > 100_000
    out, packed_h, scales_h = run_decode(K, w)
    rng = np.random.default_rng(6)
    worst = 0.0
    for b in range(w.num_seqs):
        for h in rng.choice(8, size=2, replace=False):
            heads = [(b, int(h) * 8 + int(j)) for j in rng.choice(8, size=2, replace=False)]
            ref = O.decode(w.q, packed_h, scales_h, w.tail, w.block_table, w.seq_lens, 8, 4, 2, heads=heads)
            err, bnd, _ = decode_errors(out, ref, heads)
            assert np.all(err <= bnd), (b, int(h))
            worst = max(worst, float(err.max()))
    print(f"llama3_70b lengths {w.seq_lens.tolist()}: max abs err {worst:.2e}")


def test_tensor_parallel_kv_head_shards_on_gpu(K):
    """Tensor parallelism over KV heads (the pages' TP=2 setting, [hypho]
    这就是 KVarN 想解决的问题): each of two shards quantises and decodes only
    its own KV heads and the query heads that read them, on its own cache
    slice, through the CUDA path; the concatenated outputs equal the oracle's
    decode of the whole problem."""
    from bit_kv_cache_15_b200.sharding import kv_head_shard
    w = inputs.make_decode_workload("tp", [9 * 128 + 70, 3 * 128, 200, 20 * 128 + 1], 32, 8, seed=960,
                                    pool_blocks=40)
    cfg = K.config()
    out = np.zeros_like(w.q)
    caches = []
    for rank in range(2):
        kv, qh = kv_head_shard(8, 32, rank, 2)
        ks, qs = slice(kv.start, kv.stop), slice(qh.start, qh.stop)
        packed, scales = K.alloc_cache(cfg, w.num_blocks, len(kv))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        K.quantize_tiles(_dev(w.k_full[:, ks]), _dev(w.v_full[:, ks]), _dev(w.slot_mapping), packed, scales, cfg,
                         dev_status=status)
        o = K.decode_attention(_dev(w.q[:, qs]), packed, scales, _dev(w.tail[:, :, ks]), _dev(w.block_table),
                               _dev(w.seq_lens), cfg, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        out[:, qs] = o.cpu().numpy()
        caches.append((packed.cpu().numpy(), scales.cpu().numpy()))
    packed_all = np.concatenate([c[0] for c in caches], axis=1)
    scales_all = np.concatenate([c[1] for c in caches], axis=1)
    ref = O.decode(w.q, packed_all, scales_all, w.tail, w.block_table, w.seq_lens, 8, 4, 2)
    err, bnd, _ = decode_errors(out, ref, [(b, j) for b in range(w.num_seqs) for j in range(32)])
    print(f"TP=2 over KV heads: max abs err {err.max():.2e}")
    assert np.all(err <= bnd)
    # each shard's cache is the whole problem's cache for its heads
    ref_p, ref_s = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, 8, w.num_blocks, 4, 2,
                                    groups=range(2))
    blk = [int(w.slot_mapping[g * 128]) // 128 for g in range(2)]
    mism = float((packed_all[blk] != ref_p[blk]).mean())
    assert mism < 1e-3, mism


@pytest.mark.parametrize("lens,hq,hkv,heads", [
    ([60000 + 77, 5000, 1153, 127, 0], 64, 8, [(0, 0), (0, 37), (1, 8), (2, 63), (3, 5), (4, 0)]),
    ([40000], 8, 1, [(0, 0), (0, 7)]),
])
def test_decode_long_ragged_sampled(K, lens, hq, hkv, heads):
    """Long, ragged sequences: a pair's tiles span many CTAs of the work split
    (one 40K sequence alone spreads over every CTA), so the merge walks many
    records.  Sampled heads against the oracle on the GPU's own cache."""
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("long", lens, hq, hkv, seed=700 + hkv, pool_blocks=full + 3)
    out, packed_h, scales_h = run_decode(K, w)
    ref = O.decode(w.q, packed_h, scales_h, w.tail, w.block_table, w.seq_lens, hkv, 4, 2, heads=heads)
    err, bnd, _ = decode_errors(out, ref, heads)
    print(f"long ragged Hkv={hkv}: decode max err {err.max():.2e}")
    assert np.all(err <= bnd)
    assert np.all(out[[b for b, L in enumerate(lens) if L == 0]] == 0)


# ------------------------------------------------------------------ multi-query

@pytest.mark.parametrize("hq,hkv,qlen", [(64, 8, 4), (8, 8, 3), (16, 2, 2), (8, 2, 1), (8, 8, 128), (16, 2, 37)])
def test_decode_multiquery_parity(K, hq, hkv, qlen):
    """q_len queries per sequence, causal: (query, head) columns in groups of
    8 per KV head (4 groups at 64/8 heads x 4 queries, 128 at 8/8 x 128).
    Lengths cover a query block ending a full tile, queries inside the last
    full tile (tail shorter than q_len - 1, or no tail at all), a tail-only
    sequence, long sequences and one shorter than q_len."""
    lens = [256 + qlen - 1, 1024 + 127, 40 * 128 + 10, 7 + qlen, 128 + max(qlen - 2, 0), 3 * 128 + 50,
            5 * 128, 2 * 128 + 1, max(qlen - 1, 0)]
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("mq", lens, hq, hkv, seed=800 + qlen, pool_blocks=full + 2)
    cfg = K.config()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, hkv)
    K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
    q = np.random.default_rng(801).standard_normal((len(lens), qlen, hq, 128)).astype(np.float16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.decode_attention_multiquery(_dev(q), packed, scales, _dev(w.tail), _dev(w.block_table), _dev(w.seq_lens),
                                        cfg, dev_status=status).cpu().numpy()
    torch.cuda.synchronize()
    # q_len = 1 is plain decode, where an empty sequence is valid (output 0)
    bad = [b for b, L in enumerate(lens) if qlen > 1 and L < qlen]
    assert int(status.item()) == (3 if bad else 0)
    inside = [b for b, L in enumerate(lens) if L >= qlen and L >= 128 and L % 128 + 1 < qlen]
    if qlen > 2:
        assert inside, "some sequence must place queries inside its last full tile"
    ref = O.decode_multiquery(q, packed.cpu().numpy(), scales.cpu().numpy(), w.tail, w.block_table, w.seq_lens,
                              hkv, 4, 2)
    err = np.abs(out.astype(np.float64) - ref.astype(np.float64))
    bnd = decode_bound(ref)
    print(f"multiquery {hq}/{hkv} q_len={qlen}: max err {err.max():.2e} (inside a packed tile: {inside})")
    assert np.all(err <= bnd)
    for b in bad:
        assert np.all(out[b] == 0)


def test_decode_many_short_sequences(K):
    """100 ragged sequences (0 to 600 tokens): the work split's start search
    scans the sequences 32 at a time, and most CTAs straddle several pairs."""
    rng = np.random.default_rng(900)
    lens = [int(x) for x in rng.integers(0, 600, size=100)]
    lens[7] = 0
    full = sum(L // 128 for L in lens)
    w = inputs.make_decode_workload("many", lens, 4, 2, seed=901, pool_blocks=full + 1)
    out, packed_h, scales_h = run_decode(K, w)
    heads = [(b, j) for b in range(0, 100, 3) for j in (0, 3)]
    ref = O.decode(w.q, packed_h, scales_h, w.tail, w.block_table, w.seq_lens, 2, 4, 2, heads=heads)
    err, bnd, _ = decode_errors(out, ref, heads)
    assert np.all(err <= bnd)
    assert np.all(out[7] == 0)
    # the same cache read as 3-query verify steps (sequences shorter than 3 give 0)
    cfg = K.config()
    q = rng.standard_normal((100, 3, 4, 128)).astype(np.float16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq = K.decode_attention_multiquery(_dev(q), torch.from_numpy(packed_h).cuda(), torch.from_numpy(scales_h).cuda(),
                                       _dev(w.tail), _dev(w.block_table), _dev(w.seq_lens), cfg,
                                       dev_status=status).cpu().numpy()
    torch.cuda.synchronize()
    trip = [(b, i, j) for b in range(1, 100, 4) for i in range(3) for j in (1, 2)]
    ref3 = O.decode_multiquery(q, packed_h, scales_h, w.tail, w.block_table, w.seq_lens, 2, 4, 2, heads=trip)
    for b, i, j in trip:
        e = np.abs(mq[b, i, j].astype(np.float64) - ref3[b, i, j].astype(np.float64))
        assert np.all(e <= decode_bound(ref3[b, i, j])), (b, i, j)


def test_decode_append_consecutive_steps(K):
    """Five consecutive append steps per sequence (125 -> 130 tokens and
    252 -> 257, the tiles filling on the way), each against the oracle's step
    on the GPU's own state before it."""
    w = inputs.make_decode_workload("steps", [125, 128 + 124], 8, 2, seed=950, pool_blocks=6, max_blocks_per_seq=3)
    bt = w.block_table.copy()
    free = [i for i in range(w.num_blocks) if i != int(bt[1, 0])]   # blocks no full tile uses
    bt[0, 0], bt[0, 1], bt[1, 1], bt[1, 2] = free[:4]               # for the tiles that fill
    cfg = K.config()
    packed, scales = K.alloc_cache(cfg, w.num_blocks, 2)
    if w.k_full.shape[0]:
        K.quantize_tiles(_dev(w.k_full), _dev(w.v_full), _dev(w.slot_mapping), packed, scales, cfg)
    tail = _dev(w.tail)
    lens = w.seq_lens.copy()
    rng = np.random.default_rng(951)
    outl = inputs.pick_outlier_channels(np.random.default_rng(952), 2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(5):
        k_new, v_new = inputs.gen_k(rng, 2, 2, outl), inputs.gen_v(rng, 2, 2)
        p0, s0, t0 = packed.cpu().numpy(), scales.cpu().numpy(), tail.cpu().numpy()
        out = K.decode_attention_append(_dev(w.q), _dev(k_new), _dev(v_new), packed, scales, tail, _dev(bt),
                                        _dev(lens), cfg, dev_status=status).cpu().numpy()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref, p2, s2, t2 = O.decode_append(w.q, k_new, v_new, p0, s0, t0, bt, lens, 2, 4, 2)
        err, bnd, _ = decode_errors(out, ref, [(b, j) for b in range(2) for j in range(8)])
        assert np.all(err <= bnd), step
        assert np.array_equal(tail.cpu().numpy(), t2)
        lens = lens + 1
