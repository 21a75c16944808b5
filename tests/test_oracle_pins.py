"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against what the pages or the mathematics fix:
a closed form, an invariant, an independent algorithm, brute force on a tiny
case or a value the pages print (tests/golden/pages_facts.txt).  None of
them re-types the oracle's own formula.
"""
import os

import numpy as np
import pytest

from oracle import kvarn_oracle as O
from bit_kv_cache_15_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.txt")


def _facts():
    out = {}
    for line in open(GOLDEN, encoding="utf-8"):
        if line.startswith("#") or not line.strip():
            continue
        k, v, _ = [x.strip() for x in line.split("|", 2)]
        out[k] = v
    return out


def _tile(seed, side="K"):
    rng = np.random.default_rng(seed)
    if side == "K":
        return inputs.gen_k(rng, 128, 1)[:, 0, :]
    return inputs.gen_v(rng, 128, 1)[:, 0, :]


# ----------------------------------------------------------------- the pages

def test_config_string_from_pages():
    f = _facts()
    kb, vb, g = O.parse_config(f["config_string"])
    assert (kb, vb, g) == (int(f["default_k_bits"]), int(f["default_v_bits"]), int(f["tile_tokens"]))
    assert O.TILE == int(f["tile_tokens"])


def test_capacity_closed_form_within_pages_range():
    """k4v2 stores (8192 + 4096 + 2 * 528) / 128 = 104.25 B per token and KV
    head against 256 B of fp16 K plus 256 B of fp16 V: 4.91x, inside the
    pages' 3-5x."""
    f = _facts()
    b = O.capacity_bytes_per_token_head(4, 2)
    assert b == 104.25
    ratio = 512.0 / b
    assert float(f["capacity_vs_fp16_min"]) <= ratio <= float(f["capacity_vs_fp16_max"])
    # the other precisions, for the record: k8v8 and k4v4 fall below 3x, k2v2 above 5x
    assert O.capacity_bytes_per_token_head(8, 8) == 264.25
    assert O.capacity_bytes_per_token_head(2, 2) == 72.25


# ------------------------------------------------------------ P1 / P2 rotation

def _sylvester(n):
    h = np.array([[1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _fwht_butterfly(x):
    x = np.array(x, dtype=np.float64, copy=True)
    n = x.shape[-1]
    hlen = 1
    while hlen < n:
        y = x.reshape(x.shape[:-1] + (n // (2 * hlen), 2, hlen))
        a = y[..., 0, :].copy()
        b = y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        x = y.reshape(x.shape)
        hlen *= 2
    return x


def test_hadamard_orthogonal_and_sylvester():
    H = O.hadamard()
    assert np.array_equal(H @ H.T, 128 * np.eye(128, dtype=np.int64))
    assert np.array_equal(H, _sylvester(128))
    assert np.array_equal(H, H.T)


def test_rotation_exact_against_butterfly():
    for seed in range(4):
        x = _tile(seed)
        r = O.rotate(x)
        assert np.array_equal(r, _fwht_butterfly(x.astype(np.float64)))


def test_rotation_keeps_attention_scores():
    """The pages: the rotation is orthogonal and does not change attention
    scores.  (q H) . (k H) / 128 = q . k."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal(128).astype(np.float16)
    k = _tile(3)
    lhs = (O.rotate(k) @ O.rotate(q)) / 128.0
    rhs = k.astype(np.float64) @ q.astype(np.float64)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


# ------------------------------------------------------- P3 / P4 normalisation

def _sinkhorn_knopp(A, iters=2000):
    """Textbook multiplicative Sinkhorn-Knopp: r, c > 0 with diag(r) A diag(c)
    having every row and every column sum equal to A.shape[0]."""
    n = A.shape[0]
    r = np.ones(n)
    c = np.ones(n)
    for _ in range(iters):
        c = n / (A.T @ r)
        r = n / (A @ c)
    return r, c


@pytest.mark.parametrize("side", ["K", "V"])
def test_normalisation_balances_rows_and_columns(side):
    worst_c = 0.0
    for seed in range(10):
        x = _tile(100 + seed, side)
        R = O.rotate(x)
        lt, lc = O.normalize_logscales(R, 8)
        N = R * np.exp2(-(lt[:, None] + lc[None, :]))
        rms_t = np.sqrt((N * N).mean(axis=1))
        rms_c = np.sqrt((N * N).mean(axis=0))
        assert np.max(np.abs(rms_t - 1)) < 1e-12      # last pass is the token pass
        worst_c = max(worst_c, np.max(np.abs(rms_c - 1)))
    assert worst_c < 1e-3


@pytest.mark.parametrize("side", ["K", "V"])
def test_normalisation_matches_textbook_sinkhorn(side):
    """The log-space iteration is Sinkhorn-Knopp on R*R: the combined scale
    lt[t] + lc[d] (the part that does not depend on the gauge) agrees with
    -1/2 log2(r_t c_d) of a converged multiplicative Sinkhorn-Knopp."""
    x = _tile(55, side)
    R = O.rotate(x)
    lt, lc = O.normalize_logscales(R, 8)
    r, c = _sinkhorn_knopp(R * R)
    sk = -0.5 * np.log2(r[:, None] * c[None, :])
    assert np.max(np.abs((lt[:, None] + lc[None, :]) - sk)) < 1e-5


def _rank1_tile(seed):
    rng = np.random.default_rng(seed)
    a = np.exp2(rng.integers(-2, 2, size=128)).astype(np.float64)     # 1/4 .. 2
    b = np.exp2(rng.integers(0, 3, size=128)).astype(np.float64)      # 1 .. 4
    sign = np.where(rng.random((128, 128)) < 0.5, -1.0, 1.0)
    R = sign * a[:, None] * b[None, :]
    X = R @ O.hadamard().astype(np.float64) / 128.0
    X16 = X.astype(np.float16)
    assert np.array_equal(X16.astype(np.float64), X)                  # exactly representable
    return X16, R, a, b


def test_rank_one_tile_normalises_in_one_iteration():
    X16, R, a, b = _rank1_tile(3)
    assert np.array_equal(O.rotate(X16), R)
    lt, lc = O.normalize_logscales(R, 1)
    assert np.max(np.abs(lt[:, None] + lc[None, :] - np.log2(a[:, None] * b[None, :]))) < 1e-12
    for bits in (2, 4, 8):
        r = O.quantize_tile(X16, bits, 8)
        assert set(np.unique(r["codes"])) <= {0, 2 ** bits - 1}
        assert np.array_equal(r["codes"] == 0, R < 0)


def test_zero_tile_is_floored_not_infinite():
    r = O.quantize_tile(np.zeros((128, 128), np.float16), 4, 8)
    assert np.all(np.isfinite(r["lt"])) and np.all(np.isfinite(r["lc"]))
    assert np.all(r["codes"] == 0) and r["step"] == 1.0


# ------------------------------------------------------------- P5 round trip

@pytest.mark.parametrize("bits", [2, 4, 8])
def test_round_trip_within_half_step(bits):
    for seed in range(6):
        x = _tile(200 + seed, "K" if seed % 2 == 0 else "V")
        r = O.quantize_tile(x, bits, 8)
        Z = (r["R"] * np.exp2(-r["Lt"].astype(np.float64))[:, None]) * np.exp2(-r["Lc"].astype(np.float64))[None, :]
        back = np.float64(r["zero"]) + np.float64(r["step"]) * r["codes"]
        assert np.max(np.abs(back - Z)) <= 0.5 * float(r["step"]) * (1 + 1e-5)
        assert r["codes"].flat[np.argmin(Z)] == 0
        assert r["codes"].flat[np.argmax(Z)] == 2 ** bits - 1
        assert r["codes"].min() >= 0 and r["codes"].max() <= 2 ** bits - 1


def test_dequantised_tile_bounds_in_original_domain():
    """Dequantisation returns to the original fp16 data within the bound the
    step implies: per element in the rotated domain, and (by orthogonality)
    per token row in the original domain."""
    x = _tile(11)
    r = O.quantize_tile(x, 4, 8)
    rot = O.dequantize_rotated(r["codes"], r["Lt"], r["Lc"], r["zero"], r["step"])
    scale = np.exp2(r["Lt"].astype(np.float64)[:, None] + r["Lc"].astype(np.float64)[None, :])
    bound = scale * 0.5 * float(r["step"]) * (1 + 1e-5) + 1e-3 * scale * float(r["step"])
    assert np.all(np.abs(rot - r["R"]) <= bound)
    back = O.dequantize(r["codes"], r["Lt"], r["Lc"], r["zero"], r["step"])
    err_rows = np.linalg.norm(back - x.astype(np.float64), axis=1)
    err_rot = np.linalg.norm(rot - r["R"], axis=1) / np.sqrt(128)
    assert np.allclose(err_rows, err_rot, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- layout

@pytest.mark.parametrize("side", ["K", "V"])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_layout_is_a_bijection(side, bits):
    t, d = np.meshgrid(np.arange(128), np.arange(128), indexing="ij")
    byte, bit0 = O.code_position(side, bits, t, d)
    flat = (byte * 8 + bit0).ravel()
    assert flat.min() == 0 and flat.max() == 128 * 128 * bits - bits
    assert len(np.unique(flat)) == 128 * 128
    assert np.all(flat % bits == 0)


def test_layout_hand_examples():
    # worked by hand from the layout definition for K, 4-bit codes
    cases = {(0, 0): (0, 0), (0, 1): (2, 0), (8, 0): (0, 4), (1, 0): (64, 0),
             (0, 16): (4, 0), (0, 64): (512, 0), (9, 9): (67, 4)}
    for (t, d), want in cases.items():
        got = O.code_position("K", 4, t, d)
        assert (int(got[0]), int(got[1])) == want, (t, d)
    # V, 2-bit: (t=0,d=0) first crumb; (t=16,d=0) is block 8 -> rho 32 -> word 4 -> chunk 1
    assert tuple(int(v) for v in O.code_position("V", 2, 0, 0)) == (0, 0)
    assert tuple(int(v) for v in O.code_position("V", 2, 16, 0)) == (512, 0)
    assert tuple(int(v) for v in O.code_position("V", 2, 0, 16)) == (1, 0)


@pytest.mark.parametrize("side", ["K", "V"])
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_layout_matches_mma_fragment(side, bits):
    """Lane l's 16-byte chunks, decoded as (register, half) pairs, hold the
    elements of the mma.m16n8k16 A operand fragment the PTX ISA assigns to
    lane l: a0,a1 at (row g, col 2c, 2c+1), a2,a3 at row g+8, a4,a5 at col
    +8, a6,a7 at row g+8, col +8, with g = l / 4, c = l % 4.  K tiles are
    A = codes[t][d] (rows tokens); V tiles are A = codes^T (rows channels)."""
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 2 ** bits, size=(128, 128))
    buf = O.pack_codes(codes, side, bits)
    words = buf.view("<u4")
    per = 16 // bits
    n_words = 16 * bits
    for lane in (0, 5, 31):
        g, c = lane // 4, lane % 4
        lane_words = [words[((w // 4) * 32 + lane) * 4 + w % 4] for w in range(n_words)]
        for blk in (0, 9, 63):
            rb, cb = blk // 8, blk % 8       # (token block, channel block)
            for j in range(4):
                rho = 4 * blk + j
                w = int(lane_words[rho // per])
                slot = rho % per
                lo = (w >> (bits * slot)) & (2 ** bits - 1)
                hi = (w >> (16 + bits * slot)) & (2 ** bits - 1)
                row = g + 8 * (j % 2)
                col = 2 * c + 8 * (j // 2)
                for half, val in ((0, lo), (1, hi)):
                    if side == "K":
                        t, d = 16 * rb + row, 16 * cb + col + half
                    else:
                        d, t = 16 * cb + row, 16 * rb + col + half
                    assert val == codes[t, d]


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(0)
    for side in "KV":
        for bits in (2, 4, 8):
            c = rng.integers(0, 2 ** bits, size=(128, 128))
            assert np.array_equal(O.unpack_codes(O.pack_codes(c, side, bits), side, bits), c)


# --------------------------------------------------------------- P6 / P7 decode

def _small_problem(seq_lens, Hq=4, Hkv=2, seed=5, kb=4, vb=2):
    w = inputs.make_decode_workload("t", seq_lens, Hq, Hkv, seed)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, Hkv, w.num_blocks, kb, vb)
    return w, packed, scales


def test_folded_equals_explicit_dequant():
    w, packed, scales = _small_problem([300, 128, 77, 256], Hq=4, Hkv=2)
    folded = O.decode_folded(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, 2, 4, 2)
    for b in range(4):
        for j in range(4):
            K, V = O.gather_kv(packed, scales, w.tail, w.block_table, int(w.seq_lens[b]), b, j // 2, 4, 2)
            ref = O.attention(w.q[b, j], K, V, 1 / np.sqrt(128))
            assert np.max(np.abs(folded[b, j] - ref)) < 1e-10


def _brute_attention(q, K, V, scale):
    s = [scale * sum(float(q[i]) * float(K[t][i]) for i in range(len(q))) for t in range(len(K))]
    m = max(s)
    e = [np.exp(x - m) for x in s]
    tot = sum(e)
    return np.array([sum(e[t] * V[t][i] for t in range(len(K))) / tot for i in range(len(q))])


def test_decode_special_cases():
    # tail only, one token: the output is that token's value row
    w, packed, scales = _small_problem([1, 130], Hq=2, Hkv=1)
    out = O.decode(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, 1, 4, 2)
    assert np.array_equal(out[0, 0], w.tail[0, 1, 0, 0])
    # q = 0: uniform weights, the output is the mean of the restored values
    q0 = np.zeros_like(w.q)
    out0 = O.decode(q0, packed, scales, w.tail, w.block_table, w.seq_lens, 1, 4, 2)
    K, V = O.gather_kv(packed, scales, w.tail, w.block_table, 130, 1, 0, 4, 2)
    assert np.array_equal(out0[1, 0], V.mean(axis=0).astype(np.float16))
    # a single full tile, no tail: brute-force softmax over the restored rows
    w1, p1, s1 = _small_problem([128], Hq=1, Hkv=1, seed=9)
    K1, V1 = O.gather_kv(p1, s1, w1.tail, w1.block_table, 128, 0, 0, 4, 2)
    got = O.decode(w1.q, p1, s1, w1.tail, w1.block_table, w1.seq_lens, 1, 4, 2)[0, 0]
    ref = _brute_attention(w1.q[0, 0], K1, V1, 1 / np.sqrt(128))
    assert np.array_equal(got, ref.astype(np.float16))
    # empty sequence: zeros
    w2, p2, s2 = _small_problem([0, 128], Hq=1, Hkv=1)
    assert np.all(O.decode(w2.q, p2, s2, w2.tail, w2.block_table, w2.seq_lens, 1, 4, 2)[0] == 0)


def test_more_bits_less_attention_error():
    """Reported as in the plan (P8): error against fp16 attention on the
    unquantised cache falls as bits rise."""
    seq = [512, 384]
    errs = {}
    for kb, vb in ((2, 2), (4, 2), (4, 4), (8, 8)):
        w, packed, scales = _small_problem(seq, Hq=4, Hkv=1, seed=21, kb=kb, vb=vb)
        got = O.decode(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, 1, kb, vb).astype(np.float64)
        rows_k = [w.k_full[slice(*w.token_range(b))] for b in range(2)]
        rows_v = [w.v_full[slice(*w.token_range(b))] for b in range(2)]
        ref = O.decode_uncompressed(w.q, rows_k, rows_v, w.seq_lens, 1).astype(np.float64)
        errs[(kb, vb)] = np.abs(got - ref).mean() / np.abs(ref).mean()
    assert errs[(8, 8)] < errs[(4, 4)] < errs[(4, 2)] < errs[(2, 2)]


def test_uncompressed_attention_brute_force():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((20, 1, 128)).astype(np.float16)
    V = rng.standard_normal((20, 1, 128)).astype(np.float16)
    q = rng.standard_normal((1, 1, 128)).astype(np.float16)
    got = O.decode_uncompressed(q, [K], [V], np.array([20]), 1)[0, 0]
    ref = _brute_attention(q[0, 0], K[:, 0].astype(np.float64), V[:, 0].astype(np.float64), 1 / np.sqrt(128))
    assert np.array_equal(got, ref.astype(np.float16))


def test_e4m3_codec_against_definition():
    """OCP E4M3: largest finite 448, smallest subnormal 2^-9, NaN at 0x7F."""
    t = O.e4m3_to_float(np.arange(256, dtype=np.uint8))
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and np.isnan(t[0x7F]) and t[0x38] == 1.0
    vals = t[np.isfinite(t)]
    assert np.array_equal(O.e4m3_to_float(O.float_to_e4m3(vals)), vals + 0.0)
    # ties go to the even code: 1 + 1/16 lies halfway between 1 (0x38) and 1.125 (0x39)
    assert O.float_to_e4m3(np.array([1.0625]))[0] == 0x38
    assert O.float_to_e4m3(np.array([1e6]))[0] == 0x7E


# ---------------------------------------------------------------------------
# decode step with append
# ---------------------------------------------------------------------------

def _append_case(lens, hq, hkv, seed, extra_blocks=4, kb=4, vb=2):
    full = sum(int(L) // 128 for L in lens)
    w = inputs.make_decode_workload("append", lens, hq, hkv, seed, pool_blocks=full + extra_blocks)
    k_new, v_new, bt = inputs.append_step(w, seed + 1)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, hkv, w.num_blocks, kb, vb)
    return w, k_new, v_new, bt, packed, scales


def _rows_after_append(w, k_new, v_new, b):
    """All L + 1 fp16 K / V rows of sequence b ([L+1][Hkv][128]) after the append."""
    s, e = w.token_range(b)
    tl = int(w.seq_lens[b]) % 128
    k = np.concatenate([w.k_full[s:e], w.tail[b, 0, :, :tl].transpose(1, 0, 2), k_new[b][None]])
    v = np.concatenate([w.v_full[s:e], w.tail[b, 1, :, :tl].transpose(1, 0, 2), v_new[b][None]])
    return k, v


def test_append_to_empty_sequence_returns_the_new_value():
    """One token: its softmax weight is exactly 1, so the output is v_new."""
    w, k_new, v_new, bt, packed, scales = _append_case([0, 0, 0], 4, 2, seed=41)
    out, p2, s2, tail2 = O.decode_append(w.q, k_new, v_new, packed, scales, w.tail, bt, w.seq_lens, 2, 4, 2)
    for b in range(3):
        for j in range(4):
            assert np.array_equal(out[b, j], v_new[b, j // 2])
    assert np.array_equal(tail2[:, 0, :, 0], k_new) and np.array_equal(tail2[:, 1, :, 0], v_new)
    assert np.array_equal(p2, packed) and np.array_equal(s2, scales)


def test_append_before_any_full_tile_is_textbook_attention():
    """With no full tile, every token (the one that fills the tile included)
    is attended in fp16: the output is plain softmax attention over the rows."""
    lens = [5, 64, 127, 126]
    w, k_new, v_new, bt, packed, scales = _append_case(lens, 8, 2, seed=43)
    out, *_ = O.decode_append(w.q, k_new, v_new, packed, scales, w.tail, bt, w.seq_lens, 2, 4, 2)
    rows = [_rows_after_append(w, k_new, v_new, b) for b in range(len(lens))]
    ref = O.decode_uncompressed(w.q, [r[0] for r in rows], [r[1] for r in rows], w.seq_lens + 1, 2)
    assert np.array_equal(out, ref)


def test_append_mid_tile_equals_decode_of_the_extended_cache():
    """A token that does not fill its tile is one more tail row: decode of the
    cache with seq_len + 1 over the written tail gives the same output."""
    lens = [300, 129, 256 + 5, 128]
    w, k_new, v_new, bt, packed, scales = _append_case(lens, 8, 2, seed=45)
    out, p2, s2, tail2 = O.decode_append(w.q, k_new, v_new, packed, scales, w.tail, bt, w.seq_lens, 2, 4, 2)
    assert np.array_equal(p2, packed) and np.array_equal(s2, scales)
    ref = O.decode(w.q, packed, scales, tail2, bt, w.seq_lens + 1, 2, 4, 2)
    assert np.array_equal(out, ref)


def test_append_fill_quantises_the_tile_like_the_write_path():
    """A token that fills the tail: the tile (127 tail rows + the token) lands
    in the new block exactly as the quantise-on-write path would put it there,
    only that block changes, and the output still attends the tile in fp16."""
    lens = [127, 128 + 127, 300]
    w, k_new, v_new, bt, packed, scales = _append_case(lens, 4, 2, seed=47, kb=4, vb=2)
    out, p2, s2, tail2 = O.decode_append(w.q, k_new, v_new, packed, scales, w.tail, bt, w.seq_lens, 2, 4, 2)
    changed = set()
    for b, L in enumerate(lens):
        if L % 128 != 127:
            continue
        blk = int(bt[b, L // 128])
        changed.add(blk)
        k, v = _rows_after_append(w, k_new, v_new, b)
        tile_k, tile_v = k[L // 128 * 128:], v[L // 128 * 128:]
        slot = blk * 128 + np.arange(128, dtype=np.int64)
        pw, sw = O.quantize_tiles(tile_k, tile_v, slot, 2, w.num_blocks, 4, 2)
        assert np.array_equal(p2[blk], pw[blk]) and np.array_equal(s2[blk], sw[blk])
    others = [i for i in range(w.num_blocks) if i not in changed]
    assert np.array_equal(p2[others], packed[others]) and np.array_equal(s2[others], scales[others])
    # the filled tile is attended in fp16 this step: the same output as a tail of 128 rows
    b = 0
    k, v = _rows_after_append(w, k_new, v_new, b)
    ref = O.decode_uncompressed(w.q[b:b + 1], [k], [v], np.array([128]), 2)
    assert np.array_equal(out[b], ref[0])


# ---------------------------------------------------------------------------
# multi-query attention
# ---------------------------------------------------------------------------

def test_multiquery_single_query_is_decode():
    w = inputs.make_decode_workload("mq", [300, 129, 0, 128], 8, 2, seed=61, pool_blocks=8)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, 2, w.num_blocks, 4, 2)
    out = O.decode_multiquery(w.q[:, None], packed, scales, w.tail, w.block_table, w.seq_lens, 2, 4, 2)
    ref = O.decode(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, 2, 4, 2)
    assert np.array_equal(out[:, 0], ref)


def test_multiquery_query_i_is_decode_of_the_prefix_it_sees():
    """Query i attends exactly the first L - qlen + i + 1 tokens: where that
    prefix ends in the fp16 tail or at the end of a full tile, it is the plain
    decode of the sequence cut to that length, over the same cache."""
    qlen = 5
    lens = [256 + 4, 128 + 100, 20, 128 + 3, 2 * 128 + 2]
    w = inputs.make_decode_workload("mq", lens, 8, 2, seed=63, pool_blocks=8)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, 2, w.num_blocks, 4, 2)
    q = np.random.default_rng(64).standard_normal((len(lens), qlen, 8, 128)).astype(np.float16)
    out = O.decode_multiquery(q, packed, scales, w.tail, w.block_table, w.seq_lens, 2, 4, 2)
    checked = 0
    for i in range(qlen):
        cut = np.array([L - qlen + i + 1 for L in lens], dtype=np.int32)
        ref = O.decode(q[:, i], packed, scales, w.tail, w.block_table, cut, 2, 4, 2)
        for b, L in enumerate(lens):
            if cut[b] // 128 == L // 128:           # the prefix keeps every full tile
                assert np.array_equal(out[b, i], ref[b])
                checked += 1
    # sequences 3 and 4: the queries before the tail sit in the last full
    # tile; the one at its final token is the decode of exactly the full tiles
    assert checked == 3 * qlen + 4 + 3
    assert np.all(out[:, :, :, :].astype(np.float32).any(axis=-1))


def test_multiquery_inside_a_packed_tile_is_causal():
    """Queries whose position lies inside the last full tile (so that tile
    must be masked per query): changing the stored codes of tokens after a
    query's position, or the fp16 tail, leaves its output unchanged; changing
    the codes of a token it sees changes it."""
    qlen = 6
    L = 3 * 128 + 2                                   # queries at 380..385: 380..383 in tile 2
    w = inputs.make_decode_workload("mqc", [L], 4, 1, seed=65, pool_blocks=4)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, 1, w.num_blocks, 4, 2)
    q = np.random.default_rng(66).standard_normal((1, qlen, 4, 128)).astype(np.float16)
    base = O.decode_multiquery(q, packed, scales, w.tail, w.block_table, w.seq_lens, 1, 4, 2)
    blk = int(w.block_table[0, 2])

    def with_codes(edit):
        """The cache with tile 2's K and V codes ([t][d]) passed through edit."""
        p = packed.copy()
        for side, bits, off in (("K", 4, 0), ("V", 2, O.side_bytes(4))):
            n = O.side_bytes(bits)
            c = O.unpack_codes(p[blk, 0, off:off + n], side, bits)
            p[blk, 0, off:off + n] = O.pack_codes(edit(c, 2 ** bits - 1), side, bits)
        return p

    for i in range(4):                                # query i sits at tile-2 token 124 + i
        t = 124 + i

        def later(c, lb):
            c = c.copy()
            c[t + 1:] = lb - c[t + 1:]
            return c

        def own(c, lb):
            c = c.copy()
            c[t] = lb - c[t]
            return c

        t2 = w.tail.copy()
        t2[0, :, 0, :2] = -t2[0, :, 0, :2]
        got = O.decode_multiquery(q, with_codes(later), scales, t2, w.block_table, w.seq_lens, 1, 4, 2)
        assert np.array_equal(got[0, i], base[0, i]), i
        assert not np.array_equal(got[0, 4:], base[0, 4:])   # the tail queries see both changes
        got3 = O.decode_multiquery(q, with_codes(own), scales, w.tail, w.block_table, w.seq_lens, 1, 4, 2)
        assert not np.array_equal(got3[0, i], base[0, i]), i


def test_append_steps_across_a_tile_fill():
    """Five consecutive steps from 125 to 130 tokens: the tile fills at the
    third step.  While every token is fp16 the output is textbook attention;
    after the fill the step reads the packed tile like decode does."""
    w, _, _, bt, packed, scales = _append_case([125], 4, 2, seed=71, extra_blocks=2)
    rng = np.random.default_rng(72)
    outl = inputs.pick_outlier_channels(np.random.default_rng(73), 2)
    tail, lens = w.tail.copy(), w.seq_lens.copy()
    rows_k = [w.tail[0, 0, :, :125].transpose(1, 0, 2)]
    rows_v = [w.tail[0, 1, :, :125].transpose(1, 0, 2)]
    for step in range(5):
        k_new = inputs.gen_k(rng, 1, 2, outl)
        v_new = inputs.gen_v(rng, 1, 2)
        out, packed, scales, tail = O.decode_append(w.q, k_new, v_new, packed, scales, tail, bt, lens, 2, 4, 2)
        rows_k.append(k_new)
        rows_v.append(v_new)
        L1 = int(lens[0]) + 1
        if L1 <= 128:      # nothing quantised yet: plain fp16 attention
            ref = O.decode_uncompressed(w.q, [np.concatenate(rows_k)], [np.concatenate(rows_v)], np.array([L1]), 2)
        else:              # the first tile is packed now; decode reads the same cache
            ref = O.decode(w.q, packed, scales, tail, bt, np.array([L1], dtype=np.int32), 2, 4, 2)
        assert np.array_equal(out, ref), step
        lens = lens + 1
    assert int(lens[0]) == 130
