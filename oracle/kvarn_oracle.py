"""KVarN CPU oracle: a plain, slow, fp64 restatement of the method.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this module.  It shares no code
with the CUDA library (no kernels, headers, tables or helpers) and the
library never calls it.

Sources (cited as [page, section]):
  [hypho]  "KV-cache 量化终于能跑生产了？KVarN 用方差归一化打破 vLLM 的吞吐量魔咒"
           (blog.hypho.cn), sections "它怎么做到的：四步流水线" (four-step
           pipeline), "工程实践：一行配置启用" (usage), "需要关注的几个问题"
           (block size 128 only).
  [lehuy]  "KVarN: Backend lượng tử hóa KV-cache gốc của Huawei giúp vLLM tăng
           hiệu suất vượt trội" (lehuy.net), sections "Cơ chế hoạt động: Chuẩn
           hóa phương sai" (4 stages per fixed token tile, scales folded on
           read) and "Dễ dàng tích hợp và sử dụng" (block_size = tile size).

What the pages fix:  a tile of 128 tokens x head_dim channels [lehuy, Cơ chế
hoạt động; hypho, 需要关注的几个问题 item 3]; (1) the raw fp16 tile, (2) a
Hadamard rotation along the channel dimension, orthogonal, leaving attention
scores unchanged [hypho, 四步流水线 step 2; lehuy, stage 2], (3) variance
normalisation by alternating row / column std normalisation in log space,
Sinkhorn-like [hypho, step 3; lehuy, stage 3], (4) asymmetric low-bit
round-to-nearest with the scales restored when read, keys 4 bit and values
2 bit by default, "kvarn_k4v2_g128" [hypho, step 4; lehuy, stage 4].

Readings where the pages are silent (the kernels follow the same ones):
  * H is the unnormalised Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i&j),
    applied on the right of each token row: R = X H.  H H^T = 128 I, so the
    inverse is H / 128.
  * "std" is the root-mean-square about zero; rows of the (channels x tokens)
    tile are channels, so each of the N (default 8) iterations normalises
    channels first, then tokens.  Mean squares are floored at 2^-48.
  * log-scales are base 2 and stored as fp16 (round to nearest even).
  * one asymmetric (zero, step) pair per tile and per K / V, from the min and
    max of the normalised tile, stored as fp32.  Z is formed in fp64 from the
    stored fp16 log-scales, and codes are round-half-even of (Z - zero) / step
    in fp64 from the stored fp32 zero and step, clamped to [0, 2^b - 1].
  * decode: softmax scale 1/sqrt(128), q head j reads KV head j // (Hq / Hkv);
    the partial last tile of each sequence (seq_len % 128 tokens) is attended
    in fp16 from a separate tail buffer; the output is fp16 (round to nearest).
The packed byte layout is this project's own (the pages give none); it is
written out in `code_position` from its definition and nothing else.
"""
from __future__ import annotations

import functools

import numpy as np

TILE = 128
HEAD_DIM = 128
LOG_FLOOR = 2.0 ** -48
SCALE_BLOCK_BYTES = 528            # per (block, head) and per K or V
SCALE_DTYPE = np.dtype([("lt", "<f2", (TILE,)), ("lc", "<f2", (HEAD_DIM,)),
                        ("zero", "<f4"), ("step", "<f4"), ("pad", "u1", (8,))])
assert SCALE_DTYPE.itemsize == SCALE_BLOCK_BYTES


# ---------------------------------------------------------------------------
# configuration string  [hypho, 工程实践：一行配置启用; lehuy, Dễ dàng tích hợp]
# ---------------------------------------------------------------------------

def parse_config(s: str) -> tuple[int, int, int]:
    """"kvarn_k{kb}v{vb}_g{group}" -> (kb, vb, group)."""
    if not s.startswith("kvarn_k"):
        raise ValueError(s)
    body = s[len("kvarn_k"):]
    kpart, rest = body.split("v", 1)
    vpart, g = rest.split("_g", 1)
    return int(kpart), int(vpart), int(g)


# ---------------------------------------------------------------------------
# step 2: Hadamard rotation along channels  [hypho, 四步流水线 step 2]
# ---------------------------------------------------------------------------

def hadamard(n: int = HEAD_DIM) -> np.ndarray:
    """Sylvester Hadamard matrix with entries (-1)^popcount(i & j), int64."""
    i = np.arange(n, dtype=np.int64)
    parity = (np.bitwise_count(i[:, None] & i[None, :]) & 1).astype(np.int64)
    return 1 - 2 * parity


def rotate(x16: np.ndarray) -> np.ndarray:
    """R = X H for a [..., 128] fp16 array, in fp64.

    Every partial sum is an integer multiple of 2^-24 below 2^23 in
    magnitude, so fp64 holds it exactly: R is the exact product."""
    return x16.astype(np.float64) @ hadamard().astype(np.float64)


# ---------------------------------------------------------------------------
# step 3: log-space alternating std normalisation  [hypho, step 3; lehuy, stage 3]
# ---------------------------------------------------------------------------

def normalize_logscales(R: np.ndarray, iters: int) -> tuple[np.ndarray, np.ndarray]:
    """Return (lt[128] tokens, lc[128] channels), fp64 log2 scales.

    Each iteration: channel pass, then token pass, each setting the RMS of
    R * 2^-(lt[t] + lc[d]) along that axis to 1.
    """
    A = R * R                                   # [t][d]
    lt = np.zeros(R.shape[0])
    lc = np.zeros(R.shape[1])
    for _ in range(iters):
        ms_c = (A * np.exp2(-2.0 * lt)[:, None]).mean(axis=0)
        lc = 0.5 * np.log2(np.maximum(ms_c, LOG_FLOOR))
        ms_t = (A * np.exp2(-2.0 * lc)[None, :]).mean(axis=1)
        lt = 0.5 * np.log2(np.maximum(ms_t, LOG_FLOOR))
    return lt, lc


# ---------------------------------------------------------------------------
# step 4: asymmetric round-to-nearest  [hypho, step 4; lehuy, stage 4]
# ---------------------------------------------------------------------------

def quantize_given_scales(R: np.ndarray, Lt16: np.ndarray, Lc16: np.ndarray, bits: int,
                          zero: np.float32 | None = None, step: np.float32 | None = None):
    """Codes of a rotated tile given its stored fp16 log-scales, in fp64.

    Z = R * 2^-(Lt + Lc) with the stored fp16 log-scales; zero = fp32(min Z);
    step = fp32((max Z - zero) / (2^b - 1)), taken from that stored zero (1 if
    it is 0); code = clamp(rne((Z - zero) / step), 0, 2^b - 1), the division
    and the rounding in fp64 from the stored fp32 zero and step.
    zero / step may be given (to re-derive codes from stored values).
    Returns (codes int32 [128][128], zero f32, step f32, y f64 [128][128])
    where y = (Z - zero) / step before rounding.
    """
    Lb = 2 ** bits - 1
    R = np.asarray(R, dtype=np.float64)
    Z = R * np.exp2(-(Lt16.astype(np.float64)[:, None] + Lc16.astype(np.float64)[None, :]))
    if zero is None:
        zero = np.float32(Z.min())
        step = np.float32((Z.max() - np.float64(zero)) / Lb)
        if step == 0:
            step = np.float32(1.0)
    zero = np.float32(zero)
    step = np.float32(step)
    y = (Z - np.float64(zero)) / np.float64(step)
    codes = np.clip(np.rint(y), 0, Lb).astype(np.int32)
    return codes, zero, step, y


def quantize_tile(x16: np.ndarray, bits: int, iters: int = 8) -> dict:
    """Steps 1-4 for one 128-token x 128-channel fp16 tile ([t][d])."""
    assert x16.shape == (TILE, HEAD_DIM) and x16.dtype == np.float16
    R = rotate(x16)
    lt, lc = normalize_logscales(R, iters)
    Lt16 = lt.astype(np.float16)
    Lc16 = lc.astype(np.float16)
    codes, zero, step, y = quantize_given_scales(R, Lt16, Lc16, bits)
    return dict(R=R, lt=lt, lc=lc, Lt=Lt16, Lc=Lc16, codes=codes, zero=zero, step=step, y=y)


def dequantize_rotated(codes, Lt16, Lc16, zero, step) -> np.ndarray:
    """The stored tile restored in the rotated domain, fp64:
    2^(Lt[t] + Lc[d]) * (zero + step * code)."""
    s = np.exp2(Lt16.astype(np.float64)[:, None] + Lc16.astype(np.float64)[None, :])
    return s * (np.float64(zero) + np.float64(step) * codes.astype(np.float64))


def dequantize(codes, Lt16, Lc16, zero, step) -> np.ndarray:
    """Explicit dequantisation back to the original domain: (...) H / 128."""
    return dequantize_rotated(codes, Lt16, Lc16, zero, step) @ hadamard().astype(np.float64) / 128.0


# ---------------------------------------------------------------------------
# packed layout (this project's own definition, written out in code_position)
# ---------------------------------------------------------------------------

def code_position(side: str, bits: int, t, d):
    """Byte offset and bit offset, inside one side's code block, of the code
    of token t, channel d.  Works elementwise on integer arrays.

    blk  = (t // 16) * 8 + d // 16
    (row, col) = (t % 16, d % 16) for K,  (d % 16, t % 16) for V
    lane = (row % 8) * 4 + (col % 8) // 2
    j    = row // 8 + 2 * (col // 8);  h = col % 2
    rho  = 4 * blk + j;  per = 16 // bits;  word = rho // per;  slot = rho % per
    bit  = bits * slot + 16 * h  (inside the little-endian 32-bit word)
    word address = ((word // 4) * 32 + lane) * 4 + word % 4
    """
    t = np.asarray(t, dtype=np.int64)
    d = np.asarray(d, dtype=np.int64)
    blk = (t // 16) * 8 + d // 16
    if side == "K":
        row, col = t % 16, d % 16
    elif side == "V":
        row, col = d % 16, t % 16
    else:
        raise ValueError(side)
    lane = (row % 8) * 4 + (col % 8) // 2
    j = row // 8 + 2 * (col // 8)
    h = col % 2
    rho = 4 * blk + j
    per = 16 // bits
    word = rho // per
    slot = rho % per
    bit = bits * slot + 16 * h
    waddr = ((word // 4) * 32 + lane) * 4 + word % 4
    return waddr * 4 + bit // 8, bit % 8


def side_bytes(bits: int) -> int:
    return TILE * HEAD_DIM * bits // 8


@functools.lru_cache(maxsize=None)
def _tile_positions(side: str, bits: int):
    """code_position of every (t, d) of one tile, computed once per layout."""
    t, d = np.meshgrid(np.arange(TILE), np.arange(HEAD_DIM), indexing="ij")
    byte, bit0 = code_position(side, bits, t, d)
    byte.setflags(write=False)
    bit0.setflags(write=False)
    return byte, bit0


def pack_codes(codes: np.ndarray, side: str, bits: int) -> np.ndarray:
    byte, bit0 = _tile_positions(side, bits)
    out = np.zeros(side_bytes(bits), dtype=np.uint8)
    c = codes.astype(np.int64)
    for b in range(bits):
        # a code never straddles a byte: bits divides 8
        np.bitwise_or.at(out, byte.ravel(), (((c >> b) & 1) << (bit0 + b)).ravel().astype(np.uint8))
    return out


def unpack_codes(buf: np.ndarray, side: str, bits: int) -> np.ndarray:
    byte, bit0 = _tile_positions(side, bits)
    return ((buf[byte].astype(np.int64) >> bit0) & ((1 << bits) - 1)).astype(np.int32)


def pack_scales(Lt16, Lc16, zero, step) -> np.ndarray:
    rec = np.zeros(1, dtype=SCALE_DTYPE)
    rec["lt"][0] = Lt16
    rec["lc"][0] = Lc16
    rec["zero"][0] = zero
    rec["step"][0] = step
    return rec.view(np.uint8)


def unpack_scales(buf: np.ndarray):
    rec = np.frombuffer(np.ascontiguousarray(buf).tobytes(), dtype=SCALE_DTYPE)[0]
    return (rec["lt"].copy(), rec["lc"].copy(), np.float32(rec["zero"]), np.float32(rec["step"]))


def code_block_bytes(kb: int, vb: int) -> int:
    """Bytes of codes per (block, KV head): K codes then V codes."""
    return side_bytes(kb) + side_bytes(vb)


# ---------------------------------------------------------------------------
# whole-cache quantisation: the paged write path
# ---------------------------------------------------------------------------

def quantize_tiles(k, v, slot_mapping, num_kv_heads: int, num_blocks: int,
                   kb: int, vb: int, iters: int = 8, packed=None, scales=None,
                   groups=None):
    """Quantise every 128-token group of k, v ([n][Hkv][128] fp16) into the
    paged cache.  Group g goes to block slot_mapping[128 g] // 128.

    packed: uint8 [num_blocks][Hkv][code_block_bytes]; scales: uint8
    [num_blocks][Hkv][2][528]; both created (zeroed) when None.  `groups`
    restricts the work to a subset of token groups.
    """
    n = k.shape[0]
    assert n % TILE == 0
    cb = code_block_bytes(kb, vb)
    if packed is None:
        packed = np.zeros((num_blocks, num_kv_heads, cb), dtype=np.uint8)
    if scales is None:
        scales = np.zeros((num_blocks, num_kv_heads, 2, SCALE_BLOCK_BYTES), dtype=np.uint8)
    if groups is None:
        groups = range(n // TILE)
    for g in groups:
        blk = int(slot_mapping[g * TILE]) // TILE
        for h in range(num_kv_heads):
            for side, src, bits, off in (("K", k, kb, 0), ("V", v, vb, side_bytes(kb))):
                r = quantize_tile(np.ascontiguousarray(src[g * TILE:(g + 1) * TILE, h, :]), bits, iters)
                packed[blk, h, off:off + side_bytes(bits)] = pack_codes(r["codes"], side, bits)
                scales[blk, h, 0 if side == "K" else 1] = pack_scales(r["Lt"], r["Lc"], r["zero"], r["step"])
    return packed, scales


def read_tile(packed, scales, blk: int, h: int, side: str, kb: int, vb: int):
    """(codes, Lt, Lc, zero, step) of one stored tile."""
    if side == "K":
        buf = packed[blk, h, :side_bytes(kb)]
        codes = unpack_codes(buf, "K", kb)
        Lt, Lc, z, s = unpack_scales(scales[blk, h, 0])
    else:
        buf = packed[blk, h, side_bytes(kb):side_bytes(kb) + side_bytes(vb)]
        codes = unpack_codes(buf, "V", vb)
        Lt, Lc, z, s = unpack_scales(scales[blk, h, 1])
    return codes, Lt, Lc, z, s


# ---------------------------------------------------------------------------
# decode attention over the packed cache  [lehuy, stage 4: scales folded on read]
# ---------------------------------------------------------------------------

def gather_kv(packed, scales, tail, block_table, seq_len: int, b: int, h: int, kb: int, vb: int,
              cache=None, tail_len=None):
    """Explicitly dequantised K, V ([seq_len][128] fp64) of sequence b, head h.

    The last `tail_len` tokens (default seq_len % 128) come from the fp16
    tail, the ones before from the packed cache."""
    tl = seq_len % TILE if tail_len is None else int(tail_len)
    assert 0 <= tl <= TILE and (seq_len - tl) % TILE == 0
    n_full = (seq_len - tl) // TILE
    ks, vs = [], []
    for i in range(n_full):
        blk = int(block_table[b][i])
        key = (blk, h)
        if cache is not None and key in cache:
            kd, vd = cache[key]
        else:
            kd = dequantize(*read_tile(packed, scales, blk, h, "K", kb, vb))
            vd = dequantize(*read_tile(packed, scales, blk, h, "V", kb, vb))
            if cache is not None:
                cache[key] = (kd, vd)
        ks.append(kd)
        vs.append(vd)
    if tl:
        ks.append(tail[b, 0, h, :tl, :].astype(np.float64))
        vs.append(tail[b, 1, h, :tl, :].astype(np.float64))
    if not ks:
        return np.zeros((0, HEAD_DIM)), np.zeros((0, HEAD_DIM))
    return np.concatenate(ks), np.concatenate(vs)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, sm_scale: float) -> np.ndarray:
    """Textbook softmax attention of one query over K, V rows, fp64."""
    if K.shape[0] == 0:
        return np.zeros(HEAD_DIM)
    s = sm_scale * (K @ q.astype(np.float64))
    p = np.exp(s - s.max())
    return (p @ V) / p.sum()


def decode(q, packed, scales, tail, block_table, seq_lens, num_kv_heads: int, kb: int, vb: int,
           sm_scale: float | None = None, heads=None) -> np.ndarray:
    """Decode attention on the explicitly dequantised cache.

    q: [B][Hq][128] fp16.  Returns out [B][Hq][128] fp16 (RNE of the fp64
    result).  `heads`: optional iterable of (b, j) pairs to compute; the
    other outputs are left 0.
    """
    B, Hq, _ = q.shape
    G = Hq // num_kv_heads
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    out = np.zeros((B, Hq, HEAD_DIM), dtype=np.float16)
    pairs = heads if heads is not None else [(b, j) for b in range(B) for j in range(Hq)]
    cache = {}
    for b, j in pairs:
        h = j // G
        K, V = gather_kv(packed, scales, tail, block_table, int(seq_lens[b]), b, h, kb, vb, cache)
        out[b, j] = attention(q[b, j], K, V, sm_scale).astype(np.float16)
    return out


def decode_append(q, k_new, v_new, packed, scales, tail, block_table, seq_lens, num_kv_heads: int,
                  kb: int, vb: int, iters: int = 8, sm_scale: float | None = None, heads=None):
    """One decode step that first appends each sequence's new token.

    Reading (the pages fix only that whole 128-token tiles are quantised
    [lehuy, Cơ chế hoạt động; hypho, 需要关注的几个问题 item 3]): the newest
    seq_len % 128 tokens wait unquantised in the fp16 tail; the step's token
    (k_new / v_new [B][Hkv][128] fp16) becomes tail row L % 128, where L =
    seq_lens[b] is the length before the step; the output attends all L + 1
    tokens, the tail rows [0, L % 128] in fp16; a tail that the token fills
    is attended in fp16 this step and quantised (quantize_tile, as on write)
    into block block_table[b][L // 128] for the steps after.

    Returns (out, packed, scales, tail), the last three as new arrays.
    """
    B, Hq, _ = q.shape
    G = Hq // num_kv_heads
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    tail2, packed2, scales2 = tail.copy(), packed.copy(), scales.copy()
    for b in range(B):
        L = int(seq_lens[b])
        r = L % TILE
        tail2[b, 0, :, r, :] = k_new[b]
        tail2[b, 1, :, r, :] = v_new[b]
        if r == TILE - 1:
            blk = int(block_table[b][L // TILE])
            for h in range(num_kv_heads):
                for sidx, side, bits, off in ((0, "K", kb, 0), (1, "V", vb, side_bytes(kb))):
                    t = quantize_tile(np.ascontiguousarray(tail2[b, sidx, h]), bits, iters)
                    packed2[blk, h, off:off + side_bytes(bits)] = pack_codes(t["codes"], side, bits)
                    scales2[blk, h, sidx] = pack_scales(t["Lt"], t["Lc"], t["zero"], t["step"])
    out = np.zeros((B, Hq, HEAD_DIM), dtype=np.float16)
    pairs = heads if heads is not None else [(b, j) for b in range(B) for j in range(Hq)]
    cache = {}
    for b, j in pairs:
        h = j // G
        L = int(seq_lens[b])
        K, V = gather_kv(packed, scales, tail2, block_table, L + 1, b, h, kb, vb, cache, tail_len=L % TILE + 1)
        out[b, j] = attention(q[b, j], K, V, sm_scale).astype(np.float16)
    return out, packed2, scales2, tail2


def decode_multiquery(q, packed, scales, tail, block_table, seq_lens, num_kv_heads: int, kb: int, vb: int,
                      sm_scale: float | None = None, heads=None) -> np.ndarray:
    """Multi-query attention over the cache, causal.

    Reading (the pages quote time-to-first-token but fix no multi-query
    kernel): q is [B][qlen][Hq][128] fp16; query i of sequence b sits at
    position L - qlen + i (L = seq_lens[b], counting the queries' own tokens)
    and attends keys [0, L - qlen + i], each read as decode reads it: keys of
    full tiles dequantised from the packed cache (also when the query sits
    inside that tile), the last L % 128 from the fp16 tail.  Defined when
    L >= qlen; other sequences, and empty ones, give 0.
    `heads`: optional (b, i, j) triples to compute.  Returns [B][qlen][Hq][128] fp16.
    """
    B, qlen, Hq, _ = q.shape
    G = Hq // num_kv_heads
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    out = np.zeros((B, qlen, Hq, HEAD_DIM), dtype=np.float16)
    trip = heads if heads is not None else [(b, i, j) for b in range(B) for i in range(qlen) for j in range(Hq)]
    cache = {}
    for b, i, j in trip:
        L = int(seq_lens[b])
        if L < qlen or L == 0:
            continue
        K, V = gather_kv(packed, scales, tail, block_table, L, b, j // G, kb, vb, cache)
        lim = L - qlen + i + 1
        out[b, i, j] = attention(q[b, i, j], K[:lim], V[:lim], sm_scale).astype(np.float16)
    return out


def decode_folded(q, packed, scales, tail, block_table, seq_lens, num_kv_heads: int, kb: int, vb: int,
                  sm_scale: float | None = None, heads=None) -> np.ndarray:
    """The same attention with every scale folded in on read, fp64 (returns
    the unrounded fp64 output).  Key side: q is rotated by H and multiplied by
    the channel scales, token scales multiply the scores; value side: token
    scales multiply the softmax weights, channel scales and the inverse
    Hadamard apply to the output.  Used only to check the folding algebra."""
    B, Hq, _ = q.shape
    G = Hq // num_kv_heads
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    H = hadamard().astype(np.float64)
    out = np.zeros((B, Hq, HEAD_DIM))
    pairs = heads if heads is not None else [(b, j) for b in range(B) for j in range(Hq)]
    for b, j in pairs:
        h = j // G
        L = int(seq_lens[b])
        n_full, tl = L // TILE, L % TILE
        qf = q[b, j].astype(np.float64)
        q_rot = qf @ H
        scores, vparts = [], []
        for i in range(n_full):
            blk = int(block_table[b][i])
            ck, Ltk, Lck, zk, sk = read_tile(packed, scales, blk, h, "K", kb, vb)
            qp = q_rot * np.exp2(Lck.astype(np.float64))
            dots = ck.astype(np.float64) @ qp
            s = (sm_scale / 128.0) * np.exp2(Ltk.astype(np.float64)) * (float(zk) * qp.sum() + float(sk) * dots)
            scores.append(s)
            vparts.append(("tile", blk))
        if tl:
            kt = tail[b, 0, h, :tl, :].astype(np.float64)
            scores.append(sm_scale * (kt @ qf))
            vparts.append(("tail", None))
        if not scores:
            continue
        m = max(s.max() for s in scores)
        l = sum(np.exp(s - m).sum() for s in scores)
        acc_rot = np.zeros(HEAD_DIM)
        acc_tail = np.zeros(HEAD_DIM)
        for s, (kind, blk) in zip(scores, vparts):
            p = np.exp(s - m)
            if kind == "tile":
                cv, Ltv, Lcv, zv, sv = read_tile(packed, scales, blk, h, "V", kb, vb)
                pp = p * np.exp2(Ltv.astype(np.float64))
                acc_rot += np.exp2(Lcv.astype(np.float64)) * (float(zv) * pp.sum() + float(sv) * (pp @ cv.astype(np.float64)))
            else:
                acc_tail += p @ tail[b, 1, h, :tl, :].astype(np.float64)
        out[b, j] = (acc_rot @ H / 128.0 + acc_tail) / l
    return out


# ---------------------------------------------------------------------------
# uncompressed references (quality figure and the fp16 / fp8 baselines)
# ---------------------------------------------------------------------------

def decode_uncompressed(q, k_rows, v_rows, seq_lens, num_kv_heads: int, sm_scale=None, heads=None):
    """Attention over per-sequence fp16 K/V rows: k_rows[b] is [seq_len][Hkv][128]."""
    B, Hq, _ = q.shape
    G = Hq // num_kv_heads
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(HEAD_DIM)
    out = np.zeros((B, Hq, HEAD_DIM), dtype=np.float16)
    pairs = heads if heads is not None else [(b, j) for b in range(B) for j in range(Hq)]
    for b, j in pairs:
        h = j // G
        K = k_rows[b][:, h, :].astype(np.float64)
        V = v_rows[b][:, h, :].astype(np.float64)
        out[b, j] = attention(q[b, j], K, V, sm_scale).astype(np.float16)
    return out


def e4m3_to_float(u8: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 (bias 7, no infinities, 0x7F/0xFF NaN) to fp64."""
    u = u8.astype(np.int64)
    s = np.where(u & 0x80, -1.0, 1.0)
    e = (u >> 3) & 0xF
    m = u & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


def float_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round fp64 to the nearest E4M3 value (ties to even), saturating at 448."""
    table = e4m3_to_float(np.arange(256, dtype=np.uint8))
    finite = np.where(np.isnan(table), np.inf, table)
    pos = np.arange(0, 127, dtype=np.uint8)          # codes 0x00..0x7E, increasing values
    pv = finite[pos]
    ax = np.minimum(np.abs(np.asarray(x, dtype=np.float64)), 448.0)
    idx = np.searchsorted(pv, ax)                     # pv[idx-1] < ax <= pv[idx]
    idx = np.clip(idx, 1, len(pv) - 1)
    lo, hi = pv[idx - 1], pv[idx]
    pick_hi = (ax - lo > hi - ax) | ((ax - lo == hi - ax) & ((pos[idx] & 1) == 0))
    code = np.where(pick_hi, pos[idx], pos[idx - 1])
    code = np.where(ax <= 0.0, 0, code).astype(np.uint8)
    neg = np.asarray(x) < 0
    return np.where(neg & (code != 0), code | 0x80, code).astype(np.uint8)


def capacity_bytes_per_token_head(kb: int, vb: int) -> float:
    """Stored bytes per token per KV head: codes plus both scale blocks."""
    return (code_block_bytes(kb, vb) + 2 * SCALE_BLOCK_BYTES) / TILE
