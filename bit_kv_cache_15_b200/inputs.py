"""Seeded synthetic inputs for the KVarN quantizer and paged decode attention.

This module only draws random numbers and lays them out in the shapes the
C-ABI takes; it holds none of the method's arithmetic.  The CUDA path, the
CPU oracle, the tests and the benchmark all take their inputs from here.

Distributions (the pages give shapes, not data; these stand in for the
Llama/Qwen GQA workloads and 4K-128K contexts they name):
  * K rows ~ N(0, 1); per KV head, 8 of the 128 channels (chosen by the seed)
    are scaled x10 (outlier channels); each token row of each head is then
    multiplied by exp(N(0, 0.5)) (lognormal per-token scale).
  * V ~ N(0, 1);  q ~ N(0, 1).
  * The paged pool is a seeded random permutation, so block tables are
    shuffled.
All tensors are fp16 (the pages' KV dtype), indices int32 / int64.
"""
from __future__ import annotations

import dataclasses

import numpy as np

TILE = 128
HEAD_DIM = 128


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


def gen_k(rng: np.random.Generator, num_tokens: int, num_kv_heads: int,
          outlier_channels: np.ndarray | None = None) -> np.ndarray:
    """K rows [num_tokens][Hkv][128] fp16 with outlier channels and lognormal token scale."""
    x = rng.standard_normal((num_tokens, num_kv_heads, HEAD_DIM), dtype=np.float32)
    if outlier_channels is None:
        outlier_channels = pick_outlier_channels(rng, num_kv_heads)
    for h in range(num_kv_heads):
        x[:, h, outlier_channels[h]] *= 10.0
    tok = np.exp(0.5 * rng.standard_normal((num_tokens, num_kv_heads), dtype=np.float32))
    x *= tok[:, :, None]
    return x.astype(np.float16)


def gen_v(rng: np.random.Generator, num_tokens: int, num_kv_heads: int) -> np.ndarray:
    return rng.standard_normal((num_tokens, num_kv_heads, HEAD_DIM), dtype=np.float32).astype(np.float16)


def pick_outlier_channels(rng: np.random.Generator, num_kv_heads: int, n: int = 8) -> np.ndarray:
    return np.stack([rng.choice(HEAD_DIM, size=n, replace=False) for _ in range(num_kv_heads)])


@dataclasses.dataclass
class DecodeWorkload:
    """One paged decode problem plus the fp16 K/V that fill its full tiles.

    k_full / v_full: [n_full_tokens][Hkv][128] fp16, the tokens of every full
      128-token tile, sequence by sequence; slot_mapping[i] is the paged slot
      (block * 128 + offset) of token i.
    block_table: [B][max_blocks] int32; seq_lens: [B] int32.
    tail: [B][2][Hkv][128][128] fp16; rows [0, seq_len % 128) of [b][0] (K)
      and [b][1] (V) hold each sequence's partial last tile.
    q: [B][Hq][128] fp16.
    """
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    num_blocks: int
    max_blocks_per_seq: int
    seq_lens: np.ndarray
    block_table: np.ndarray
    slot_mapping: np.ndarray
    k_full: np.ndarray
    v_full: np.ndarray
    tail: np.ndarray
    q: np.ndarray
    seed: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def full_tiles(self, b: int) -> int:
        return int(self.seq_lens[b]) // TILE

    def token_range(self, b: int) -> tuple[int, int]:
        """Range of rows of k_full / v_full that belong to sequence b."""
        start = sum(self.full_tiles(i) for i in range(b)) * TILE
        return start, start + self.full_tiles(b) * TILE


def make_decode_workload(name: str, seq_lens, num_q_heads: int, num_kv_heads: int,
                         seed: int, pool_blocks: int | None = None,
                         max_blocks_per_seq: int | None = None) -> DecodeWorkload:
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = len(seq_lens)
    n_full = seq_lens // TILE
    total_full = int(n_full.sum())
    need = max(total_full, 1)
    num_blocks = int(pool_blocks) if pool_blocks is not None else need
    if num_blocks < total_full:
        raise ValueError("pool smaller than the number of full tiles")
    if max_blocks_per_seq is None:
        max_blocks_per_seq = int(max(1, int(np.max((seq_lens + TILE - 1) // TILE)) if B else 1))
    perm = _rng(seed, 1).permutation(num_blocks).astype(np.int32)
    block_table = np.zeros((B, max_blocks_per_seq), dtype=np.int32)
    slot_mapping = np.zeros(total_full * TILE, dtype=np.int64)
    nxt = 0
    for b in range(B):
        for i in range(int(n_full[b])):
            blk = int(perm[nxt])
            block_table[b, i] = blk
            slot_mapping[nxt * TILE:(nxt + 1) * TILE] = blk * TILE + np.arange(TILE)
            nxt += 1
    rk = _rng(seed, 2)
    outl = pick_outlier_channels(rk, num_kv_heads)
    # generate sequence by sequence to bound host temporaries
    k_parts, v_parts = [], []
    rv = _rng(seed, 3)
    for b in range(B):
        n = int(n_full[b]) * TILE
        k_parts.append(gen_k(rk, n, num_kv_heads, outl))
        v_parts.append(gen_v(rv, n, num_kv_heads))
    k_full = np.concatenate(k_parts) if k_parts else np.zeros((0, num_kv_heads, HEAD_DIM), np.float16)
    v_full = np.concatenate(v_parts) if v_parts else np.zeros((0, num_kv_heads, HEAD_DIM), np.float16)
    tail = np.zeros((B, 2, num_kv_heads, TILE, HEAD_DIM), dtype=np.float16)
    rt = _rng(seed, 4)
    for b in range(B):
        tl = int(seq_lens[b]) % TILE
        if tl:
            kt = gen_k(rt, tl, num_kv_heads, outl)      # [tl][Hkv][128]
            vt = gen_v(rt, tl, num_kv_heads)
            tail[b, 0, :, :tl, :] = kt.transpose(1, 0, 2)
            tail[b, 1, :, :tl, :] = vt.transpose(1, 0, 2)
    q = _rng(seed, 5).standard_normal((B, num_q_heads, HEAD_DIM), dtype=np.float32).astype(np.float16)
    return DecodeWorkload(name, B, num_q_heads, num_kv_heads, num_blocks, max_blocks_per_seq,
                          seq_lens, block_table, slot_mapping, k_full, v_full, tail, q, seed)


def append_step(w: DecodeWorkload, seed: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Inputs of one decode step with append on workload w: (k_new, v_new,
    block_table).  k_new / v_new [B][Hkv][128] fp16 are each sequence's new
    token (same generators and outlier channels as the workload's K and V).
    The block table is w's, plus a free pool block (one no full tile uses,
    in shuffled order) at entry seq_len // 128 of every sequence whose tail
    the token fills (seq_len % 128 == 127)."""
    B, hkv = w.num_seqs, w.num_kv_heads
    outl = pick_outlier_channels(_rng(w.seed, 2), hkv)
    r = _rng(seed, 7)
    k_new = gen_k(r, B, hkv, outl)          # one token per sequence: [B][Hkv][128]
    v_new = gen_v(r, B, hkv)
    bt = w.block_table.copy()
    used = set()
    for b in range(B):
        used.update(int(x) for x in bt[b, :int(w.seq_lens[b]) // TILE])
    free = [int(x) for x in r.permutation(w.num_blocks) if int(x) not in used]
    for b in range(B):
        L = int(w.seq_lens[b])
        if L % TILE == TILE - 1:
            if L // TILE >= bt.shape[1] or not free:
                raise ValueError("no block-table entry or free block for the filled tile")
            bt[b, L // TILE] = free.pop()
    return k_new, v_new, bt


# ---------------------------------------------------------------------------
# The named workloads (sizes as given for the pages' Llama/Qwen shapes)
# ---------------------------------------------------------------------------

def tiny(seed: int = 1001) -> DecodeWorkload:
    """1 KV head, 1 q head, one 128-token tile, no tail."""
    return make_decode_workload("tiny", [128], 1, 1, seed)


def llama3_8b(seed: int = 1002, batch: int = 16, seq: int = 4096) -> DecodeWorkload:
    """32 q / 8 KV heads, batch 16, every sequence 4096 tokens, pool 512 blocks shuffled."""
    pool = max(512, batch * (seq // TILE))
    return make_decode_workload("llama3_8b_b16_4k", [seq] * batch, 32, 8, seed, pool_blocks=pool)


def qwen3_32b(seed: int = 1003, batch: int = 8, ctx: int = 16384) -> DecodeWorkload:
    """64 q / 8 KV heads, batch 8, 16384 tokens + ragged fp16 tail U{0..127}."""
    tails = _rng(seed, 6).integers(0, TILE, size=batch)
    lens = ctx + tails
    pool = max(1024, batch * (ctx // TILE))
    return make_decode_workload("qwen3_32b_b8_16k_tail", lens, 64, 8, seed, pool_blocks=pool)


def llama3_70b(seed: int = 1004, batch: int = 4, lo: int = 1024, hi: int = 131072) -> DecodeWorkload:
    """64 q / 8 KV heads, batch 4, seq lengths uniform in [1024, 131072]."""
    lens = _rng(seed, 6).integers(lo, hi + 1, size=batch)
    return make_decode_workload("llama3_70b_b4_1k_128k", lens, 64, 8, seed)


def prefill_append(seed: int = 1005, batch: int = 8, ctx: int = 16384,
                   append_tokens: int = 32768) -> tuple[DecodeWorkload, np.ndarray]:
    """Batch-8 16K decode (64 q / 8 KV heads, ragged tail) whose last
    append_tokens // batch full-tile tokens per sequence are the prefill-append
    batch.  Returns the workload and the row indices into k_full / v_full of
    the appended tokens (32768 tokens x 8 KV heads = 4096 K+V tiles)."""
    tails = _rng(seed, 6).integers(0, TILE, size=batch)
    w = make_decode_workload("prefill_append_32k_b8_16k", ctx + tails, 64, 8, seed,
                             pool_blocks=batch * (ctx // TILE))
    per_seq = append_tokens // batch
    rows = []
    for b in range(batch):
        s, e = w.token_range(b)
        rows.append(np.arange(e - per_seq, e))
    return w, np.concatenate(rows)


def quantize_batch(seed: int, num_tokens: int, num_kv_heads: int,
                   num_blocks: int | None = None) -> dict:
    """A plain quantize problem: k, v [num_tokens][Hkv][128] fp16 written to a
    shuffled set of num_tokens / 128 blocks out of num_blocks."""
    assert num_tokens % TILE == 0
    groups = num_tokens // TILE
    nb = num_blocks if num_blocks is not None else groups
    perm = _rng(seed, 1).permutation(nb)[:groups]
    slot = (perm[:, None] * TILE + np.arange(TILE)[None, :]).reshape(-1).astype(np.int64)
    rk = _rng(seed, 2)
    k = gen_k(rk, num_tokens, num_kv_heads)
    v = gen_v(_rng(seed, 3), num_tokens, num_kv_heads)
    return dict(k=k, v=v, slot_mapping=slot, num_blocks=nb, num_kv_heads=num_kv_heads)


WORKLOADS = {
    "tiny": tiny,
    "llama3_8b": llama3_8b,
    "qwen3_32b": qwen3_32b,
    "llama3_70b": llama3_70b,
}
