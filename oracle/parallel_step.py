"""One whole benchmark step of the CPU oracle, spread over the host's cores.

TEST INFRASTRUCTURE ONLY, like kvarn_oracle: only the benchmark's CPU
baseline and its reference arm run this.  It adds no arithmetic of its own:
every tile is quantised by kvarn_oracle.quantize_tile / pack_codes and every
(sequence, KV head) decode is kvarn_oracle.decode, unchanged.

The work is split over a pool of worker processes, one numpy / BLAS thread
each.  The pool is forked when the step is built, which must happen before
the calling process first touches a GPU (a process forked after that can
hang); the workers inherit the step's inputs and never touch a GPU.
  * quantise: every K and V tile of the appended token groups (one task per
    chunk of tiles; the packed bytes come back to the parent, which writes
    them into its cache);
  * decode: then every (sequence, KV head) pair decodes its query heads over
    that cache (one task per pair, given the pair's blocks of the cache).
"""
from __future__ import annotations

import multiprocessing as mp
import os
import time

import numpy as np

_STEP = {}         # inputs of the step, set before the pool is forked
_LIMITS = None     # keeps a worker's BLAS thread limit alive


def _init():
    global _LIMITS
    try:
        from threadpoolctl import threadpool_limits
        _LIMITS = threadpool_limits(1)
    except Exception:
        pass


def _quantize_chunk(args):
    """Quantise tiles (row group, head, side) of k / v; returns their bytes."""
    from oracle import kvarn_oracle as O
    tiles, src_name, kb, vb, iters = args
    k, v = _STEP[src_name]
    res = []
    for g, h, side in tiles:
        bits = kb if side == 0 else vb
        x = np.ascontiguousarray((k if side == 0 else v)[g * 128:(g + 1) * 128, h])
        r = O.quantize_tile(x, bits, iters)
        res.append((g, h, side, O.pack_codes(r["codes"], "K" if side == 0 else "V", bits),
                    O.pack_scales(r["Lt"], r["Lc"], r["zero"], r["step"])))
    return res


def _decode_pair(args):
    """Decode every query head of (sequence b, KV head h); packed / scales
    hold only the pair's blocks, in block-table order."""
    from oracle import kvarn_oracle as O
    b, h, packed, scales, kb, vb = args
    q, tail, seq_lens = _STEP["q"], _STEP["tail"], _STEP["seq_lens"]
    hkv = tail.shape[2]
    G = q.shape[1] // hkv
    bt = np.arange(packed.shape[0], dtype=np.int32)[None, :]
    out = O.decode(q[b:b + 1, h * G:(h + 1) * G], packed, scales, tail[b:b + 1, :, h:h + 1], bt,
                   seq_lens[b:b + 1], 1, kb, vb)
    return b, h, out[0]


class OracleStep:
    """The benchmark step -- quantise the appended token groups into the paged
    cache, then decode every sequence -- run by the oracle over `workers`
    forked processes.  Build it before the process first uses a GPU."""

    def __init__(self, w, rows, kb: int = 4, vb: int = 2, iters: int = 8, workers: int | None = None):
        from oracle import kvarn_oracle as O
        self.workers = int(workers or len(os.sched_getaffinity(0)) or 1)
        self.kb, self.vb, self.iters = kb, vb, iters
        self.w = w
        self.hkv = w.num_kv_heads
        self.rows = np.asarray(rows)
        self.app_groups = len(rows) // 128
        self.app_blocks = [int(x) // 128 for x in w.slot_mapping[self.rows[::128]]]
        self.packed = np.zeros((w.num_blocks, self.hkv, O.code_block_bytes(kb, vb)), np.uint8)
        self.scales = np.zeros((w.num_blocks, self.hkv, 2, O.SCALE_BLOCK_BYTES), np.uint8)
        _STEP.clear()
        _STEP.update(full=(w.k_full, w.v_full), app=(w.k_full[self.rows], w.v_full[self.rows]),
                     q=w.q, tail=w.tail, seq_lens=w.seq_lens)
        self.pool = mp.get_context("fork").Pool(self.workers, initializer=_init)

    def _quantize(self, src_name, groups, blocks):
        tiles = [(g, h, s) for s in (0, 1) for g in groups for h in range(self.hkv)]
        n_chunks = min(len(tiles), 4 * self.workers)
        chunks = [tiles[i::n_chunks] for i in range(n_chunks)]
        off_v = 2048 * self.kb
        for res in self.pool.imap_unordered(_quantize_chunk, [(c, src_name, self.kb, self.vb, self.iters)
                                                              for c in chunks]):
            for g, h, side, codes, rec in res:
                blk = blocks[g]
                off = 0 if side == 0 else off_v
                self.packed[blk, h, off:off + codes.size] = codes
                self.scales[blk, h, side] = rec

    def prefill(self):
        """Quantise the rest of each sequence's cache (untimed set-up, as the
        GPU benchmark's one-time prefill)."""
        w = self.w
        n_groups = w.k_full.shape[0] // 128
        appended = set(int(r) // 128 for r in self.rows[::128])
        groups = [g for g in range(n_groups) if g not in appended]
        blocks = {g: int(w.slot_mapping[g * 128]) // 128 for g in groups}
        self._quantize("full", groups, blocks)

    def step(self) -> np.ndarray:
        """One whole step; returns the decode output [B][Hq][128] fp16."""
        self._quantize("app", range(self.app_groups), dict(enumerate(self.app_blocks)))
        w = self.w
        G = w.num_q_heads // self.hkv
        out = np.zeros((w.num_seqs, w.num_q_heads, 128), np.float16)
        tasks = []
        for b in range(w.num_seqs):
            blks = w.block_table[b, :int(w.seq_lens[b]) // 128]
            for h in range(self.hkv):
                tasks.append((b, h, self.packed[blks, h:h + 1], self.scales[blks, h:h + 1], self.kb, self.vb))
        for b, h, o in self.pool.imap_unordered(_decode_pair, tasks):
            out[b, h * G:(h + 1) * G] = o
        return out

    def timed_steps(self, n: int) -> list[float]:
        ts = []
        for _ in range(n):
            t0 = time.perf_counter()
            self.step()
            ts.append(time.perf_counter() - t0)
        return ts

    def close(self):
        self.pool.close()
        self.pool.join()
