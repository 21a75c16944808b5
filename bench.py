"""Benchmark of the KVarN hot path on B200: one JSON line on rank 0.

A step is one pass of the whole path over one batch of the prefill-append
workload (the one that names both halves): quantise-on-write of a 32768-token
x 8-KV-head append batch (4096 K+V tiles, k4v2, 8 normalisation passes) into
the paged cache, then one k4v2 decode-attention step for batch 8 at 16384
context plus a ragged fp16 tail (Hq = 64, Hkv = 8, head_dim 128).  The rest of
each sequence's 16K cache is quantised once before timing.

  value  decode tokens/s of the whole step (B tokens per step, quantise
         included), summed over ranks;
  e2e    the same through the C-ABI with the step's inputs copied from pinned
         host memory and the output read back inside the timed region.
Per-kernel CUDA-event times give the quantise tiles/s, the decode-only
tokens/s and each kernel's HBM GB/s from algorithmic bytes.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
--impl reference times the CPU oracle (the fp64 restatement in oracle/) on
whole steps of the same workload, spread over all of the host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "k4v2 decode attn tokens/s & HBM GB/s vs ~8 TB/s peak; quantize tiles/s"
WORKLOAD = ("prefill-append + decode: quantize 32768 new tokens x 8 KV heads (4096 K+V tiles) into the paged "
            "cache, then batch-8 decode at 16384 + ragged fp16 tail U{0..127}, Hq=64, Hkv=8, head_dim=128, "
            "kvarn_k4v2_g128, 8 Sinkhorn iters")
BATCH = 8
HQ, HKV = 64, 8
# FP32 work per 128x128 tile that the method itself needs (flops; an FMA counts 2):
# 8 normalisation iterations x 2 passes x 16384 FMA, R*R, a 7-stage Hadamard
# butterfly (7 x 16384 adds) and about 4 ops per element to form Z and the code.
QUANT_FLOPS_PER_TILE = 2 * 8 * 16384 * 2 + 16384 + 7 * 16384 + 4 * 16384
ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks (NVML, sampled in a thread)

class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        names = {0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, n in names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def start_region(self, timeout_s: float = 1.0):
        """Wait until the sampler runs, then keep only samples taken from now on."""
        t0 = time.perf_counter()
        while self._ok and not self.samples and time.perf_counter() - t0 < timeout_s:
            time.sleep(0.0002)
        self.samples.clear()
        self.reasons.clear()

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ workload and byte counts

def build_workload(rank: int = 0):
    """This rank's batch: 8 sequences of its own (weak scaling, global batch 8 x N)."""
    from bit_kv_cache_15_b200 import inputs
    from bit_kv_cache_15_b200.sharding import rank_seed
    seed = 1005 if rank == 0 else rank_seed(1005, rank)
    w, append_rows = inputs.prefill_append(seed=seed)
    return w, append_rows


def algorithmic_bytes(w, n_append_tokens):
    """Bytes the path must move, per step (no workspace, no re-reads)."""
    groups = n_append_tokens // 128
    pairs = groups * HKV
    q_bytes = pairs * ((32768 + 8192 + 528) + (32768 + 4096 + 528) + 2 * 8)   # in + codes + scales + slot
    d_bytes = 0
    for b in range(w.num_seqs):
        L = int(w.seq_lens[b])
        n_full, tl = L // 128, L % 128
        d_bytes += HKV * (n_full * (12288 + 1056) + tl * 2 * 256 + n_full * 4)
    d_bytes += 2 * w.num_seqs * HQ * 256                                             # q in, out
    return q_bytes, d_bytes


def source_sha(files):
    """Hash of a kernel's source files (the .cu and the headers it includes)."""
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "bit_kv_cache_15_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_record(kernel):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's
    sources are unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    return rec["bytes_per_launch"] if source_sha(rec["sources"]) == rec["sources_sha"] else None


# ------------------------------------------------------------------ our arm

def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w, rows = build_workload(rank)
    oracle_step = None
    if world == 1 and not args.no_cpu_baseline:
        # the CPU baseline's worker pool is forked now, before this process
        # first touches the GPU
        from oracle.parallel_step import OracleStep
        oracle_step = OracleStep(w, rows)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from bit_kv_cache_15_b200 import kvarn as K

    cfg = K.config("kvarn_k4v2_g128")
    packed, scales = K.alloc_cache(cfg, w.num_blocks, HKV, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # one-time prefill of every full tile
    K.quantize_tiles(torch.from_numpy(w.k_full).to(dev), torch.from_numpy(w.v_full).to(dev),
                     torch.from_numpy(w.slot_mapping).to(dev), packed, scales, cfg, dev_status=status)
    k_app = torch.from_numpy(np.ascontiguousarray(w.k_full[rows])).to(dev)
    v_app = torch.from_numpy(np.ascontiguousarray(w.v_full[rows])).to(dev)
    slot_app = torch.from_numpy(np.ascontiguousarray(w.slot_mapping[rows])).to(dev)
    q = torch.from_numpy(w.q).to(dev)
    tail = torch.from_numpy(w.tail).to(dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    d = K.dims(BATCH, HQ, HKV, w.max_blocks_per_seq, w.num_blocks)
    ws = torch.empty(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step():
        # NVTX: one range per step on a timeline (the library marks each of its calls too)
        torch.cuda.nvtx.range_push("kvarn.step")
        K.quantize_tiles(k_app, v_app, slot_app, packed, scales, cfg, dev_status=status, stream=stream)
        K.decode_attention(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws, dev_status=status,
                           stream=stream)
        torch.cuda.nvtx.range_pop()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status after warm-up"

    # per-kernel event timing (separate pass, same work)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        ev[3 * i].record(stream)
        K.quantize_tiles(k_app, v_app, slot_app, packed, scales, cfg, dev_status=status, stream=stream)
        ev[3 * i + 1].record(stream)
        K.decode_attention(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws, dev_status=status,
                           stream=stream)
        ev[3 * i + 2].record(stream)
    torch.cuda.synchronize()
    tq = [ev[3 * i].elapsed_time(ev[3 * i + 1]) for i in range(args.steps)]
    td = [ev[3 * i + 1].elapsed_time(ev[3 * i + 2]) for i in range(args.steps)]

    # the timed region: exactly K steps, barrier + sync on both sides
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        sampler.start_region()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        while not e1.query():          # yield to the sampler thread while the GPU runs
            time.sleep(0.0002)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    assert int(status.item()) == 0, "device status after timing"

    # end to end through the C-ABI: pinned host inputs in, output back, every step
    h_k = torch.from_numpy(np.ascontiguousarray(w.k_full[rows])).pin_memory()
    h_v = torch.from_numpy(np.ascontiguousarray(w.v_full[rows])).pin_memory()
    h_slot = torch.from_numpy(np.ascontiguousarray(w.slot_mapping[rows])).pin_memory()
    h_q = torch.from_numpy(w.q).pin_memory()
    h_tail = torch.from_numpy(w.tail).pin_memory()
    h_bt = torch.from_numpy(w.block_table).pin_memory()
    h_sl = torch.from_numpy(w.seq_lens).pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_k, h_v, h_slot, h_q, h_tail, h_bt, h_sl))
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        k_app.copy_(h_k, non_blocking=True)
        v_app.copy_(h_v, non_blocking=True)
        slot_app.copy_(h_slot, non_blocking=True)
        q.copy_(h_q, non_blocking=True)
        tail.copy_(h_tail, non_blocking=True)
        bt.copy_(h_bt, non_blocking=True)
        sl.copy_(h_sl, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = f0.elapsed_time(f1)

    if world > 1:   # the job's time is the slowest rank's
        from bit_kv_cache_15_b200.sharding import max_over_ranks
        ms, ms_e2e = max_over_ranks(ms), max_over_ranks(ms_e2e)

    if rank == 0:
        hbm_peak, peak_kind = load_peaks()
        q_bytes, d_bytes = algorithmic_bytes(w, len(rows))
        tq_ms, td_ms = statistics.median(tq), statistics.median(td)
        q_gbs = q_bytes / (tq_ms * 1e-3) / 1e9
        d_gbs = d_bytes / (td_ms * 1e-3) / 1e9
        tiles = (len(rows) // 128) * HKV * 2
        dominant = "quantize" if tq_ms >= td_ms else "decode"
        # the quantizer is bound by its FP32 pipes: rate its algorithmic flops against
        # 148 SMs x 128 lanes x 2 flop x 1.965 GHz; the decode is rated on HBM bytes
        q_flops = (len(rows) // 128) * HKV * 2 * QUANT_FLOPS_PER_TILE
        q_tflops = q_flops / (tq_ms * 1e-3) / 1e12
        if dominant == "quantize":
            roof = {"bound": "alu", "kernel": "quantize_kernel", "achieved": q_tflops, "peak": ALU_PEAK_TFLOPS,
                    "unit": "TFLOP/s", "frac": q_tflops / ALU_PEAK_TFLOPS,
                    "traffic": traffic_record("quantize_kernel"), "algorithmic_bytes": q_bytes,
                    "peak_kind": "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1965 MHz (clocks.max.sm)",
                    "hbm_view": {"achieved_gbs": q_gbs, "peak_gbs": hbm_peak, "frac": q_gbs / hbm_peak,
                                 "peak_kind": f"{peak_kind} (burst copy)"}}
        else:
            roof = {"bound": "hbm", "kernel": "decode_kernel", "achieved": d_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": d_gbs / hbm_peak, "traffic": traffic_record("decode_kernel"),
                    "algorithmic_bytes": d_bytes, "peak_kind": f"{peak_kind} (burst copy)"}
        clocks = sampler.summary()
        line = {
            "metric": METRIC,
            "value": world * BATCH * args.steps / (ms * 1e-3),
            "unit": "decode tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32 (fp16 in/out, k4v2 codes, fp32 arithmetic and accumulation)",
            "data": "synthetic (seeded; Llama/Qwen-shaped GQA, outlier channels + lognormal token scales)",
            "config": {"workload": WORKLOAD, "global_batch": BATCH * world, "seq_len": 16384,
                       "parallelism": f"data-parallel x{world}: each rank its own 8 sequences, no collective on the path",
                       "l2": f"inputs larger than L2: {(q_bytes + d_bytes) / 1e6:.0f} MB of algorithmic traffic per step"},
            "e2e": {"value": world * BATCH * args.steps / (ms_e2e * 1e-3), "unit": "decode tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            # our kernels per step: quantize_kernel, decode_kernel and the decode's merge_kernel
            "gpu_launches": 3 * args.steps,
            "roofline": roof,
            "kernels": {
                "quantize": {"us": tq_ms * 1e3, "tiles_per_s": tiles / (tq_ms * 1e-3), "tflops": q_tflops,
                             "algorithmic_bytes": q_bytes, "hbm_gbs": q_gbs, "frac_of_measured_hbm": q_gbs / hbm_peak,
                             "frac_of_8tbs": q_gbs / 8000.0},
                "decode": {"us": td_ms * 1e3, "tokens_per_s": BATCH / (td_ms * 1e-3),
                           "context_tokens_per_s": float(np.sum(w.seq_lens)) / (td_ms * 1e-3),
                           "algorithmic_bytes": d_bytes, "hbm_gbs": d_gbs, "frac_of_measured_hbm": d_gbs / hbm_peak,
                           "frac_of_8tbs": d_gbs / 8000.0},
            },
            "clocks": clocks,
        }
        if world == 1 and not args.no_sweep:
            line["sweep"] = {"workload": "decode only, batch 8 at 16384 + ragged tail, Hq=64 Hkv=8, L2 flushed "
                                         "before each call", "results": precision_sweep(w, rows, dev)}
        if oracle_step is not None:
            line["cpu_baseline"] = cpu_baseline(oracle_step)
        print(json.dumps(line), flush=True)
    if oracle_step is not None:
        oracle_step.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ precision sweep (outside the timed step)

def precision_sweep(w, rows, dev, iters=30):
    """Decode-only time of the same batch-8 16K (+tail) problem at k8v8 / k4v4 /
    k4v2 / k2v2 and over uncompressed fp16 and e4m3 caches (the in-library
    baselines); the quantiser on the step's 4096 appended tiles at each width;
    and the k4v2 decode of the Llama-3-8B- and Llama-3-70B-shaped workloads.
    Each call is timed alone with CUDA events after a 256 MB write that
    flushes L2.  Returns {name: {us, ...}}."""
    import torch
    from bit_kv_cache_15_b200 import kvarn as K
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    q = torch.from_numpy(w.q).to(dev)
    tail = torch.from_numpy(w.tail).to(dev)
    bt = torch.from_numpy(w.block_table).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    out = torch.empty_like(q)
    lens = [int(x) for x in w.seq_lens]
    n_full_tok = sum(L // 128 * 128 for L in lens)
    tail_tok = sum(L % 128 for L in lens)
    res = {}

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(iters):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e3

    kf = torch.from_numpy(w.k_full).to(dev)
    vf = torch.from_numpy(w.v_full).to(dev)
    slot = torch.from_numpy(w.slot_mapping).to(dev)
    k_app, v_app, slot_app = kf[rows], vf[rows], slot[rows]
    tiles = len(rows) // 128 * HKV * 2
    hbm_peak, _ = load_peaks()
    for kb, vb in ((8, 8), (4, 4), (4, 2), (2, 2)):
        cfg = K.config(f"kvarn_k{kb}v{vb}_g128")
        packed, scales = K.alloc_cache(cfg, w.num_blocks, HKV, device=dev)
        K.quantize_tiles(kf, vf, slot, packed, scales, cfg)
        us = timed(lambda: K.quantize_tiles(k_app, v_app, slot_app, packed, scales, cfg))
        qbytes = len(rows) // 128 * HKV * (2 * 32768 + 2048 * (kb + vb) + 2 * 528 + 16)
        res[f"quantize_k{kb}v{vb}"] = {"us": us, "tiles_per_s": tiles / (us * 1e-6), "tiles": tiles,
                                        "hbm_gbs": qbytes / (us * 1e-6) / 1e9,
                                        "frac_of_measured_hbm": qbytes / (us * 1e-6) / 1e9 / hbm_peak,
                                        "tflops": tiles * QUANT_FLOPS_PER_TILE / (us * 1e-6) / 1e12}
        d = K.dims(BATCH, HQ, HKV, w.max_blocks_per_seq, w.num_blocks)
        ws = torch.empty(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device=dev)
        us = timed(lambda: K.decode_attention(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws))
        nbytes = HKV * (n_full_tok // 128 * (2048 * (kb + vb) + 1056) + tail_tok * 512) + 2 * BATCH * HQ * 256
        res[f"k{kb}v{vb}"] = {"us": us, "tokens_per_s": BATCH / (us * 1e-6), "hbm_gbs": nbytes / (us * 1e-6) / 1e9,
                              "bytes": nbytes}
        if (kb, vb) == (4, 2):
            res.update(append_step(w, dev, cfg, kf, vf, slot, q, tail, sl, out, ws, nbytes, timed))
            res.update(multiquery_step(w, dev, cfg, packed, scales, tail, bt, timed))
        del packed, scales
    # uncompressed caches: full tiles from the same K/V, the tail in one extra block per sequence
    nb = w.num_blocks + BATCH
    kc = torch.zeros((nb, HKV, 128, 128), dtype=torch.float16, device=dev)
    vc = torch.zeros_like(kc)
    blk = torch.from_numpy(w.slot_mapping[::128] // 128).to(dev)
    kc[blk] = kf.view(-1, 128, HKV, 128).transpose(1, 2)
    vc[blk] = vf.view(-1, 128, HKV, 128).transpose(1, 2)
    bt2 = w.block_table.copy()
    for b, L in enumerate(lens):
        if L % 128:
            bt2[b, L // 128] = w.num_blocks + b
            kc[w.num_blocks + b] = tail[b, 0]
            vc[w.num_blocks + b] = tail[b, 1]
    bt2d = torch.from_numpy(bt2).to(dev)
    d = K.dims(BATCH, HQ, HKV, w.max_blocks_per_seq, nb)
    wsb = torch.empty(K.baseline_workspace_bytes(d), dtype=torch.uint8, device=dev)
    us = timed(lambda: K.decode_attention_fp16(q, kc, vc, bt2d, sl, out=out, workspace=wsb))
    nbytes = HKV * (n_full_tok + tail_tok) * 512 + 2 * BATCH * HQ * 256
    res["fp16"] = {"us": us, "tokens_per_s": BATCH / (us * 1e-6), "hbm_gbs": nbytes / (us * 1e-6) / 1e9, "bytes": nbytes}
    k_scale = float(kc.abs().max()) / 448.0
    v_scale = float(vc.abs().max()) / 448.0
    k8 = (kc.float() / k_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (vc.float() / v_scale).to(torch.float8_e4m3fn).view(torch.uint8)
    del kc, vc
    us = timed(lambda: K.decode_attention_fp8(q, k8, v8, bt2d, sl, k_scale, v_scale, out=out, workspace=wsb))
    nbytes = HKV * (n_full_tok + tail_tok) * 256 + 2 * BATCH * HQ * 256
    res["fp8"] = {"us": us, "tokens_per_s": BATCH / (us * 1e-6), "hbm_gbs": nbytes / (us * 1e-6) / 1e9, "bytes": nbytes}
    del k8, v8, wsb
    res.update(config_decodes(dev, timed))
    return res


def config_decodes(dev, timed):
    """k4v2 decode of the Llama-3-8B-shaped (B=16 x 4096, 32/8 heads) and the
    Llama-3-70B-shaped (B=4, lengths U[1024, 131072], 64/8 heads) workloads,
    each cache quantised first, the decode timed alone."""
    import torch
    from bit_kv_cache_15_b200 import inputs
    from bit_kv_cache_15_b200 import kvarn as K
    hbm_peak, kind = load_peaks()
    res = {}
    for name, make in (("llama3_8b_b16_4k", inputs.llama3_8b), ("llama3_70b_b4_1k_128k", inputs.llama3_70b)):
        w = make()
        cfg = K.config("kvarn_k4v2_g128")
        packed, scales = K.alloc_cache(cfg, w.num_blocks, w.num_kv_heads, device=dev)
        K.quantize_tiles(torch.from_numpy(w.k_full).to(dev), torch.from_numpy(w.v_full).to(dev),
                         torch.from_numpy(w.slot_mapping).to(dev), packed, scales, cfg)
        q = torch.from_numpy(w.q).to(dev)
        tail = torch.from_numpy(w.tail).to(dev)
        bt = torch.from_numpy(w.block_table).to(dev)
        sl = torch.from_numpy(w.seq_lens).to(dev)
        out = torch.empty_like(q)
        d = K.dims(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.max_blocks_per_seq, w.num_blocks)
        ws = torch.empty(K.decode_workspace_bytes(cfg, d), dtype=torch.uint8, device=dev)
        us = timed(lambda: K.decode_attention(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws))
        lens = [int(x) for x in w.seq_lens]
        nbytes = (w.num_kv_heads * sum(L // 128 * (12288 + 1056 + 4) + L % 128 * 512 for L in lens)
                  + 2 * w.num_seqs * w.num_q_heads * 256)
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"us": us, "tokens_per_s": w.num_seqs / (us * 1e-6),
                     "context_tokens_per_s": sum(lens) / (us * 1e-6), "seq_lens": lens, "bytes": nbytes,
                     "hbm_gbs": gbs, "frac_of_measured_hbm": gbs / hbm_peak, "frac_of_8tbs": gbs / 8000.0}
        del packed, scales, w
        torch.cuda.empty_cache()
    return res


def multiquery_step(w, dev, cfg, packed, scales, tail, bt, timed, q_len=4):
    """Multi-query attention (a verify step of q_len draft tokens) on the same
    cache: every sequence's tail holds at least q_len - 1 rows so that all
    queries sit after its last full tile.  Reports query tokens per second."""
    import torch
    from bit_kv_cache_15_b200 import kvarn as K
    lens = [int(L) // 128 * 128 + max(int(L) % 128, q_len - 1) for L in w.seq_lens]
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev).manual_seed(78)
    q = torch.randn((BATCH, q_len, HQ, 128), generator=g, device=dev).half()
    out = torch.empty_like(q)
    d = K.dims(BATCH, HQ, HKV, w.max_blocks_per_seq, w.num_blocks)
    ws = torch.empty(K.decode_multiquery_workspace_bytes(cfg, d, q_len), dtype=torch.uint8, device=dev)
    us = timed(lambda: K.decode_attention_multiquery(q, packed, scales, tail, bt, sl, cfg, out=out, workspace=ws))
    return {f"multiquery{q_len}_k4v2": {"us": us, "query_tokens_per_s": BATCH * q_len / (us * 1e-6),
                                        "q_len": q_len}}


def append_step(w, dev, cfg, kf, vf, slot, q, tail, sl, out, ws, decode_bytes, timed):
    """The decode step with append (k4v2) on the same problem: (a) as the
    workload stands (its tails are U{0..127}; a sequence at 127 fills), and
    (b) with every sequence's tail at 127 rows, so each (sequence, KV head)
    quantises a tile inside the step (the worst case, 64 tiles of K and V).
    Repeated calls rewrite the same tail row and block, so they are identical."""
    import torch
    from bit_kv_cache_15_b200 import kvarn as K
    g = torch.Generator(device=dev).manual_seed(77)
    k_new = torch.randn((BATCH, HKV, 128), generator=g, device=dev).half()
    v_new = torch.randn((BATCH, HKV, 128), generator=g, device=dev).half()
    lens = [int(x) for x in w.seq_lens]
    nb = w.num_blocks + BATCH
    packed, scales = K.alloc_cache(cfg, nb, HKV, device=dev)
    K.quantize_tiles(kf, vf, slot, packed, scales, cfg)
    bt = w.block_table.copy()
    fills = 0
    for b, L in enumerate(lens):
        if L % 128 == 127:
            bt[b, L // 128] = w.num_blocks + b
            fills += 1
    btd = torch.from_numpy(bt).to(dev)
    tl = tail.clone()
    new_bytes = 2 * BATCH * HKV * 256 * 2          # k_new / v_new read, tail rows written
    tile_bytes = HKV * (2 * 32768 + 2048 * 6 + 1056)  # per filled sequence: both tiles read, codes + scales written
    us = timed(lambda: K.decode_attention_append(q, k_new, v_new, packed, scales, tl, btd, sl, cfg, out=out,
                                                 workspace=ws))
    res = {"append_k4v2": {"us": us, "tokens_per_s": BATCH / (us * 1e-6), "fills": fills,
                           "bytes": decode_bytes + new_bytes + fills * tile_bytes}}
    lens_f = [L // 128 * 128 + 127 for L in lens]
    bt_f = w.block_table.copy()
    for b, L in enumerate(lens_f):
        if L // 128 >= bt_f.shape[1]:
            return res
        bt_f[b, L // 128] = w.num_blocks + b
    btf = torch.from_numpy(bt_f).to(dev)
    slf = torch.tensor(lens_f, dtype=torch.int32, device=dev)
    us = timed(lambda: K.decode_attention_append(q, k_new, v_new, packed, scales, tl, btf, slf, cfg, out=out,
                                                 workspace=ws))
    res["append_fill_all_k4v2"] = {"us": us, "tokens_per_s": BATCH / (us * 1e-6), "fills": BATCH,
                                   "quantised_tiles": 2 * BATCH * HKV}
    return res


# ------------------------------------------------------------------ the oracle (CPU baseline / reference arm)

ORACLE_STEP = ("one whole step of the same workload: the oracle (numpy fp64) quantises the 4096 appended K+V "
               "tiles into the paged cache, then decodes all 64 (sequence, KV head) pairs; one process per host "
               "core, one BLAS thread each; the rest of the cache is quantised once before timing")


def cpu_baseline(oracle_step, steps=1):
    """The oracle timed on whole steps over all host cores (no extrapolation)."""
    oracle_step.prefill()
    ts = oracle_step.timed_steps(steps)
    t = statistics.median(ts)
    return {"value": BATCH / t, "unit": "decode tokens/s", "cores": oracle_step.workers, "kind": "oracle",
            "sample": f"{ORACLE_STEP}; {steps} step(s), {t:.2f} s each"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle.parallel_step import OracleStep
    w, rows = build_workload()
    st = OracleStep(w, rows)
    try:
        st.prefill()
        st.timed_steps(args.warmup)
        t_steps = st.timed_steps(args.steps)
    finally:
        st.close()
    total = float(np.sum(t_steps))
    t_mean = total / len(t_steps)
    value = BATCH / t_mean
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "decode tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_mean * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic (seeded)",
        "config": {"workload": WORKLOAD, "global_batch": BATCH, "seq_len": 16384,
                   "parallelism": f"none (CPU: {st.workers} worker processes)"},
        "cpu_baseline": {"value": value, "unit": "decode tokens/s", "cores": st.workers, "kind": "oracle",
                         "sample": f"{ORACLE_STEP}; {args.steps} timed steps after {args.warmup} warm-up steps, "
                                   f"{total:.1f} s timed in total"},
        "e2e": {"value": value, "unit": "decode tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
