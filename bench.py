#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path on B200.

One step = one pass of every step of the path over the Wan-1.3B-like layer
(12 heads x 128, bf16, history 21 frames x 1,560 = 32,760 tokens, query chunk
4,680 tokens, 256 centroids per head, K INT2 / V INT2, group 16):

  fit centroids (K, V; 2 k-means rounds) -> encode (K, V) -> decode (K, V)
  -> joint head-channel code of the same history (K, V: rank 192, INT4,
     group 32, orthonormal W_enc): encode, then decode
  -> attention of the chunk over the compressed history in 2 blocks
  -> LSE merge of the 2 partial results.

Inputs are seeded synthetic tensors resident in HBM before timing starts;
L2 is flushed (256 MiB write) before every timed step, outside the step's
events.  The headline value is history tokens per second of whole steps,
summed over ranks.  ``--impl reference`` times the CPU oracle instead on a
bounded sample of the same workload.

Beside the step (after its timed region, L2 flushed before each call) the
line's ``next_rows`` reports the current chunk's full-layer attention --
the compressed history plus the chunk's own 4,680 uncompressed keys under one
softmax (kvq_layer_attention) -- and its dense part alone
(kvq_attention_dense_lse), each as mean device time and TFLOP/s of
4 Tq keys d H flops.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "encode history-tokens/s (HBM GB/s) and compressed-KV attention TFLOP/s, 1×B200"
UNIT = "history-tokens/s"
WORKLOAD = "wan13b"
HISTORY_BLOCKS = 2
FLUSH_BYTES = 256 << 20
# DRAM bytes (read + write) of one attention_pair_kernel launch of this
# workload, from the ncu capture summarised in profiles/attention_pair_wan13b.md;
# None whenever the kernel has changed since that capture.  The last capture
# (92.6 MB per launch) predates the per-codec instantiation of the kernel.
ATTN_NCU_TRAFFIC_BYTES = None


def _joint():
    """The joint head-channel workload (same history shape as WORKLOAD)."""
    from kv_cache_compression_head_b200 import synth

    return synth.workload("joint")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


# ----------------------------------------------------------------------------
# distributed plumbing (replicas: every rank runs the full workload)
# ----------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, backend):
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds
    by a background thread through NVML (read-only queries) between start()
    and stop(); falls back to `nvidia-smi -lms` where NVML is unavailable."""

    PERIOD_S = 0.005
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.thread = None
        self.stop_flag = False
        self.nvml = None
        try:
            import pynvml

            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [v for v in vis.split(",") if v.strip()]
            phys = int(ids[gpu_index]) if gpu_index < len(ids) and ids[gpu_index].strip().isdigit() else gpu_index
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.masks = [(n, getattr(pynvml, c, 0)) for n, c in self.REASONS]
            self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _poll(self):
        nv = self.nvml
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.rows.append((float(sm), float(self.sm_max), pw, [n for n, m in self.masks if m and rs & m]))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def start(self):
        if self.nvml is None:
            return
        import threading

        self.rows = []
        self.stop_flag = False
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.nvml is None or self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable"]}
        self.stop_flag = True
        self.thread.join(timeout=5)
        rows = self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = sorted({n for r in loaded for n in r[3]})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows), "sampler": "NVML every 5 ms"}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------
# algorithmic work per step (roofline numerators)
# ----------------------------------------------------------------------------

def work_model(w):
    T, H, d, Tq, C, G = w.history_tokens, w.num_heads, w.head_dim, w.query_tokens, w.num_centroids, w.group_size
    th = T * H

    def stored(bits):  # bytes written per token-head by encode
        return d * bits // 8 + 8 * (d // G) + 2

    enc_bytes = sum(th * (2 * d + stored(b)) for b in (w.bits_k, w.bits_v))
    dec_bytes = sum(th * (stored(b) + 2 * d) for b in (w.bits_k, w.bits_v))  # read compressed, write bf16
    attn_flops = 4.0 * Tq * T * d * H
    merge_bytes = (HISTORY_BLOCKS + 1) * Tq * H * d * 4 + (HISTORY_BLOCKS + 1) * Tq * H * 4
    # fit, per k-means round and token-head: the assignment reads x and writes
    # its index, the accumulation reads x and the index (K and V)
    fit_bytes = 2 * w.kmeans_iters * th * (2 * d + 2 + 2 * d + 2)
    # joint code, K and V: the assignment pass reads x and writes idx; the
    # projection pass reads x and idx and writes r*b/8 code bytes and r/G
    # {s, z} pairs per token; the decoder reads those and writes bf16 x^
    wj = _joint()
    jstored = wj.joint_rank * wj.bits_k // 8 + 8 * (wj.joint_rank // wj.joint_group)
    joint_enc_bytes = 2 * T * (2 * (2 * H * d + 2 * H) + jstored)
    joint_dec_bytes = 2 * T * (2 * H + jstored + 2 * H * d)
    joint_flops = 2 * T * 2.0 * H * d * wj.joint_rank  # one GEMM per direction, K and V
    return {"encode_bytes": enc_bytes, "decode_bytes": dec_bytes, "attention_flops": attn_flops,
            "merge_bytes": merge_bytes, "fit_bytes": fit_bytes, "joint_enc_bytes": joint_enc_bytes,
            "joint_dec_bytes": joint_dec_bytes, "joint_gemm_flops": joint_flops}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

class Pipeline:
    """Device buffers and the per-step call sequence through the public API."""

    ROWS = ("fit", "encode", "decode", "joint_encode", "joint_decode", "attention", "merge")

    def __init__(self, w, device):
        import torch

        from kv_cache_compression_head_b200 import kvq as K

        self.K = K
        self.w = w
        self.dev = device
        T, H, d, Tq = w.history_tokens, w.num_heads, w.head_dim, w.query_tokens
        self.codec_k = K.Codec(H, d, w.num_centroids, w.bits_k, w.group_size)
        self.codec_v = K.Codec(H, d, w.num_centroids, w.bits_v, w.group_size)
        bf = torch.bfloat16
        self.xk = torch.empty((T, H, d), dtype=bf, device=device)
        self.xv = torch.empty((T, H, d), dtype=bf, device=device)
        self.q = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.cent = [torch.empty((H, w.num_centroids, d), dtype=bf, device=device) for _ in range(2)]
        self.enc = [K.alloc_encoded(c, T, device) for c in (self.codec_k, self.codec_v)]
        self.ws = K.alloc_workspace(K.KVQ_OP_FIT, self.codec_k, T, device)
        self.ws_attn = K.alloc_workspace(K.KVQ_OP_ATTENTION, self.codec_k, T, device, num_queries=Tq)
        self.dec = [torch.empty((T, H, d), dtype=bf, device=device) for _ in range(2)]
        self.o_parts = [torch.empty((Tq, H, d), dtype=torch.float32, device=device) for _ in range(HISTORY_BLOCKS)]
        self.l_parts = [torch.empty((H, Tq), dtype=torch.float32, device=device) for _ in range(HISTORY_BLOCKS)]
        self.o = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.lse = torch.empty((H, Tq), dtype=torch.float32, device=device)
        self.edges = [T * i // HISTORY_BLOCKS for i in range(HISTORY_BLOCKS + 1)]
        self.comp = [K.Compressed(c, T, self.cent[i], *self.enc[i])
                     for i, c in enumerate((self.codec_k, self.codec_v))]
        # joint head-channel code of the same history (same centres)
        from kv_cache_compression_head_b200 import synth

        wj = _joint()
        self.codec_j = [K.Codec(H, d, w.num_centroids, b, wj.joint_group, wj.joint_rank)
                        for b in (wj.bits_k, wj.bits_v)]
        w_enc = synth.make_orthonormal_encoder(wj)
        self.w_enc = torch.from_numpy(w_enc.view(np.int16)).view(bf).to(device)
        self.w_dec = self.w_enc.t().contiguous()
        self.enc_j = [K.alloc_encoded(c, T, device) for c in self.codec_j]
        self.comp_j = [K.Compressed(c, T, self.cent[i], *self.enc_j[i], w_dec=self.w_dec)
                       for i, c in enumerate(self.codec_j)]
        # full-layer attention (outside the step): the chunk's own keys and
        # values follow the history; one call = compressed part + dense part
        # + their merge
        self.kc = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.vc = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.ws_layer = K.alloc_workspace(K.KVQ_OP_LAYER_ATTENTION, self.codec_k, T, device, num_queries=Tq)
        self.o_layer = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.lse_layer = torch.empty((H, Tq), dtype=torch.float32, device=device)
        # fit: seed + (assign + 4 sort + 3 update kernels) per round; encode 1;
        # decode 1; joint encode 2 (assign, projection), joint decode 1;
        # attention 2 per block (split + its merge); final merge 1 -- K and V
        self.launches_per_step = (2 * (1 + 8 * w.kmeans_iters) + 2 + 2 + 2 * 2 + 2 + 2 * HISTORY_BLOCKS + 1)

    def outputs(self):
        outs = [self.o, self.lse]
        for i in range(2):
            outs += [self.cent[i], *self.enc[i], *self.enc_j[i]]
        return outs

    def step(self, ev=None):
        """Run one step; ev (optional) is a dict row -> (start, end) events."""
        K, w = self.K, self.w

        def mark(row, i):
            if ev is not None:
                ev[row][i].record()

        mark("fit", 0)
        K.kvq_fit_centroids(self.codec_k, self.xk, w.kmeans_iters, self.cent[0], self.ws)
        K.kvq_fit_centroids(self.codec_v, self.xv, w.kmeans_iters, self.cent[1], self.ws)
        mark("fit", 1)
        mark("encode", 0)
        K.kvq_encode(self.codec_k, self.xk, self.cent[0], *self.enc[0])
        K.kvq_encode(self.codec_v, self.xv, self.cent[1], *self.enc[1])
        mark("encode", 1)
        mark("decode", 0)
        K.kvq_decode(self.comp[0], self.dec[0])
        K.kvq_decode(self.comp[1], self.dec[1])
        mark("decode", 1)
        mark("joint_encode", 0)
        K.kvq_encode(self.codec_j[0], self.xk, self.cent[0], *self.enc_j[0], w_enc=self.w_enc)
        K.kvq_encode(self.codec_j[1], self.xv, self.cent[1], *self.enc_j[1], w_enc=self.w_enc)
        mark("joint_encode", 1)
        mark("joint_decode", 0)
        K.kvq_decode(self.comp_j[0], self.dec[0])
        K.kvq_decode(self.comp_j[1], self.dec[1])
        mark("joint_decode", 1)
        mark("attention", 0)
        for b in range(HISTORY_BLOCKS):
            K.kvq_attention_lse(self.q, self.comp[0], self.comp[1], self.o_parts[b], self.l_parts[b],
                                t_begin=self.edges[b], t_end=self.edges[b + 1], workspace=self.ws_attn)
        mark("attention", 1)
        mark("merge", 0)
        K.kvq_lse_merge(self.o_parts, self.l_parts, self.o, self.lse)
        mark("merge", 1)


    def layer_attention(self):
        self.K.kvq_layer_attention(self.q, self.comp[0], self.comp[1], self.kc, self.vc, self.o_layer,
                                   self.lse_layer, self.ws_layer)

    def dense_attention(self):
        self.K.kvq_attention_dense_lse(self.q, self.kc, self.vc, self.o_layer, self.lse_layer,
                                       workspace=self.ws_attn)


def time_calls(fn, reps, warmup, flush):
    """Mean device time (ms) of fn() over reps calls, L2 flushed before each."""
    import torch

    for _ in range(warmup):
        flush.zero_()
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def run_gpu(args):
    import torch

    from kv_cache_compression_head_b200 import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = synth.workload(WORKLOAD)

    # seeded inputs: generated on the host, staged in pinned memory
    hk = synth.make_history(w, "K")
    hv = synth.make_history(w, "V")
    hq = synth.make_queries(w)
    pin = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    pk, pv, pq = pin(hk), pin(hv), pin(hq)

    pipe = Pipeline(w, device)
    pipe.xk.copy_(pk)
    pipe.xv.copy_(pv)
    pipe.q.copy_(pq)
    pipe.kc.copy_(pin(synth.make_chunk(w, "K")))
    pipe.vc.copy_(pin(synth.make_chunk(w, "V")))
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        pipe.step()
    torch.cuda.synchronize()
    st = pipe.K.kvq_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {pipe.K.status_string(st)}")

    ev = [{r: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for r in Pipeline.ROWS}
          for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t_wall = time.perf_counter()
    for k in range(args.steps):
        flush.zero_()
        pipe.step(ev[k])
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_wall
    barrier(world)
    clk = clocks.stop()
    st = pipe.K.kvq_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status after timing: {pipe.K.status_string(st)}")

    # next to the step: the current chunk's full-layer attention (compressed
    # history + its own uncompressed keys, merged by LSE) and the dense part
    # alone, on the step's freshly encoded history
    layer_ms = max_over_ranks(time_calls(pipe.layer_attention, args.steps, args.warmup, flush), world, device)
    dense_ms = max_over_ranks(time_calls(pipe.dense_attention, args.steps, args.warmup, flush), world, device)
    st = pipe.K.kvq_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status after the layer attention: {pipe.K.status_string(st)}")

    row_ms = {r: [e[r][0].elapsed_time(e[r][1]) for e in ev] for r in Pipeline.ROWS}
    step_ms = [ev[k]["fit"][0].elapsed_time(ev[k]["merge"][1]) for k in range(args.steps)]
    ms_step_local = statistics.mean(step_ms)
    ms_step = max_over_ranks(ms_step_local, world, device)
    row_mean = {r: statistics.mean(v) for r, v in row_ms.items()}

    # end-to-end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        outs = pipe.outputs()
        host_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
        h2d = sum(t.numel() * t.element_size() for t in (pk, pv, pq))
        d2h = sum(t.numel() * t.element_size() for t in outs)
        e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        for k in range(args.steps + 1):  # first pass untimed
            if k > 0:
                e_ev[k - 1][0].record()
            pipe.xk.copy_(pk, non_blocking=True)
            pipe.xv.copy_(pv, non_blocking=True)
            pipe.q.copy_(pq, non_blocking=True)
            pipe.step()
            for ho, o in zip(host_outs, outs):
                ho.copy_(o, non_blocking=True)
            if k > 0:
                e_ev[k - 1][1].record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in e_ev), world, device)
        e2e = {"value": world * w.history_tokens / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank == 0:
        wm = work_model(w)
        hbm, tfl, peak_kind = measured_peaks()
        attn_launch_ms = row_mean["attention"] / HISTORY_BLOCKS
        attn_launch_flops = wm["attention_flops"] / HISTORY_BLOCKS
        attn_tflops = attn_launch_flops / (attn_launch_ms / 1e3) / 1e12
        enc_gbps = wm["encode_bytes"] / (row_mean["encode"] / 1e3) / 1e9
        dec_gbps = wm["decode_bytes"] / (row_mean["decode"] / 1e3) / 1e9
        merge_gbps = wm["merge_bytes"] / (row_mean["merge"] / 1e3) / 1e9
        fit_gbps = wm["fit_bytes"] / (row_mean["fit"] / 1e3) / 1e9
        jenc_gbps = wm["joint_enc_bytes"] / (row_mean["joint_encode"] / 1e3) / 1e9
        jdec_gbps = wm["joint_dec_bytes"] / (row_mean["joint_decode"] / 1e3) / 1e9
        jdec_tflops = wm["joint_gemm_flops"] / 2 / (row_mean["joint_decode"] / 1e3) / 1e12
        jenc_tflops = wm["joint_gemm_flops"] / 2 / (row_mean["joint_encode"] / 1e3) / 1e12
        rows = {
            "fit": {"ms": row_mean["fit"], "gbps": fit_gbps, "hbm_frac": fit_gbps / hbm},
            "encode": {"ms": row_mean["encode"], "tokens_per_s": w.history_tokens / (row_mean["encode"] / 1e3),
                       "gbps": enc_gbps, "hbm_frac": enc_gbps / hbm},
            "decode": {"ms": row_mean["decode"], "gbps": dec_gbps, "hbm_frac": dec_gbps / hbm},
            "joint_encode": {"ms": row_mean["joint_encode"], "gbps": jenc_gbps, "hbm_frac": jenc_gbps / hbm,
                             "gemm_tflops": jenc_tflops},
            "joint_decode": {"ms": row_mean["joint_decode"], "gbps": jdec_gbps, "hbm_frac": jdec_gbps / hbm,
                             "gemm_tflops": jdec_tflops},
            "attention": {"ms": row_mean["attention"], "launches": HISTORY_BLOCKS, "tflops": attn_tflops,
                          "frac": attn_tflops / tfl},
            "merge": {"ms": row_mean["merge"], "gbps": merge_gbps, "hbm_frac": merge_gbps / hbm},
        }
        Tq, H, d = w.query_tokens, w.num_heads, w.head_dim
        layer_flops = 4.0 * Tq * (w.history_tokens + Tq) * d * H
        dense_flops = 4.0 * Tq * Tq * d * H
        next_rows = {
            "layer_attention": {"ms": layer_ms, "calls": 1, "keys": w.history_tokens + Tq,
                                "tflops": layer_flops / (layer_ms / 1e3) / 1e12,
                                "frac": layer_flops / (layer_ms / 1e3) / 1e12 / tfl,
                                "what": "kvq_layer_attention: 32760 compressed history keys + the 4680-key chunk "
                                        "(bf16), one softmax, LSE merge inside the call"},
            "dense_attention": {"ms": dense_ms, "calls": 1, "keys": Tq,
                                "tflops": dense_flops / (dense_ms / 1e3) / 1e12,
                                "frac": dense_flops / (dense_ms / 1e3) / 1e12 / tfl,
                                "what": "kvq_attention_dense_lse over the 4680-key chunk alone"},
        }
        line = {
            "metric": METRIC,
            "value": world * w.history_tokens / (ms_step / 1e3),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded AR(1) frames + heavy-tailed outlier channels)",
            "config": {"workload": "wan13b-like layer: 12 heads x 128, history 32760 tokens (21 frames x 1560), "
                                   "query chunk 4680, C=256, K2V2, group 16, fit 2 rounds, 2 history blocks; "
                                   "joint code of the same history: rank 192, K4V4, group 32",
                       "history_tokens": w.history_tokens, "query_tokens": w.query_tokens,
                       "heads": w.num_heads, "head_dim": w.head_dim, "centroids": w.num_centroids,
                       "bits_k": w.bits_k, "bits_v": w.bits_v, "group": w.group_size,
                       "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before each step"},
            "roofline": {"kernel": "attention_pair_kernel<2, 2, false> (time of the whole kvq_attention_lse call, "
                                   "incl. its in-call LSE merge)", "bound": "tensor", "achieved": attn_tflops,
                         "peak": tfl, "unit": "TFLOP/s", "frac": attn_tflops / tfl, "peak_kind": peak_kind,
                         "traffic": ATTN_NCU_TRAFFIC_BYTES,
                         "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
            "rows": rows,
            "next_rows": next_rows,
            "clocks": clk,
            "gpu_launches": pipe.launches_per_step * args.steps,
            "wall_s_timed_region": wall,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    barrier(world)


# ----------------------------------------------------------------------------
# CPU oracle: baseline leg and reference arm
# ----------------------------------------------------------------------------

CPU_SAMPLE_T = 4096
CPU_SAMPLE_TQ = 256


def oracle_step_times(w):
    """Time the oracle on a bounded sample of the workload: fit+encode+decode
    of the first CPU_SAMPLE_T history tokens (all heads, K and V) and attention
    (2 blocks) + merge of CPU_SAMPLE_TQ queries over them.  Returns the
    extrapolated seconds of one full step and the raw sample times."""
    from kv_cache_compression_head_b200 import synth
    from oracle import oracle as O

    Ts, Tqs = CPU_SAMPLE_T, CPU_SAMPLE_TQ
    xk = synth.make_history(w, "K", max_tokens=Ts)
    xv = synth.make_history(w, "V", max_tokens=Ts)
    q = synth.make_queries(w, max_tokens=Tqs)
    t0 = time.perf_counter()
    decs = []
    for x, bits in ((xk, w.bits_k), (xv, w.bits_v)):
        cent = O.fit(x, w.num_centroids, w.kmeans_iters)
        e = O.encode(x, cent, bits, w.group_size)
        decs.append(O.decode(*e, cent, bits, w.group_size))
    t1 = time.perf_counter()
    edges = [Ts * i // HISTORY_BLOCKS for i in range(HISTORY_BLOCKS + 1)]
    parts = [O.attention(q, decs[0][a:b], decs[1][a:b]) for a, b in zip(edges[:-1], edges[1:])]
    O.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    t2 = time.perf_counter()
    codec_s, attn_s = t1 - t0, t2 - t1
    full = codec_s * (w.history_tokens / Ts) + attn_s * (w.history_tokens * w.query_tokens) / (Ts * Tqs)
    return full, codec_s, attn_s


def _omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline(w):
    full, codec_s, attn_s = oracle_step_times(w)
    return {"value": w.history_tokens / full, "unit": UNIT, "cores": _omp_threads(), "kind": "oracle",
            "sample": f"fit+encode+decode of {CPU_SAMPLE_T}/{w.history_tokens} history tokens (12 heads, K and V): "
                      f"{codec_s:.2f}s; attention (2 blocks)+merge of {CPU_SAMPLE_TQ}/{w.query_tokens} queries "
                      f"over them: {attn_s:.2f}s; scaled per history token and per query x history token",
            "extrapolated_s_per_step": full}


def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 alone runs and prints; any
    other rank exits at once without work (and without joining a group)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from kv_cache_compression_head_b200 import synth

    w = synth.workload(WORKLOAD)
    for _ in range(args.warmup):
        oracle_step_times(w)
    fulls = []
    t_wall = time.perf_counter()
    for _ in range(args.steps):
        fulls.append(oracle_step_times(w)[0])
    wall = time.perf_counter() - t_wall
    s = statistics.mean(fulls)
    value = w.history_tokens / s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)", "data": "synthetic",
        "config": {"workload": "wan13b-like layer (bounded sample per step, extrapolated)",
                   "history_tokens": w.history_tokens, "query_tokens": w.query_tokens,
                   "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _omp_threads(), "kind": "oracle",
                         "sample": f"each step: fit+encode+decode of {CPU_SAMPLE_T} history tokens and attention "
                                   f"of {CPU_SAMPLE_TQ} queries over them, extrapolated to the full step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s_timed_region": wall,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.warmup < 0 or args.steps < 1:
        raise SystemExit("need --steps >= 1 and --warmup >= 0")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist

        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
