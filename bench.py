#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path on B200.

The headline step runs every step of the path over the 14B-like layer, the
largest workload that fits one GPU: 40 heads x 128, bf16; a history of
60 frames x 1,560 = 93,600 tokens; a query chunk of 4,680 tokens; 512
centroids per head; K INT4 / V INT2; group 32.  The step is

  fit centroids (K, V; 2 k-means rounds) -> encode (K, V) -> decode (K, V)
  -> joint head-channel code (K, V: rank 192, INT4, group 32, orthonormal
     W_enc; encode, then decode) of the joint workload's 32,760-token,
     12-head history, which is the shape the joint code is defined on
  -> attention of the chunk over the compressed history in 8 blocks
  -> LSE merge of the 8 partial results.

After the headline, the Wan-1.3B-like step (12 heads, 32,760 history tokens,
C = 256, K2V2, group 16, 2 blocks) is timed the same way and reported under
``config2``.  Next to the steps (after their timed regions, L2 flushed before
each call), ``next_rows`` reports the Wan-like chunk's full-layer attention:
the compressed history plus the chunk's own 4,680 uncompressed keys under one
softmax (kvq_layer_attention), and its dense part alone
(kvq_attention_dense_lse); QuantWM's QSAC encode, PSAC coefficients and PSAC
attention on the Wan-like layer; and NanoKV-Fast on the joint workload (the
history decoded into a 64-dim space per head, low-space attention with query
reduction and output restoration) beside its full-dimensional counterpart;
and the second residual stage's encode and decode on the Wan-like layer.

Inputs are seeded synthetic tensors resident in HBM before timing starts;
L2 is flushed (256 MiB write) before every timed step, outside the step's
events.  The headline value is history tokens per second of whole steps,
summed over ranks.

``--impl reference`` times the CPU oracle instead: every step runs the oracle
on a bounded sample of the headline workload; ``ms_per_step`` is the wall
time of that sample and ``value`` the full step's rate extrapolated from it.
``--sweep PATH`` times encode, decode and attention on a covering set of the
12-head sweep points and writes one JSON line per point to PATH.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--sweep PATH]
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
HEADLINE = "14b"
SECONDARY = "wan13b"
JOINT = "joint"
FLUSH_BYTES = 256 << 20
# DRAM bytes (read + write) of one attention kernel launch of the headline
# workload from an ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of
# the first two history-block launches of a timed step: 352.7 and 349.6 MB,
# against 329 MB of algorithmic bytes -- the block's compressed K and V, the
# centres, Q and the binary32 partials of its two sub-ranges).  The kernel has
# changed since (its bounded waits read their poll limit from constant memory;
# its softmax warps drain the last commit after a give-up), so the line
# reports traffic as null and the captured figure beside it, labelled.
ATTN_NCU_TRAFFIC_BYTES = None
ATTN_NCU_TRAFFIC_BEFORE_CHANGE = 351.1e6


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true")
    p.add_argument("--sweep", default=None, help="write per-point sweep timings (JSON lines) to this path")
    p.add_argument("--workload", default=HEADLINE, choices=["14b", "wan13b"],
                   help="the step's workload (14b: the headline; wan13b: a smaller case for profiling)")
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
    and stop().  Without NVML the line records "NVML unavailable" and no
    clock figures."""

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
# algorithmic work (roofline numerators)
# ----------------------------------------------------------------------------

def stored_bytes(d, bits, G):
    """Bytes encode writes per token-head: packed codes, {s, z} pairs, index."""
    return d * bits // 8 + 8 * (d // G) + 2


def work_model(w):
    """Algorithmic bytes and flops of one step's rows on workload w."""
    T, H, d, Tq, C, G = w.history_tokens, w.num_heads, w.head_dim, w.query_tokens, w.num_centroids, w.group_size
    th = T * H
    blocks = w.history_blocks
    enc_bytes = sum(th * (2 * d + stored_bytes(d, b, G)) for b in (w.bits_k, w.bits_v))
    dec_bytes = sum(th * (stored_bytes(d, b, G) + 2 * d) for b in (w.bits_k, w.bits_v))
    return {
        "encode_bytes": enc_bytes,
        # the assignment filter, X mu^T: 2 C d flop per token-head (K and V)
        "encode_flops": 2 * th * 2.0 * C * d,
        "decode_bytes": dec_bytes,
        "attention_flops": 4.0 * Tq * T * d * H,
        "merge_bytes": (blocks + 1) * Tq * H * d * 4 + (blocks + 1) * Tq * H * 4,
        # per k-means round and token-head: the assignment reads x and writes
        # its index, the update reads x and the index (K and V)
        "fit_bytes": 2 * w.kmeans_iters * th * (2 * d + 2 + 2 * d + 2),
    }


def joint_work_model(wj):
    """Joint code of K and V: x read once, idx and the coefficient codes and
    {s, z} written (the encoder); the decoder reads those and writes bf16."""
    T, H, d, r = wj.history_tokens, wj.num_heads, wj.head_dim, wj.joint_rank
    jstored = r * wj.bits_k // 8 + 8 * (r // wj.joint_group)
    return {"joint_enc_bytes": 2 * T * (2 * H * d + 2 * H + jstored),
            "joint_dec_bytes": 2 * T * (2 * H + jstored + 2 * H * d),
            # one GEMM per direction and branch, plus the assignment filter
            "joint_gemm_flops": 2 * T * 2.0 * H * d * r,
            "joint_filter_flops": 2 * T * H * 2.0 * wj.num_centroids * d}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def to_device_bf16(a, device):
    import torch

    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def pinned_bf16(a):
    import torch

    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()


class JointRows:
    """The joint head-channel code (rows a4 and its decoder) on the joint
    workload's history: centres fitted once at set-up (not timed), then per
    step the joint encode and decode of K and V."""

    def __init__(self, device):
        import torch

        from kv_cache_compression_head_b200 import kvq as K
        from kv_cache_compression_head_b200 import synth

        self.K = K
        wj = synth.workload(JOINT)
        self.w = wj
        T, H, d = wj.history_tokens, wj.num_heads, wj.head_dim
        bf = torch.bfloat16
        self.x = [to_device_bf16(synth.make_history(wj, which), device) for which in ("K", "V")]
        fit_codec = K.Codec(H, d, wj.num_centroids, 2, 16)
        self.cent = [torch.empty((H, wj.num_centroids, d), dtype=bf, device=device) for _ in range(2)]
        for x, c in zip(self.x, self.cent):
            K.kvq_fit_centroids(fit_codec, x, wj.kmeans_iters, c)
        self.codec = [K.Codec(H, d, wj.num_centroids, b, wj.joint_group, wj.joint_rank)
                      for b in (wj.bits_k, wj.bits_v)]
        w_enc = synth.make_orthonormal_encoder(wj)
        self.w_enc = to_device_bf16(w_enc, device)
        self.w_dec = self.w_enc.t().contiguous()
        self.enc = [K.alloc_encoded(c, T, device) for c in self.codec]
        self.comp = [K.Compressed(c, T, self.cent[i], *self.enc[i], w_dec=self.w_dec)
                     for i, c in enumerate(self.codec)]
        self.dec = [torch.empty((T, H, d), dtype=bf, device=device) for _ in range(2)]
        self.launches = 2 * 2 + 2  # per branch: assignment + projection; decoder

    def encode(self):
        for i in range(2):
            self.K.kvq_encode(self.codec[i], self.x[i], self.cent[i], *self.enc[i], w_enc=self.w_enc)

    def decode(self):
        for i in range(2):
            self.K.kvq_decode(self.comp[i], self.dec[i])

    def outputs(self):
        return [t for e in self.enc for t in e]


class Pipeline:
    """Device buffers of one workload and its per-step call sequence through
    the public API."""

    def __init__(self, w, device, joint=None, layer=False):
        import torch

        from kv_cache_compression_head_b200 import kvq as K

        self.K = K
        self.w = w
        self.dev = device
        self.joint = joint
        T, H, d, Tq = w.history_tokens, w.num_heads, w.head_dim, w.query_tokens
        self.blocks = w.history_blocks if w.history_blocks > 1 else 2
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
        self.o_parts = [torch.empty((Tq, H, d), dtype=torch.float32, device=device) for _ in range(self.blocks)]
        self.l_parts = [torch.empty((H, Tq), dtype=torch.float32, device=device) for _ in range(self.blocks)]
        self.o = torch.empty((Tq, H, d), dtype=bf, device=device)
        self.lse = torch.empty((H, Tq), dtype=torch.float32, device=device)
        self.edges = [T * i // self.blocks for i in range(self.blocks + 1)]
        self.comp = [K.Compressed(c, T, self.cent[i], *self.enc[i])
                     for i, c in enumerate((self.codec_k, self.codec_v))]
        self.layer = layer
        if layer:
            # full-layer attention (outside the step): the chunk's own keys and
            # values follow the history; one call = compressed part + dense
            # part + their merge
            self.kc = torch.empty((Tq, H, d), dtype=bf, device=device)
            self.vc = torch.empty((Tq, H, d), dtype=bf, device=device)
            self.ws_layer = K.alloc_workspace(K.KVQ_OP_LAYER_ATTENTION, self.codec_k, T, device, num_queries=Tq)
            self.o_layer = torch.empty((Tq, H, d), dtype=bf, device=device)
            self.lse_layer = torch.empty((H, Tq), dtype=torch.float32, device=device)
        # fit: seed + (assign + 7 sort/update kernels) per round, K and V;
        # encode 1; decode 1 (K and V); attention: one launch per block plus
        # the call's own merge when it splits the range; final merge 1
        self.launches_per_step = (2 * (1 + 8 * w.kmeans_iters) + 2 + 2 + 2 * self.blocks + 1
                                  + (joint.launches if joint is not None else 0))

    @property
    def rows(self):
        r = ["fit", "encode", "decode"]
        if self.joint is not None:
            r += ["joint_encode", "joint_decode"]
        return tuple(r + ["attention", "merge"])

    def load_inputs(self, hk, hv, hq):
        self.xk.copy_(hk)
        self.xv.copy_(hv)
        self.q.copy_(hq)

    def outputs(self):
        outs = [self.o, self.lse]
        for i in range(2):
            outs += [self.cent[i], *self.enc[i]]
        if self.joint is not None:
            outs += self.joint.outputs()
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
        if self.joint is not None:
            mark("joint_encode", 0)
            self.joint.encode()
            mark("joint_encode", 1)
            mark("joint_decode", 0)
            self.joint.decode()
            mark("joint_decode", 1)
        mark("attention", 0)
        for b in range(self.blocks):
            K.kvq_attention_lse(self.q, self.comp[0], self.comp[1], self.o_parts[b], self.l_parts[b],
                                t_begin=self.edges[b], t_end=self.edges[b + 1], workspace=self.ws_attn)
        mark("attention", 1)
        mark("merge", 0)
        K.kvq_lse_merge(self.o_parts, self.l_parts, self.o, self.lse)
        mark("merge", 1)

    def attention_block(self, b):
        self.K.kvq_attention_lse(self.q, self.comp[0], self.comp[1], self.o_parts[b], self.l_parts[b],
                                 t_begin=self.edges[b], t_end=self.edges[b + 1], workspace=self.ws_attn)

    def layer_attention(self):
        self.K.kvq_layer_attention(self.q, self.comp[0], self.comp[1], self.kc, self.vc, self.o_layer,
                                   self.lse_layer, self.ws_layer)

    def dense_attention(self):
        self.K.kvq_attention_dense_lse(self.q, self.kc, self.vc, self.o_layer, self.lse_layer,
                                       workspace=self.ws_attn)


def quantwm_rows(p2, steps, warmup, flush, world, device, tfl, hbm):
    """QuantWM's two additions on the Wan-like layer (its K history, after the
    timed steps have fitted and encoded it): the QSAC encode (M = 4, channel
    weights from the chunk's queries) beside the plain encode, the PSAC
    coefficients, and the PSAC attention per history block beside the plain
    one.  Basis U: the 8 leading eigenvectors of the queries' second moments
    (set-up, not timed)."""
    import torch

    K, w = p2.K, p2.w
    T, H, d, Tq = w.history_tokens, w.num_heads, w.head_dim, w.query_tokens
    qf = p2.q.float()
    Mq = torch.einsum("thc,the->hce", qf, qf) / Tq
    wts = torch.diagonal(Mq, dim1=1, dim2=2).contiguous()
    U = torch.linalg.eigh(Mq.double())[1][:, :, -8:].flip(-1).float().contiguous()
    idx, codes, meta = K.alloc_encoded(p2.codec_k, T, device)
    coef = torch.empty((H, T, 8), dtype=torch.float32, device=device)
    qsac_ms = max_over_ranks(time_calls(lambda: K.kvq_encode_qsac(p2.codec_k, p2.xk, p2.cent[0], wts, idx, codes,
                                                                  meta, M=4), steps, warmup, flush), world, device)
    plain_ms = max_over_ranks(time_calls(lambda: K.kvq_encode(p2.codec_k, p2.xk, p2.cent[0], idx, codes, meta),
                                         steps, warmup, flush), world, device)
    coef_ms = max_over_ranks(time_calls(lambda: K.kvq_psac_coefficients(p2.comp[0], p2.xk, U, coef), steps, warmup,
                                        flush), world, device)
    o, lse = p2.o_parts[0], p2.l_parts[0]
    e = p2.edges

    def psac_blocks():
        for b in range(p2.blocks):
            K.kvq_attention_psac_lse(p2.q, p2.comp[0], p2.comp[1], U, coef, o, lse, t_begin=e[b], t_end=e[b + 1],
                                     workspace=p2.ws_attn)

    def plain_blocks():
        for b in range(p2.blocks):
            K.kvq_attention_lse(p2.q, p2.comp[0], p2.comp[1], o, lse, t_begin=e[b], t_end=e[b + 1],
                                workspace=p2.ws_attn)

    psac_ms = max_over_ranks(time_calls(psac_blocks, steps, warmup, flush), world, device)
    base_ms = max_over_ranks(time_calls(plain_blocks, steps, warmup, flush), world, device)
    check_status(K, "after the QuantWM rows")
    flops = 4.0 * Tq * T * d * H
    coef_bytes = T * H * (d * 2 + d * w.bits_k / 8 + (d // w.group_size) * 8 + 2 + 8 * 4)
    return {
        "qsac_encode": {"ms": qsac_ms, "plain_encode_ms": plain_ms, "M": 4,
                        "what": "kvq_encode_qsac of the Wan-like K history (32760 x 12 x 128, C = 256, INT2 "
                                "G = 16): exact weighted distances to every centre on CUDA cores, top-4, "
                                "group-range score"},
        "psac_coefficients": {"ms": coef_ms, "gbs": coef_bytes / (coef_ms / 1e3) / 1e9,
                              "frac": coef_bytes / (coef_ms / 1e3) / 1e9 / hbm,
                              "what": "kvq_psac_coefficients: reads x (bf16) and the compressed K, writes 8 "
                                      "binary32 per token-head"},
        "psac_attention": {"ms": psac_ms, "plain_ms": base_ms, "calls": p2.blocks,
                           "tflops": flops / (psac_ms / 1e3) / 1e12, "frac": flops / (psac_ms / 1e3) / 1e12 / tfl,
                           "what": "kvq_attention_psac_lse over the Wan-like history (2 blocks), beside "
                                   "kvq_attention_lse on the same blocks"},
    }


def stages_rows(p2, steps, warmup, flush, world, device, hbm):
    """The second residual stage on the Wan-like layer (its K and V histories
    and fitted centres): the two-stage encode beside the one-stage encode, and
    the two-stage decode beside the one-stage decode."""
    import torch

    K, w = p2.K, p2.w
    T = w.history_tokens
    codecs = [K.Codec(c.num_heads, c.head_dim, c.num_centroids, c.bits, c.group_size, 0, K.KVQ_META_F32, 2)
              for c in (p2.codec_k, p2.codec_v)]
    enc = []
    for c in codecs:
        idx, codes, meta = K.alloc_encoded(c, T, device)
        enc.append((idx, codes, meta, torch.empty_like(codes), torch.empty_like(meta)))
    xs = (p2.xk, p2.xv)

    def encode2():
        for i in range(2):
            K.kvq_encode_stages(codecs[i], xs[i], p2.cent[i], *enc[i])

    enc_ms = max_over_ranks(time_calls(encode2, steps, warmup, flush), world, device)
    comps = [K.Compressed(codecs[i], T, p2.cent[i], *enc[i][:3], codes2=enc[i][3], meta2=enc[i][4]) for i in range(2)]
    dec_ms = max_over_ranks(time_calls(lambda: [K.kvq_decode(comps[i], p2.dec[i]) for i in range(2)], steps, warmup,
                                       flush), world, device)
    check_status(K, "after the two-stage rows")
    H, d = w.num_heads, w.head_dim
    dec_bytes = sum(T * H * (2 + 2 * (d * c.bits // 8 + 8 * d // c.group_size) + 2 * d) for c in codecs)
    return {"two_stage": {"encode_ms": enc_ms, "decode_ms": dec_ms,
                          "decode_gbs": dec_bytes / (dec_ms / 1e3) / 1e9,
                          "decode_frac": dec_bytes / (dec_ms / 1e3) / 1e9 / hbm,
                          "what": "second residual stage on the Wan-like layer (K and V, INT2 G16 twice): "
                                  "kvq_encode_stages (tensor-core filter) and the two-stage kvq_decode to bf16"}}


def fast_rows(joint, steps, warmup, flush, world, device, tfl, d_low=64):
    """NanoKV-Fast on the joint workload: its K and V joint codes decoded
    straight into a 64-dim space per head (folded analytical maps, set up
    with torch, not timed) and the low-space attention with query reduction
    and output restoration, beside the full-dimensional decode + dense
    attention of the same history."""
    import torch

    from kv_cache_compression_head_b200 import synth

    K, wj = joint.K, joint.w
    T, H, d, Tq, r = wj.history_tokens, wj.num_heads, wj.head_dim, wj.query_tokens, wj.joint_rank
    q = torch.from_numpy(synth.make_queries(wj).view(np.int16)).to(device).view(torch.bfloat16)
    Wf = joint.w_dec.float().view(r, H, d)
    P = torch.stack([torch.linalg.svd(Wf[:, h].double(), full_matrices=True)[2][:d_low].t() for h in range(H)])
    lows, dec_low, dec_full = [], [], []
    for i in range(2):
        Wl = torch.einsum("rhd,hdl->rhl", Wf.double(), P).reshape(r, H * d_low).to(torch.bfloat16).contiguous()
        cl = torch.einsum("hcd,hdl->hcl", joint.cent[i].double(), P).to(torch.bfloat16).contiguous()
        codec = K.Codec(H, d_low, wj.num_centroids, joint.codec[i].bits, wj.joint_group, r)
        lows.append(K.Compressed(codec, T, cl, *joint.enc[i], w_dec=Wl))
        dec_low.append(torch.empty((T, H, d_low), dtype=torch.bfloat16, device=device))
        dec_full.append(torch.empty((T, H, d), dtype=torch.bfloat16, device=device))
    Pb = P.to(torch.bfloat16).contiguous()
    Rb = P.transpose(1, 2).to(torch.bfloat16).contiguous()
    o = torch.empty((Tq, H, d), dtype=torch.float32, device=device)
    lse = torch.empty((H, Tq), dtype=torch.float32, device=device)
    fws = K.fast_attention_workspace(H, d, d_low, Tq, device)
    aws = K.alloc_workspace(K.KVQ_OP_ATTENTION, joint.codec[0], T, device, num_queries=Tq)
    low_dec_ms = max_over_ranks(time_calls(lambda: [K.kvq_decode(lows[i], dec_low[i]) for i in range(2)], steps,
                                           warmup, flush), world, device)
    low_att_ms = max_over_ranks(time_calls(lambda: K.kvq_fast_attention_lse(q, dec_low[0], dec_low[1], Pb, Rb, o, lse,
                                                                            fws), steps, warmup, flush), world, device)
    full_dec_ms = max_over_ranks(time_calls(lambda: [K.kvq_decode(joint.comp[i], dec_full[i]) for i in range(2)],
                                            steps, warmup, flush), world, device)
    full_att_ms = max_over_ranks(time_calls(lambda: K.kvq_attention_dense_lse(q, dec_full[0], dec_full[1], o, lse,
                                                                              workspace=aws), steps, warmup, flush),
                                 world, device)
    check_status(K, "after the NanoKV-Fast rows")
    fl_low = 4.0 * Tq * T * d_low * H
    fl_full = 4.0 * Tq * T * d * H
    return {"nanokv_fast": {
        "d_low": d_low, "decode_ms": low_dec_ms, "attention_ms": low_att_ms,
        "attention_tflops": fl_low / (low_att_ms / 1e3) / 1e12,
        "attention_frac": fl_low / (low_att_ms / 1e3) / 1e12 / tfl,
        "full_decode_ms": full_dec_ms, "full_attention_ms": full_att_ms,
        "full_attention_tflops": fl_full / (full_att_ms / 1e3) / 1e12,
        "history_macs_ratio": d_low / d,
        "what": "joint workload (32760 keys, 12 heads x 128, rank 192, INT4): low-space decode of K and V "
                "(d_low = 64) + kvq_fast_attention_lse, beside the full decode + kvq_attention_dense_lse"}}


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


def check_status(K, when):
    st = K.kvq_last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {when}: {K.status_string(st)}")


def time_steps(pipe, steps, warmup, flush, world, device, sample_clocks=None):
    """Warm-up, then `steps` timed steps between barriers; returns per-row
    mean ms, mean step ms (max over ranks), wall seconds and clocks."""
    import torch

    for _ in range(warmup):
        flush.zero_()
        pipe.step()
    torch.cuda.synchronize()
    check_status(pipe.K, "after warm-up")
    ev = [{r: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for r in pipe.rows}
          for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    if sample_clocks is not None:
        sample_clocks.start()
    t_wall = time.perf_counter()
    for k in range(steps):
        flush.zero_()
        pipe.step(ev[k])
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_wall
    barrier(world)
    clk = sample_clocks.stop() if sample_clocks is not None else None
    check_status(pipe.K, "after timing")
    first, last = pipe.rows[0], pipe.rows[-1]
    row_ms = {r: statistics.mean(e[r][0].elapsed_time(e[r][1]) for e in ev) for r in pipe.rows}
    step_ms = statistics.mean(e[first][0].elapsed_time(e[last][1]) for e in ev)
    return row_ms, max_over_ranks(step_ms, world, device), wall, clk


def time_e2e(pipes, host_inputs, steps, world, device):
    """The step through the public API with pinned host inputs copied in and
    every result copied back inside the timed region, pipelined over two sets
    of device buffers: step k + 1's inputs cross PCIe (one copy stream) and
    step k - 1's results come back (another) while step k computes."""
    import torch

    hk, hv, hq = host_inputs
    outs = [p.outputs() for p in pipes]
    host_outs = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in ob] for ob in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hq))
    d2h = sum(t.numel() * t.element_size() for t in outs[0])
    comp = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in pipes]
    ev_done = [torch.cuda.Event() for _ in pipes]
    ev_out = [torch.cuda.Event() for _ in pipes]

    def one(k):
        b = k % len(pipes)
        p = pipes[b]
        with torch.cuda.stream(h2d_s):
            h2d_s.wait_event(ev_done[b])  # the step that last read these inputs has finished
            p.xk.copy_(hk, non_blocking=True)
            p.xv.copy_(hv, non_blocking=True)
            p.q.copy_(hq, non_blocking=True)
            ev_in[b].record(h2d_s)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])  # this buffer set's previous results are home
        p.step()
        ev_done[b].record(comp)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(ev_done[b])
            for ho, o in zip(host_outs[b], outs[b]):
                ho.copy_(o, non_blocking=True)
            ev_out[b].record(d2h_s)

    for k in range(len(pipes)):  # untimed
        one(k)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d_s)
    for k in range(steps):
        one(k)
    t1.record(d2h_s)
    torch.cuda.synchronize()
    for p in pipes:
        check_status(p.K, "after the end-to-end steps")
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, device)
    return {"value": world * pipes[0].w.history_tokens / (e2e_ms / 1e3), "unit": UNIT, "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "what": "the whole step through the Python binding of the C ABI; every step's history and queries "
                    "cross PCIe in and every result (centres, idx, codes, {s, z}, joint codes, O, LSE) crosses "
                    "back inside the timed region, the copies of neighbouring steps overlapping the compute "
                    "(two sets of device buffers, one stream each way)"}


def row_report(pipe, row_ms, hbm, tfl):
    """Per-row ms and roofline fractions of one workload's step."""
    w = pipe.w
    wm = work_model(w)
    gbps = lambda b, ms: b / (ms / 1e3) / 1e9
    tflops = lambda f, ms: f / (ms / 1e3) / 1e12
    enc_hbm = gbps(wm["encode_bytes"], row_ms["encode"])
    enc_tc = tflops(wm["encode_flops"], row_ms["encode"])
    attn = tflops(wm["attention_flops"], row_ms["attention"])
    enc_hbm_roof_ms = wm["encode_bytes"] / (hbm * 1e9) * 1e3
    enc_tc_roof_ms = wm["encode_flops"] / (tfl * 1e12) * 1e3
    rows = {
        "fit": {"ms": row_ms["fit"], "gbps": gbps(wm["fit_bytes"], row_ms["fit"]),
                "hbm_frac": gbps(wm["fit_bytes"], row_ms["fit"]) / hbm},
        "encode": {"ms": row_ms["encode"], "tokens_per_s": w.history_tokens / (row_ms["encode"] / 1e3),
                   "gbps": enc_hbm, "hbm_frac": enc_hbm / hbm,
                   "filter_tflops": enc_tc, "tensor_frac": enc_tc / tfl,
                   "binding_roof": "tensor" if enc_tc_roof_ms > enc_hbm_roof_ms else "hbm",
                   "roof_ms": max(enc_tc_roof_ms, enc_hbm_roof_ms),
                   "roof_frac": max(enc_tc_roof_ms, enc_hbm_roof_ms) / row_ms["encode"]},
        "decode": {"ms": row_ms["decode"], "gbps": gbps(wm["decode_bytes"], row_ms["decode"]),
                   "hbm_frac": gbps(wm["decode_bytes"], row_ms["decode"]) / hbm},
        "attention": {"ms": row_ms["attention"], "launches": pipe.blocks, "tflops": attn, "frac": attn / tfl},
        "merge": {"ms": row_ms["merge"], "gbps": gbps(wm["merge_bytes"], row_ms["merge"]),
                  "hbm_frac": gbps(wm["merge_bytes"], row_ms["merge"]) / hbm},
    }
    if pipe.joint is not None:
        jm = joint_work_model(pipe.joint.w)
        je, jd = row_ms["joint_encode"], row_ms["joint_decode"]
        rows["joint_encode"] = {"ms": je, "gbps": gbps(jm["joint_enc_bytes"], je),
                                "hbm_frac": gbps(jm["joint_enc_bytes"], je) / hbm,
                                "tflops": tflops(jm["joint_gemm_flops"] / 2 + jm["joint_filter_flops"], je),
                                "tensor_frac": tflops(jm["joint_gemm_flops"] / 2 + jm["joint_filter_flops"], je) / tfl,
                                "workload": "joint (12 heads, 32,760 tokens, rank 192, K4V4, G 32)"}
        rows["joint_decode"] = {"ms": jd, "gbps": gbps(jm["joint_dec_bytes"], jd),
                                "hbm_frac": gbps(jm["joint_dec_bytes"], jd) / hbm,
                                "gemm_tflops": tflops(jm["joint_gemm_flops"] / 2, jd),
                                "workload": "joint (12 heads, 32,760 tokens, rank 192, K4V4, G 32)"}
    return rows


def workload_config(w, world, extra=""):
    return {"workload": f"{w.name}-like layer: {w.num_heads} heads x {w.head_dim}, history {w.history_tokens} "
                        f"tokens ({w.frames} frames x {w.tokens_per_frame}), query chunk {w.query_tokens}, "
                        f"C={w.num_centroids}, K{w.bits_k}V{w.bits_v}, group {w.group_size}, fit "
                        f"{w.kmeans_iters} rounds, {max(w.history_blocks, 2)} history blocks{extra}",
            "history_tokens": w.history_tokens, "query_tokens": w.query_tokens, "heads": w.num_heads,
            "head_dim": w.head_dim, "centroids": w.num_centroids, "bits_k": w.bits_k, "bits_v": w.bits_v,
            "group": w.group_size, "history_blocks": max(w.history_blocks, 2),
            "parallelism": f"replicas x{world}", "l2": "flushed (256 MiB write) before each step"}


def run_gpu(args):
    import torch

    from kv_cache_compression_head_b200 import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    hbm, tfl, peak_kind = measured_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    # ---- headline: the 14B-like layer, with the joint rows on their workload
    w = synth.workload(args.workload)
    hk, hv, hq = (pinned_bf16(synth.make_history(w, "K")), pinned_bf16(synth.make_history(w, "V")),
                  pinned_bf16(synth.make_queries(w)))
    joint = JointRows(device)
    pipe = Pipeline(w, device, joint=joint)
    pipe.load_inputs(hk, hv, hq)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    row_ms, ms_step, wall, clk = time_steps(pipe, args.steps, args.warmup, flush, world, device, clocks)
    rows = row_report(pipe, row_ms, hbm, tfl)
    # the attention launches of one step, one block per call: mean time per call
    attn_call_ms = max_over_ranks(
        statistics.mean(time_calls(lambda b=b: pipe.attention_block(b), max(3, args.steps // 4), 1, flush)
                        for b in range(pipe.blocks)), world, device)
    e2e = None
    if not args.no_e2e:
        pipe2 = Pipeline(w, device, joint=JointRows(device))
        e2e = time_e2e([pipe, pipe2], (hk, hv, hq), args.steps, world, device)
        del pipe2
    launches = pipe.launches_per_step * args.steps
    del pipe, hk, hv, hq
    torch.cuda.empty_cache()

    # ---- the Wan-1.3B-like step, then its chunk's full-layer attention
    secondary = None
    next_rows = None
    if not args.no_secondary:
        w2 = synth.workload(SECONDARY)
        p2 = Pipeline(w2, device, layer=True)
        p2.load_inputs(pinned_bf16(synth.make_history(w2, "K")), pinned_bf16(synth.make_history(w2, "V")),
                       pinned_bf16(synth.make_queries(w2)))
        p2.kc.copy_(pinned_bf16(synth.make_chunk(w2, "K")))
        p2.vc.copy_(pinned_bf16(synth.make_chunk(w2, "V")))
        torch.cuda.synchronize()
        r2, ms2, _, _ = time_steps(p2, args.steps, args.warmup, flush, world, device)
        secondary = {"value": world * w2.history_tokens / (ms2 / 1e3), "unit": UNIT, "ms_per_step": ms2,
                     "config": workload_config(w2, world), "rows": row_report(p2, r2, hbm, tfl)}
        layer_ms = max_over_ranks(time_calls(p2.layer_attention, args.steps, args.warmup, flush), world, device)
        dense_ms = max_over_ranks(time_calls(p2.dense_attention, args.steps, args.warmup, flush), world, device)
        check_status(p2.K, "after the layer attention")
        Tq, H, d = w2.query_tokens, w2.num_heads, w2.head_dim
        layer_flops = 4.0 * Tq * (w2.history_tokens + Tq) * d * H
        dense_flops = 4.0 * Tq * Tq * d * H
        next_rows = {
            "layer_attention": {"ms": layer_ms, "calls": 1, "keys": w2.history_tokens + Tq,
                                "tflops": layer_flops / (layer_ms / 1e3) / 1e12,
                                "frac": layer_flops / (layer_ms / 1e3) / 1e12 / tfl,
                                "what": "kvq_layer_attention on the Wan-like layer: 32760 compressed history "
                                        "keys + the 4680-key chunk (bf16), one softmax, LSE merge in the call"},
            "dense_attention": {"ms": dense_ms, "calls": 1, "keys": Tq,
                                "tflops": dense_flops / (dense_ms / 1e3) / 1e12,
                                "frac": dense_flops / (dense_ms / 1e3) / 1e12 / tfl,
                                "what": "kvq_attention_dense_lse over the Wan-like 4680-key chunk alone"},
        }
        next_rows.update(quantwm_rows(p2, args.steps, args.warmup, flush, world, device, tfl, hbm))
        next_rows.update(fast_rows(joint, args.steps, args.warmup, flush, world, device, tfl))
        next_rows.update(stages_rows(p2, args.steps, args.warmup, flush, world, device, hbm))
        launches += p2.launches_per_step * args.steps
        del p2
        torch.cuda.empty_cache()

    if rank == 0:
        wm = work_model(w)
        attn_tflops = wm["attention_flops"] / pipe_blocks(w) / (attn_call_ms / 1e3) / 1e12
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
            "config": workload_config(w, world, extra="; the step also runs the joint head-channel code "
                                                      "(rank 192, K4V4, group 32) of the joint workload's "
                                                      "32,760-token, 12-head history"),
            "roofline": {"kernel": "compressed-history attention, one kvq_attention_lse call per history block "
                                   "(11,700 keys; incl. the call's own LSE merge of its sub-ranges)",
                         "bound": "tensor", "achieved": attn_tflops, "peak": tfl, "unit": "TFLOP/s",
                         "frac": attn_tflops / tfl, "peak_kind": f"{peak_kind} (bf16 dense, burst)",
                         "traffic": ATTN_NCU_TRAFFIC_BYTES,
                         "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
                         "traffic_before_change": ATTN_NCU_TRAFFIC_BEFORE_CHANGE,
                         "traffic_note": "captured before the give-up changes (wait limit read from constant "
                                         "memory, drain after a give-up); not re-captured since",
                         "ms_per_launch": attn_call_ms},
            "rows": rows,
            "config2": secondary,
            "next_rows": next_rows,
            "clocks": clk,
            "gpu_launches": launches,
            "wall_s_timed_region": wall,
            "e2e": e2e,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    barrier(world)


def pipe_blocks(w):
    return w.history_blocks if w.history_blocks > 1 else 2


# ----------------------------------------------------------------------------
# sweep: encode, decode and attention per point (covering set)
# ----------------------------------------------------------------------------

def sweep_points():
    """A covering set of the 12-head sweep: every (b_K, b_V), every G, every
    C and every T of 4k-128k appear; both query-chunk lengths appear."""
    Ts = [4096, 8192, 16384, 32768, 65536, 131072]
    pts = []
    combos = [(2, 2, 16, 64), (2, 4, 32, 256), (4, 2, 64, 1024), (4, 4, 16, 256), (2, 2, 64, 256),
              (4, 4, 32, 64)]
    for i, T in enumerate(Ts):
        bk, bv, G, C = combos[i % len(combos)]
        pts.append((T, 4680 if i % 2 == 0 else 1560, bk, bv, G, C))
    pts.append((131072, 4680, 2, 2, 16, 1024))
    pts.append((4096, 1560, 4, 4, 64, 1024))
    return pts


def run_sweep(args):
    import torch

    from kv_cache_compression_head_b200 import kvq as K
    from kv_cache_compression_head_b200 import synth

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    hbm, tfl, _ = measured_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    base = synth.sweep_point(131072, 4680, 2, 2, 16, 256)
    full_k = to_device_bf16(synth.make_history(base, "K"), device)
    full_v = to_device_bf16(synth.make_history(base, "V"), device)
    full_q = to_device_bf16(synth.make_queries(base), device)
    with open(args.sweep, "w") as out:
        for (T, Tq, bk, bv, G, C) in sweep_points():
            w = synth.sweep_point(T, Tq, bk, bv, G, C)
            H, d = w.num_heads, w.head_dim
            xk, xv, q = full_k[:T].contiguous(), full_v[:T].contiguous(), full_q[:Tq].contiguous()
            ck, cv = K.Codec(H, d, C, bk, G), K.Codec(H, d, C, bv, G)
            cent = [torch.empty((H, C, d), dtype=torch.bfloat16, device=device) for _ in range(2)]
            ws = K.alloc_workspace(K.KVQ_OP_FIT, ck, T, device)
            K.kvq_fit_centroids(ck, xk, 2, cent[0], ws)
            K.kvq_fit_centroids(cv, xv, 2, cent[1], ws)
            enc = [K.alloc_encoded(c, T, device) for c in (ck, cv)]
            comp = [K.Compressed(c, T, cent[i], *enc[i]) for i, c in enumerate((ck, cv))]
            dec = torch.empty((T, H, d), dtype=torch.bfloat16, device=device)
            o = torch.empty((Tq, H, d), dtype=torch.float32, device=device)
            lse = torch.empty((H, Tq), dtype=torch.float32, device=device)
            ws_a = K.alloc_workspace(K.KVQ_OP_ATTENTION, ck, T, device, num_queries=Tq)

            def encode():
                K.kvq_encode(ck, xk, cent[0], *enc[0])
                K.kvq_encode(cv, xv, cent[1], *enc[1])

            def decode():
                K.kvq_decode(comp[0], dec)
                K.kvq_decode(comp[1], dec)

            def attention():
                K.kvq_attention_lse(q, comp[0], comp[1], o, lse, workspace=ws_a)

            reps = 10
            enc_ms = time_calls(encode, reps, 3, flush)
            dec_ms = time_calls(decode, reps, 3, flush)
            att_ms = time_calls(attention, reps, 3, flush)
            check_status(K, f"after sweep point {w.name}")
            wm = work_model(w)
            rec = {"point": {"T": T, "Tq": Tq, "bits_k": bk, "bits_v": bv, "group": G, "centroids": C},
                   "encode_ms": enc_ms, "encode_gbps": wm["encode_bytes"] / enc_ms / 1e6,
                   "encode_hbm_frac": wm["encode_bytes"] / enc_ms / 1e6 / hbm,
                   "encode_filter_tflops": wm["encode_flops"] / enc_ms / 1e9,
                   "decode_ms": dec_ms, "decode_gbps": wm["decode_bytes"] / dec_ms / 1e6,
                   "decode_hbm_frac": wm["decode_bytes"] / dec_ms / 1e6 / hbm,
                   "attention_ms": att_ms, "attention_tflops": wm["attention_flops"] / att_ms / 1e9,
                   "attention_frac": wm["attention_flops"] / att_ms / 1e9 / tfl}
            out.write(json.dumps(rec) + "\n")
            out.flush()
            print(json.dumps(rec), flush=True)
            del xk, xv, q, cent, ws, enc, comp, dec, o, lse, ws_a
            torch.cuda.empty_cache()


# ----------------------------------------------------------------------------
# CPU oracle: baseline leg and reference arm
# ----------------------------------------------------------------------------

CPU_SAMPLE_T = 2048
CPU_SAMPLE_TQ = 256
CPU_REPEATS = 3


def oracle_step_times(w):
    """Time the oracle on a bounded sample of the workload: fit+encode+decode
    of the first CPU_SAMPLE_T history tokens (all heads, K and V) and attention
    over the same number of blocks + merge of CPU_SAMPLE_TQ queries over them.
    Returns (wall seconds of the sample, its extrapolation to one full step)."""
    from kv_cache_compression_head_b200 import synth
    from oracle import oracle as O

    Ts, Tqs = min(CPU_SAMPLE_T, w.history_tokens), min(CPU_SAMPLE_TQ, w.query_tokens)
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
    nb = pipe_blocks(w)
    edges = [Ts * i // nb for i in range(nb + 1)]
    parts = [O.attention(q, decs[0][a:b], decs[1][a:b]) for a, b in zip(edges[:-1], edges[1:])]
    O.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    t2 = time.perf_counter()
    codec_s, attn_s = t1 - t0, t2 - t1
    full = codec_s * (w.history_tokens / Ts) + attn_s * (w.history_tokens * w.query_tokens) / (Ts * Tqs)
    return t2 - t0, full


def _omp_threads():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def _sample_text(w):
    return (f"fit+encode+decode of {min(CPU_SAMPLE_T, w.history_tokens)}/{w.history_tokens} history tokens "
            f"({w.num_heads} heads, K and V, C={w.num_centroids}) and attention ({pipe_blocks(w)} blocks)+merge "
            f"of {min(CPU_SAMPLE_TQ, w.query_tokens)}/{w.query_tokens} queries over them; scaled per history "
            f"token and per query x history token to the full step")


def cpu_baseline(w):
    runs = [oracle_step_times(w) for _ in range(CPU_REPEATS)]
    rates = sorted(w.history_tokens / full for _, full in runs)
    return {"value": statistics.median(rates), "unit": UNIT, "cores": _omp_threads(), "kind": "oracle",
            "repeats": CPU_REPEATS, "min": rates[0], "max": rates[-1],
            "spread": (rates[-1] - rates[0]) / statistics.median(rates),
            "sample": _sample_text(w), "sample_s": statistics.median(s for s, _ in runs)}


def run_reference(args):
    """The CPU oracle as the reference arm: rank 0 alone runs and prints; any
    other rank exits at once without work (and without joining a group)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from kv_cache_compression_head_b200 import synth

    w = synth.workload(HEADLINE)
    for _ in range(args.warmup):
        oracle_step_times(w)
    samples, fulls = [], []
    t_wall = time.perf_counter()
    for _ in range(args.steps):
        s, full = oracle_step_times(w)
        samples.append(s)
        fulls.append(full)
    wall = time.perf_counter() - t_wall
    value = w.history_tokens / statistics.median(fulls)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (CPU oracle)",
        "data": "synthetic",
        "config": {**workload_config(w, world), "parallelism": "rank 0 only",
                   "sample": "each step runs the bounded sample below; value is the full step's rate "
                             "extrapolated from it"},
        "extrapolated_ms_per_full_step": statistics.median(fulls) * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _omp_threads(), "kind": "oracle",
                         "sample": _sample_text(w)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s_timed_region": wall,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.warmup < 0 or args.steps < 1:
        raise SystemExit("need --steps >= 1 and --warmup >= 0")
    if args.sweep:
        run_sweep(args)
        return
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
