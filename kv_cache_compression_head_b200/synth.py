"""Seeded synthetic KV-cache workloads shaped like the pages' video models.

This module only draws random numbers and lays them out; it holds none of the
compression method's arithmetic.  Both the CUDA path's tests/bench and the CPU
oracle take their inputs from here, so the two sides see identical bytes.

Shapes follow the pages' workloads:

* 1,560 tokens per latent frame = a 30 x 52 latent grid at 832 x 480
  (TempoKV: Predictive KV Cache Quantization for Autoregressive Video
  Generation, Sec. 4.1); 12 heads x 128 for the Wan-1.3B class; 40 heads x 128
  for the 14B-class layer (NanoKV page, Table 9).
* Token index t = frame * S + spatial position (frame-major), the layout in
  which a cache block is filled one chunk at a time.

Random streams use NumPy PCG64 with seed ``1000 * config + {0: K, 1: V, 2: Q}``.
Values are drawn in float64 and rounded once to the workload dtype (bf16 with
round-to-nearest-even via torch, or float32 for the tiny config).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "make_history",
    "make_queries",
    "make_chunk",
    "make_orthonormal_encoder",
    "bf16_bits_from_f64",
    "bf16_bits_to_f32",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: history/query shapes plus the codec settings."""

    name: str
    config_id: int
    num_heads: int
    head_dim: int
    frames: int
    tokens_per_frame: int
    query_tokens: int
    dtype: str  # "f32" or "bf16"
    num_centroids: int
    kmeans_iters: int
    bits_k: int
    bits_v: int
    group_size: int
    generator: str  # "smooth" or "ar1"
    outlier_channels: int
    joint_rank: int = 0
    joint_group: int = 32
    history_blocks: int = 1

    @property
    def history_tokens(self) -> int:
        return self.frames * self.tokens_per_frame


WORKLOADS = {
    "tiny": Workload(
        name="tiny", config_id=1, num_heads=2, head_dim=64, frames=4,
        tokens_per_frame=256, query_tokens=256, dtype="f32", num_centroids=16,
        kmeans_iters=5, bits_k=2, bits_v=2, group_size=32, generator="smooth",
        outlier_channels=2),
    "wan13b": Workload(
        name="wan13b", config_id=2, num_heads=12, head_dim=128, frames=21,
        tokens_per_frame=1560, query_tokens=4680, dtype="bf16", num_centroids=256,
        kmeans_iters=2, bits_k=2, bits_v=2, group_size=16, generator="ar1",
        outlier_channels=4),
    "joint": Workload(
        name="joint", config_id=3, num_heads=12, head_dim=128, frames=21,
        tokens_per_frame=1560, query_tokens=4680, dtype="bf16", num_centroids=256,
        kmeans_iters=2, bits_k=4, bits_v=4, group_size=32, generator="ar1",
        outlier_channels=4, joint_rank=192, joint_group=32),
    "14b": Workload(
        name="14b", config_id=4, num_heads=40, head_dim=128, frames=60,
        tokens_per_frame=1560, query_tokens=4680, dtype="bf16", num_centroids=512,
        kmeans_iters=2, bits_k=4, bits_v=2, group_size=32, generator="ar1",
        outlier_channels=4, history_blocks=8),
}


def workload(name: str, **overrides) -> Workload:
    """Return a named workload, optionally with fields replaced (sweep points)."""
    w = WORKLOADS[name]
    return dataclasses.replace(w, **overrides) if overrides else w


def sweep_point(history_tokens: int, query_tokens: int, bits_k: int, bits_v: int,
                group_size: int, num_centroids: int) -> Workload:
    """A point of the 12-head sweep: 4k-128k history, AR(1)+outlier generator.

    The sweep's history lengths are powers of two, not whole frames, so the
    point is described as one frame of ``history_tokens`` tokens for shape
    purposes while the AR(1) process still steps every 1,560 tokens.
    """
    return Workload(
        name=f"sweep_T{history_tokens}_Q{query_tokens}_k{bits_k}v{bits_v}_G{group_size}_C{num_centroids}",
        config_id=5, num_heads=12, head_dim=128, frames=1,
        tokens_per_frame=history_tokens, query_tokens=query_tokens, dtype="bf16",
        num_centroids=num_centroids, kmeans_iters=2, bits_k=bits_k, bits_v=bits_v,
        group_size=group_size, generator="ar1", outlier_channels=4)


# ----------------------------------------------------------------------------
# bf16 helpers (storage only: bit patterns in uint16)
# ----------------------------------------------------------------------------

def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest-even, via float32 first) and
    return the raw 16-bit patterns.  Uses torch's conversion so no rounding
    code of our own is involved in input preparation."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def _seed(w: Workload, stream: int) -> int:
    return 1000 * w.config_id + stream


def _outlier_channels(rng: np.random.Generator, H: int, d: int, n: int) -> np.ndarray:
    """n distinct channel indices per head, [H][n]."""
    return np.stack([rng.choice(d, size=n, replace=False) for _ in range(H)])


def _smooth_frames(w: Workload, rng: np.random.Generator, with_outliers: bool):
    """Tiny config: per-frame smooth spatial base + N(0, 0.1^2) noise.

    base_f[s,h,c] = a_hc * sin(2 pi (u_s alpha_hc + v_s beta_hc) + phi_fhc) on a
    square spatial grid, with a ~ U(0.5,1.5), alpha, beta ~ U(0,2) and a fresh
    phase phi ~ U(0, 2 pi) per frame.  Outlier channels are multiplied by 8.
    """
    H, d, S = w.num_heads, w.head_dim, w.tokens_per_frame
    side = int(round(math.sqrt(S)))
    assert side * side == S, "smooth generator wants a square spatial grid"
    gu, gv = np.meshgrid(np.arange(side) / side, np.arange(side) / side, indexing="ij")
    u = gu.reshape(S)[:, None, None]
    v = gv.reshape(S)[:, None, None]
    a = rng.uniform(0.5, 1.5, size=(1, H, d))
    alpha = rng.uniform(0.0, 2.0, size=(1, H, d))
    beta = rng.uniform(0.0, 2.0, size=(1, H, d))
    out_ch = _outlier_channels(rng, H, d, w.outlier_channels) if with_outliers else None
    for _f in range(w.frames):
        phi = rng.uniform(0.0, 2.0 * math.pi, size=(1, H, d))
        base = a * np.sin(2.0 * math.pi * (u * alpha + v * beta) + phi)
        x = base + rng.normal(0.0, 0.1, size=(S, H, d))
        if out_ch is not None:
            for h in range(H):
                x[:, h, out_ch[h]] *= 8.0
        yield x


def _ar1_frames(w: Workload, rng: np.random.Generator, with_outliers: bool,
                frames: int, tokens_per_frame: int):
    """AR(1) over frames at each (spatial position, head, channel):
    X_0 ~ N(0,1), X_f = 0.9 X_{f-1} + sqrt(1 - 0.81) N(0,1); observed value
    X_f + N(0, 0.1^2).  Outlier channels: value * 8 + Student-t(3) noise.
    """
    H, d, S = w.num_heads, w.head_dim, tokens_per_frame
    rho = 0.9
    innov = math.sqrt(1.0 - rho * rho)
    out_ch = _outlier_channels(rng, H, d, w.outlier_channels) if with_outliers else None
    state = rng.standard_normal(size=(S, H, d))
    for f in range(frames):
        if f > 0:
            state = rho * state + innov * rng.standard_normal(size=(S, H, d))
        x = state + rng.normal(0.0, 0.1, size=(S, H, d))
        if out_ch is not None:
            for h in range(H):
                x[:, h, out_ch[h]] = x[:, h, out_ch[h]] * 8.0 + rng.standard_t(3.0, size=(S, w.outlier_channels))
        yield x


def _frames_for(w: Workload, stream: int, tokens: int, with_outliers: bool):
    rng = np.random.Generator(np.random.PCG64(_seed(w, stream)))
    if w.generator == "smooth":
        assert tokens == w.frames * w.tokens_per_frame or stream == 2
        ww = w if stream != 2 else dataclasses.replace(
            w, frames=max(1, tokens // w.tokens_per_frame))
        yield from _smooth_frames(ww, rng, with_outliers)
        return
    # AR(1): the process steps every 1,560 tokens (one latent frame); the last
    # frame is cut to length for sweep points that are not whole frames.
    S = 1560 if w.config_id == 5 else w.tokens_per_frame
    S = min(S, tokens)
    nframes = -(-tokens // S)
    yield from _ar1_frames(w, rng, with_outliers, nframes, S)


def _collect(w: Workload, frames, tokens: int, H: int, d: int, max_tokens: Optional[int]):
    n = tokens if max_tokens is None else min(tokens, max_tokens)
    if w.dtype == "f32":
        out = np.empty((n, H, d), dtype=np.float32)
    else:
        out = np.empty((n, H, d), dtype=np.uint16)
    pos = 0
    for x in frames:
        if pos >= n:
            break
        take = min(x.shape[0], n - pos)
        chunk = x[:take]
        out[pos:pos + take] = chunk.astype(np.float32) if w.dtype == "f32" else bf16_bits_from_f64(chunk)
        pos += take
    assert pos == n
    return out


def make_history(w: Workload, which: str, max_tokens: Optional[int] = None) -> np.ndarray:
    """History keys ('K') or values ('V') as [T][H][d].

    Returns float32 for f32 workloads, else uint16 bf16 bit patterns.
    ``max_tokens`` truncates the frame-major token axis (a prefix of the same
    stream, so a truncated history is the start of the full one).
    """
    stream = {"K": 0, "V": 1}[which]
    T = w.history_tokens
    return _collect(w, _frames_for(w, stream, T, True), T, w.num_heads, w.head_dim, max_tokens)


def make_queries(w: Workload, max_tokens: Optional[int] = None) -> np.ndarray:
    """Current-chunk queries [Tq][H][d] (bf16 bits; float32 rounded to bf16 for
    the tiny config, since the attention consumes bf16 queries).

    Queries come from the same family of generator without outlier channels,
    so that logits have a moderate spread (std ~1.7 at d=128)."""
    Tq = w.query_tokens
    frames = _frames_for(w, 2, Tq, False)
    ww = dataclasses.replace(w, dtype="bf16")
    return _collect(ww, frames, Tq, w.num_heads, w.head_dim, max_tokens)


def make_chunk(w: Workload, which: str, max_tokens: Optional[int] = None) -> np.ndarray:
    """The current chunk's own keys ('K') or values ('V'), [Tq][H][d]: the
    Tq tokens that follow the history in the same random stream (the next
    frames of the same process), uncompressed, in the workload dtype."""
    stream = {"K": 0, "V": 1}[which]
    T, Tq = w.history_tokens, w.query_tokens
    if w.generator == "smooth":
        ww = dataclasses.replace(w, frames=w.frames + -(-Tq // w.tokens_per_frame))
        frames = _frames_for(ww, stream, ww.history_tokens, True)
    else:
        frames = _frames_for(w, stream, T + Tq, True)
    out = _collect(w, frames, T + Tq, w.num_heads, w.head_dim, None)[T:]
    return np.ascontiguousarray(out if max_tokens is None else out[:max_tokens])


def make_orthonormal_encoder(w: Workload, seed_stream: int = 3) -> np.ndarray:
    """Joint head-channel encoder W_enc [H*d][r] with orthonormal columns:
    QR of a seeded N(0,1) (H*d) x r matrix in float64, then rounded to bf16.
    Returned as uint16 bf16 bits.  The decoder used with it is its transpose."""
    n = w.num_heads * w.head_dim
    r = w.joint_rank
    rng = np.random.Generator(np.random.PCG64(_seed(w, seed_stream)))
    g = rng.standard_normal(size=(n, r))
    qm, rm = np.linalg.qr(g)
    qm = qm * np.sign(np.diag(rm))[None, :]
    return bf16_bits_from_f64(qm)
