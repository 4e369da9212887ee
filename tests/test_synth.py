"""The seeded input recipe (CPU only): shapes and dtypes of every workload,
determinism, the frame-major continuation of the K/V streams (a truncated
history is the prefix of the full one; the current chunk is the next frames
of the same stream), and the orthonormal joint encoder."""

import dataclasses

import numpy as np
import pytest

from kv_cache_compression_head_b200 import synth


@pytest.mark.parametrize("name", ["tiny", "wan13b"])
def test_shapes_dtypes_and_determinism(name):
    w = synth.workload(name)
    x = synth.make_history(w, "K", max_tokens=300)
    q = synth.make_queries(w, max_tokens=50)
    c = synth.make_chunk(w, "V", max_tokens=70)
    want = np.float32 if w.dtype == "f32" else np.uint16
    assert x.shape == (300, w.num_heads, w.head_dim) and x.dtype == want
    assert q.shape == (50, w.num_heads, w.head_dim) and q.dtype == np.uint16
    assert c.shape == (70, w.num_heads, w.head_dim) and c.dtype == want
    assert np.array_equal(x, synth.make_history(w, "K", max_tokens=300))
    assert not np.array_equal(x[:70], synth.make_history(w, "V", max_tokens=70))


def test_chunk_continues_the_history_stream():
    """The chunk of a history of F frames is frames F .. of the same stream:
    it equals the matching slice of a longer history."""
    for name, frames in (("tiny", 2), ("wan13b", 3)):
        w = synth.workload(name)
        short = dataclasses.replace(w, frames=frames)
        longer = dataclasses.replace(w, frames=frames + -(-w.query_tokens // w.tokens_per_frame))
        T = short.history_tokens
        for which in ("K", "V"):
            chunk = synth.make_chunk(short, which)
            hist = synth.make_history(longer, which)
            assert np.array_equal(chunk, hist[T:T + w.query_tokens]), (name, which)
            assert np.array_equal(synth.make_history(short, which), hist[:T])


def test_outlier_channels_are_heavy():
    """Four channels per head carry x8 outliers in the AR(1) workloads."""
    w = synth.workload("wan13b")
    x = synth.bf16_bits_to_f32(synth.make_history(w, "K", max_tokens=3120)).astype(np.float64)
    rms = np.sqrt((x ** 2).mean(axis=0))             # [H][d]
    top = np.sort(rms, axis=1)[:, -w.outlier_channels:]
    rest = np.sort(rms, axis=1)[:, :-w.outlier_channels]
    assert np.all(top.min(axis=1) > 4 * rest.max(axis=1))


def test_orthonormal_encoder():
    w = synth.workload("joint")
    e = synth.bf16_bits_to_f32(synth.make_orthonormal_encoder(w)).astype(np.float64)
    assert e.shape == (w.num_heads * w.head_dim, w.joint_rank)
    g = e.T @ e
    # orthonormal columns up to the bf16 rounding of each entry
    assert np.max(np.abs(g - np.eye(w.joint_rank))) < 2e-2
