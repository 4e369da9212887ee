"""GPU parity of the compact 16-bit {s, z} format (TempoKV, Table 1: b + 1
bits per value at G = 32) against the oracle's encode16 / decode16: centre
indices, codes and the binary16 {s, z} bits bit-exact (both the tensor-core
filter encode for bf16 histories and the exact CUDA-core encode for float32
ones), the binary32 reconstruction bit-exact, and the attention over the
compressed history within the attention tolerances."""

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_attention_close, bits_u16, f32_bits, to_dev, u8

pytestmark = pytest.mark.gpu


def _K():
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _encode16(codec, x_np, cent_np):
    K = _K()
    T = x_np.shape[0]
    cent = to_dev(cent_np)
    idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
    K.kvq_encode(codec, to_dev(x_np), cent, idx, codes, meta)
    return K.Compressed(codec, T, cent, idx, codes, meta)


def _check_encoded(comp, H, T, d, bits, G, ref):
    idx_r, codes_r, meta_r = ref
    assert np.array_equal(bits_u16(comp.idx).reshape(H, T), idx_r)
    assert np.array_equal(u8(comp.codes).reshape(H, T, d * bits // 8), codes_r)
    got = comp.meta.cpu().view(torch.int16).numpy().view(np.uint16).reshape(H, T, d // G, 2)
    assert np.array_equal(got, meta_r), f"meta16 mismatch at {np.argwhere(got != meta_r)[:5]}"


@pytest.mark.parametrize("name,T,bits_k,bits_v,G,C", [
    ("wan13b", 4000, 2, 2, 16, 256),
    ("14b", 3000, 4, 2, 32, 512),
    ("wan13b", 1027, 4, 4, 64, 64),
    ("14b", 700, 2, 4, 16, 1024),   # C > 512: the exact CUDA-core encode
])
def test_compact_encode_decode_attention(name, T, bits_k, bits_v, G, C):
    K = _K()
    w = synth.workload(name)
    H, d = min(w.num_heads, 6), w.head_dim
    xk = np.ascontiguousarray(synth.make_history(w, "K", max_tokens=T)[:, :H])
    xv = np.ascontiguousarray(synth.make_history(w, "V", max_tokens=T)[:, :H])
    q = np.ascontiguousarray(synth.make_queries(w, max_tokens=600)[:, :H])
    comps, decs = [], []
    for x, bits in ((xk, bits_k), (xv, bits_v)):
        cent = O.fit(x[:C], C, 0) if T >= C else O.fit(x, T, 0)
        Cc = cent.shape[1]
        codec = K.Codec(H, d, Cc, bits, G, 0, K.KVQ_META_F16)
        ref = O.encode16(x, cent, bits, G)
        comp = _encode16(codec, x, cent)
        _check_encoded(comp, H, T, d, bits, G, ref)
        dref = O.decode16(*ref, cent, bits, G)
        dec = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, dec)
        assert np.array_equal(f32_bits(dec), f32_bits(dref)), "decode16 differs"
        comps.append(comp)
        decs.append(dref)
    o = torch.empty((q.shape[0], H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=q.shape[0])
    K.kvq_attention_lse(to_dev(q), comps[0], comps[1], o, lse, workspace=ws)
    o_ref, lse_ref = O.attention(q, decs[0], decs[1])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"compact {name}")
    # a ragged sub-range
    t0, t1 = T // 5, T - T // 7
    K.kvq_attention_lse(to_dev(q), comps[0], comps[1], o, lse, t_begin=t0, t_end=t1)
    o_ref, lse_ref = O.attention(q, decs[0][t0:t1], decs[1][t0:t1])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"compact {name} range")
    assert K.kvq_last_device_status() == K.KVQ_OK


def test_compact_float32_history_and_degenerate_groups():
    """A float32 history (exact CUDA-core encode) with constant and zero groups
    and a group whose scale underflows binary16."""
    K = _K()
    rng = np.random.default_rng(71)
    T, H, d, C = 300, 2, 128, 16
    x = (rng.normal(size=(T, H, d)) * rng.uniform(0.1, 4, size=(1, H, d))).astype(np.float32)
    x[:50, :, :32] = 0.25           # constant channels
    x[50:100, :, 32:64] = 0.0
    x[100:120, :, 64:80] = np.float32(2.0 ** -28) * rng.integers(0, 3, size=(20, H, 16))
    cent = O.fit(x, C, 1)
    for bits, G in ((2, 16), (4, 32)):
        codec = K.Codec(H, d, C, bits, G, 0, K.KVQ_META_F16)
        ref = O.encode16(x, cent, bits, G)
        comp = _encode16(codec, x, cent)
        _check_encoded(comp, H, T, d, bits, G, ref)
        dec = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, dec)
        assert np.array_equal(f32_bits(dec), f32_bits(O.decode16(*ref, cent, bits, G)))
    assert K.kvq_last_device_status() == K.KVQ_OK
