"""GPU parity of the second residual stage (the reading of QVG's progressive
residual quantisation, named by TempoKV Sec. 2) against the oracle's encode2 /
decode2: centre indices, both stages' codes and {s, z} bit-exact, the binary32
two-stage reconstruction bit-exact and its bf16 output the round-to-nearest-
even of it; bf16 and float32 histories, d = 64 and 128, both code widths,
every group size; a ragged token count; the whole Wan-like K history.  bf16
histories with C <= 512 run on the tensor-core filter, the others on the
exact CUDA-core kernel; the cases cover both, and one history is run through
both (bf16 and its exact float32 widening) with identical outputs."""

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O
from tests.gpu_util import bits_u16, f32_bits, to_dev, u8

pytestmark = pytest.mark.gpu


def _K():
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _run(x, cent, bits, G):
    K = _K()
    T, H, d = x.shape
    C = cent.shape[1]
    codec = K.Codec(H, d, C, bits, G, 0, K.KVQ_META_F32, 2)
    idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
    codes2, meta2 = torch.empty_like(codes), torch.empty_like(meta)
    cd = to_dev(cent)
    K.kvq_encode_stages(codec, to_dev(x), cd, idx, codes, meta, codes2, meta2)
    comp = K.Compressed(codec, T, cd, idx, codes, meta, codes2=codes2, meta2=meta2)
    out = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
    K.kvq_decode(comp, out)
    outb = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
    K.kvq_decode(comp, outb)
    torch.cuda.synchronize()
    assert K.kvq_last_device_status() == K.KVQ_OK
    return idx, codes, meta, codes2, meta2, out, outb


def _check(x, cent, bits, G, got):
    T, H, d = x.shape
    idx, codes, meta, codes2, meta2, out, outb = got
    ref = O.encode2(x, cent, bits, G)
    assert np.array_equal(bits_u16(idx).reshape(H, T), ref[0])
    assert np.array_equal(u8(codes).reshape(ref[1].shape), ref[1])
    assert np.array_equal(f32_bits(meta).reshape(ref[2].shape), f32_bits(ref[2]))
    c2 = u8(codes2).reshape(ref[3].shape)
    assert np.array_equal(c2, ref[3]), f"stage-2 codes differ at {np.argwhere(c2 != ref[3])[:5]}"
    assert np.array_equal(f32_bits(meta2).reshape(ref[4].shape), f32_bits(ref[4]))
    dref = O.decode2(*ref, cent, bits, G)
    assert np.array_equal(f32_bits(out), f32_bits(dref)), "two-stage decode differs"
    assert np.array_equal(bits_u16(outb), bits_u16(out.to(torch.bfloat16)))


@pytest.mark.parametrize("name,T,H,bits,G,C,f32", [
    ("wan13b", 1537, 3, 2, 16, 256, False),
    ("wan13b", 1000, 2, 4, 32, 64, True),
    ("14b", 700, 2, 2, 64, 600, False),
    ("tiny", 1024, 2, 4, 16, 16, True),
    ("tiny", 333, 2, 2, 32, 7, False),
    ("14b", 901, 2, 4, 64, 300, False),     # filter, d = 128, INT4 G64
    ("14b", 515, 2, 4, 16, 512, False),     # filter, the largest C it takes
    ("tiny", 517, 2, 4, 16, 64, False),     # filter, d = 64
    ("tiny", 129, 2, 2, 16, 33, False),     # filter, d = 64, INT2 G16
])
def test_two_stage_encode_decode_bit_exact(name, T, H, bits, G, C, f32):
    w = synth.workload(name)
    x = np.ascontiguousarray(synth.make_history(w, "K", max_tokens=T)[:, :H])
    if x.dtype == np.float32 and not f32:
        x = synth.bf16_bits_from_f64(x.astype(np.float64))
    if f32 and x.dtype == np.uint16:
        x = synth.bf16_bits_to_f32(x)
    xb = x if x.dtype == np.uint16 else synth.bf16_bits_from_f64(x.astype(np.float64))
    cent = O.fit(xb[:C], C, 0)
    _check(x, cent, bits, G, _run(x, cent, bits, G))


def test_two_stage_full_wan_history():
    """The whole Wan-like K history (32,760 tokens x 12 heads, C = 256,
    INT2 G16), compared on every token-head."""
    w = synth.workload("wan13b")
    x = synth.make_history(w, "K")
    cent = O.fit(x[:w.num_centroids], w.num_centroids, 0)
    _check(x, cent, w.bits_k, w.group_size, _run(x, cent, w.bits_k, w.group_size))


def test_two_stage_filter_and_exact_paths_agree():
    """The same Wan-like history as bf16 (filter) and as its float32 widening
    (exact kernel): every output identical."""
    w = synth.workload("wan13b")
    x = np.ascontiguousarray(synth.make_history(w, "K", max_tokens=2050)[:, :4])
    cent = O.fit(x[:128], 128, 0)
    a = _run(x, cent, 2, 16)
    b = _run(synth.bf16_bits_to_f32(x), cent, 2, 16)
    for u, v in zip(a[:5], b[:5]):
        assert torch.equal(u, v)
    assert np.array_equal(f32_bits(a[5]), f32_bits(b[5]))
