"""Failure detection on the GPU without a fault: the bounded waits' give-up
path and the centre-index check, taken on purpose.

* With kvq_set_wait_limit(0) every bounded wait of the encode filter and of
  the d = 128 attention kernels (compressed history, and dense keys) gives up
  at its first poll: the call returns, kvq_last_device_status reports
  KVQ_ERR_DEVICE_TIMEOUT once (reading clears it), and after the default limit
  is restored the same calls on the same context are again bit-exact (encode)
  or in tolerance (attention) against the oracle.
* A compressed view holding centre indices >= C: decode and attention clamp
  them to centre 0 and report KVQ_ERR_INVALID_ARG; the decode equals the
  oracle's decode of the clamped indices bit for bit.
"""

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


@pytest.fixture(scope="module")
def case():
    w = synth.workload("wan13b")
    H, T, C, G = 4, 3001, 256, 16
    xk = np.ascontiguousarray(synth.make_history(w, "K", max_tokens=T)[:, :H])
    xv = np.ascontiguousarray(synth.make_history(w, "V", max_tokens=T)[:, :H])
    q = np.ascontiguousarray(synth.make_queries(w, max_tokens=700)[:, :H])
    cents = [O.fit(x[:C], C, 0) for x in (xk, xv)]
    return dict(H=H, T=T, C=C, G=G, d=128, x=(xk, xv), q=q, cent=cents)


def _with_limit(K, polls, fn):
    assert K.kvq_last_device_status() == K.KVQ_OK
    try:
        K.kvq_set_wait_limit(polls)
        fn()
        st = K.kvq_last_device_status()
    finally:
        K.kvq_set_wait_limit(K.KVQ_WAIT_LIMIT_DEFAULT)
    return st


def test_encode_filter_gives_up_then_recovers(case):
    K = _K()
    c = case
    codec = K.Codec(c["H"], c["d"], c["C"], 2, c["G"])
    x, cent = to_dev(c["x"][0]), to_dev(c["cent"][0])
    idx, codes, meta = K.alloc_encoded(codec, c["T"], "cuda")
    st = _with_limit(K, 0, lambda: K.kvq_encode(codec, x, cent, idx, codes, meta))
    assert st == K.KVQ_ERR_DEVICE_TIMEOUT
    assert K.kvq_last_device_status() == K.KVQ_OK  # reading cleared it
    K.kvq_encode(codec, x, cent, idx, codes, meta)
    assert K.kvq_last_device_status() == K.KVQ_OK
    idx_r, codes_r, meta_r = O.encode(c["x"][0], c["cent"][0], 2, c["G"])
    assert np.array_equal(bits_u16(idx).reshape(c["H"], c["T"]), idx_r)
    assert np.array_equal(u8(codes).reshape(codes_r.shape), codes_r)
    assert np.array_equal(f32_bits(meta).reshape(meta_r.shape), f32_bits(meta_r))


def test_attention_gives_up_then_recovers(case):
    K = _K()
    c = case
    H, d, T = c["H"], c["d"], c["T"]
    comps, decs = [], []
    for x, cent in zip(c["x"], c["cent"]):
        codec = K.Codec(H, d, c["C"], 2, c["G"])
        idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
        K.kvq_encode(codec, to_dev(x), to_dev(cent), idx, codes, meta)
        comps.append(K.Compressed(codec, T, to_dev(cent), idx, codes, meta))
        decs.append(O.decode(*O.encode(x, cent, 2, c["G"]), cent, 2, c["G"]))
    q = c["q"]
    qd = to_dev(q)
    o = torch.empty((q.shape[0], H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=q.shape[0])
    run = lambda: K.kvq_attention_lse(qd, comps[0], comps[1], o, lse, workspace=ws)
    assert _with_limit(K, 0, run) == K.KVQ_ERR_DEVICE_TIMEOUT
    run()
    assert K.kvq_last_device_status() == K.KVQ_OK
    o_ref, lse_ref = O.attention(q, decs[0], decs[1])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "after the give-up")
    # dense keys: the chunk's own keys and values
    kc = to_dev(c["x"][0][:900])
    vc = to_dev(c["x"][1][:900])
    run_dense = lambda: K.kvq_attention_dense_lse(qd, kc, vc, o, lse, workspace=ws)
    assert _with_limit(K, 0, run_dense) == K.KVQ_ERR_DEVICE_TIMEOUT
    run_dense()
    assert K.kvq_last_device_status() == K.KVQ_OK
    o_ref, lse_ref = O.attention(q, c["x"][0][:900], c["x"][1][:900])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "dense after the give-up")


def test_out_of_range_centre_index_is_clamped_and_reported(case):
    K = _K()
    c = case
    H, d, T, C, G = c["H"], c["d"], c["T"], c["C"], c["G"]
    enc = []
    for x, cent in zip(c["x"], c["cent"]):
        idx_r, codes_r, meta_r = O.encode(x, cent, 2, G)
        enc.append([idx_r.copy(), codes_r, meta_r])
    bad = [(0, 5), (1, 7), (3, T - 1)]
    for h, t in bad:
        enc[0][0][h, t] = C + h
    enc[1][0][2, 11] = 65535
    comps = []
    for (idx_b, codes_r, meta_r), cent in zip(enc, c["cent"]):
        comps.append(K.Compressed(K.Codec(H, d, C, 2, G), T, to_dev(cent), to_dev(idx_b.view(np.int16)),
                                  to_dev(codes_r), to_dev(meta_r)))
    out = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
    K.kvq_decode(comps[0], out)
    assert K.kvq_last_device_status() == K.KVQ_ERR_INVALID_ARG
    clamped = np.where(enc[0][0] >= C, 0, enc[0][0]).astype(np.uint16)
    ref = O.decode(clamped, enc[0][1], enc[0][2], c["cent"][0], 2, G)
    assert np.array_equal(f32_bits(out), f32_bits(ref))
    q = c["q"]
    o = torch.empty((q.shape[0], H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    K.kvq_attention_lse(to_dev(q), comps[0], comps[1], o, lse)
    assert K.kvq_last_device_status() == K.KVQ_ERR_INVALID_ARG
    vcl = np.where(enc[1][0] >= C, 0, enc[1][0]).astype(np.uint16)
    vref = O.decode(vcl, enc[1][1], enc[1][2], c["cent"][1], 2, G)
    o_ref, lse_ref = O.attention(q, ref, vref)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "clamped indices")
    assert K.kvq_last_device_status() == K.KVQ_OK
