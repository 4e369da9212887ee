"""GPU parity of the full-layer attention of the current chunk (NanoKV page,
Fig. 4(a,d): the history is read through the decoder and partial results are
merged by their log-sum-exp; Table 4: protected tokens stay uncompressed).

* kvq_attention_dense_lse: attention over uncompressed bf16 keys and values
  (the chunk's own, or raw protected tokens) against the oracle's attention
  over the same bf16 values;
* kvq_layer_attention: one softmax over a compressed history and the dense
  chunk against the oracle's attention over the union of both key sets.

Bars are those of every attention test: relative Frobenius error of O
<= 1e-2, max abs error of O <= 3e-2, max abs error of the natural-log LSE
<= 1e-3, and the same -inf pattern of the LSE.
"""

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_attention_close, to_dev

pytestmark = pytest.mark.gpu


def _K():
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _bf16_bits(a):
    return synth.bf16_bits_from_f64(np.asarray(a, np.float64))


def _status_ok():
    K = _K()
    assert K.kvq_last_device_status() == K.KVQ_OK


def _dense(q_np, k_np, v_np, t0=0, t1=None, o_dtype=torch.float32, split=False):
    K = _K()
    Tq, H, d = q_np.shape
    q, k, v = to_dev(q_np), to_dev(k_np), to_dev(v_np)
    o = torch.empty((Tq, H, d), dtype=o_dtype, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    ws = None
    if split:
        ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, K.Codec(H, d, 1, 2, 16), 0, "cuda", num_queries=Tq)
    K.kvq_attention_dense_lse(q, k, v, o, lse, t_begin=t0, t_end=t1, workspace=ws)
    return o, lse


def _compress(x_np, C, bits, G, iters=2):
    """Centres from the oracle's fit, codes from the GPU encoder (bit-exact
    with the oracle's, which the codec parity tests establish), and the
    oracle's own reconstruction as the reference history."""
    K = _K()
    T, H, d = x_np.shape
    codec = K.Codec(H, d, C, bits, G)
    cent_ref = O.fit(x_np, C, iters)
    comp = K.compress(codec, to_dev(x_np), iters, centroids=to_dev(cent_ref))
    dec_ref = O.decode(*O.encode(x_np, cent_ref, bits, G), cent_ref, bits, G)
    return comp, dec_ref


@pytest.mark.parametrize("d,Tk,Tq,t0,t1", [
    (128, 300, 130, 0, 300),      # ragged keys and queries
    (128, 4680, 600, 0, 4680),    # a full chunk of keys, several query tiles
    (128, 1000, 7, 129, 871),     # unaligned sub-range
    (64, 1, 1, 0, 1),             # a single key and query
    (64, 129, 257, 0, 129),       # one key past a tile, queries past a CTA
    (64, 2000, 300, 17, 1999),
])
def test_dense_attention_against_oracle(d, Tk, Tq, t0, t1):
    rng = np.random.default_rng(Tk * 3 + d)
    H = 3
    k = _bf16_bits(rng.normal(size=(Tk, H, d)) * rng.uniform(0.5, 2.5, size=(1, H, d)))
    v = _bf16_bits(rng.normal(size=(Tk, H, d)) * 3.0)
    q = _bf16_bits(rng.normal(size=(Tq, H, d)))
    o_ref, lse_ref = O.attention(q, k[t0:t1], v[t0:t1])
    o, lse = _dense(q, k, v, t0, t1)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "dense")
    o_s, lse_s = _dense(q, k, v, t0, t1, split=True)
    assert_attention_close(o_s.cpu().numpy(), lse_s.cpu().numpy(), o_ref, lse_ref, "dense split")
    # the bf16 output is the binary32 result rounded to nearest-even
    ob, lseb = _dense(q, k, v, t0, t1, o_dtype=torch.bfloat16)
    assert torch.equal(ob.cpu().view(torch.int16), o.cpu().to(torch.bfloat16).view(torch.int16))
    assert torch.equal(lseb.cpu(), lse.cpu())
    # an empty range: O = 0, lse = -inf
    o0, l0 = _dense(q, k, v, t0, t0)
    assert torch.all(o0 == 0) and torch.all(torch.isneginf(l0))
    _status_ok()


def test_dense_attention_selects_one_key():
    """Query i has logit 32 * 32 / sqrt(128) = 90.5 with key i mod 128 and 0
    with every other key, so its output is that key's value (the others weigh
    about e^-90) and its LSE is 90.5 plus ln(1 + 255 e^-90.5)."""
    rng = np.random.default_rng(41)
    Tq, Tk, H, d = 256, 256, 2, 128
    q = np.zeros((Tq, H, d))
    k = np.zeros((Tk, H, d))
    for i in range(Tq):
        q[i, :, i % d] = 32.0
        if i < d:
            k[i, :, i] = 32.0
    v = _bf16_bits(rng.integers(-64, 64, size=(Tk, H, d)) / 8.0)
    qb, kb = _bf16_bits(q), _bf16_bits(k)
    o, lse = _dense(qb, kb, v)
    o_ref, lse_ref = O.attention(qb, kb, v)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "one-hot keys")
    want = synth.bf16_bits_to_f32(v)[np.arange(Tq) % d]
    assert np.max(np.abs(o.cpu().numpy() - want)) < 1e-6
    _status_ok()


@pytest.mark.parametrize("d,T,Tc,Tq,C,bk,bv,G,t0,t1", [
    (128, 1000, 300, 300, 64, 2, 2, 16, 0, 1000),
    (128, 777, 129, 513, 32, 4, 2, 32, 100, 650),
    (64, 500, 257, 130, 16, 2, 4, 64, 0, 500),
    (128, 400, 0, 200, 16, 2, 2, 16, 0, 400),      # no chunk keys: the history alone
    (128, 400, 300, 200, 16, 2, 2, 16, 200, 200),  # empty history range: the chunk alone
])
def test_layer_attention_against_oracle(d, T, Tc, Tq, C, bk, bv, G, t0, t1):
    K = _K()
    rng = np.random.default_rng(T + Tc + d)
    H = 3
    xk = _bf16_bits(rng.normal(size=(T, H, d)) * rng.uniform(0.5, 2.5, size=(1, H, d)))
    xv = _bf16_bits(rng.normal(size=(T, H, d)))
    kc = _bf16_bits(rng.normal(size=(Tc, H, d)) * rng.uniform(0.5, 2.5, size=(1, H, d)))
    vc = _bf16_bits(rng.normal(size=(Tc, H, d)))
    q = _bf16_bits(rng.normal(size=(Tq, H, d)))
    ck, dk = _compress(xk, C, bk, G)
    cv, dv = _compress(xv, C, bv, G)
    o_ref, lse_ref = O.layer_attention(q, dk[t0:t1], dv[t0:t1], kc, vc)
    ws = K.alloc_workspace(K.KVQ_OP_LAYER_ATTENTION, ck.codec, T, "cuda", num_queries=Tq)
    for o_dtype in (torch.float32, torch.bfloat16):
        o = torch.empty((Tq, H, d), dtype=o_dtype, device="cuda")
        lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
        K.kvq_layer_attention(to_dev(q), ck, cv, to_dev(kc) if Tc else None, to_dev(vc) if Tc else None, o, lse,
                              ws, t_begin=t0, t_end=t1)
        assert_attention_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"layer {o_dtype}")
    _status_ok()


def test_layer_attention_both_sets_empty():
    K = _K()
    rng = np.random.default_rng(43)
    T, H, d, Tq = 300, 2, 128, 40
    x = _bf16_bits(rng.normal(size=(T, H, d)))
    ck, _ = _compress(x, 16, 2, 16)
    ws = K.alloc_workspace(K.KVQ_OP_LAYER_ATTENTION, ck.codec, T, "cuda", num_queries=Tq)
    o = torch.full((Tq, H, d), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.zeros((H, Tq), dtype=torch.float32, device="cuda")
    K.kvq_layer_attention(to_dev(_bf16_bits(rng.normal(size=(Tq, H, d)))), ck, ck, None, None, o, lse, ws,
                          t_begin=100, t_end=100)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    _status_ok()


def test_layer_attention_wan_full_size():
    """The Wan-1.3B-like layer at full size: 12 heads x 128, a K2V2 history of
    32,760 tokens (C = 256, group 16) and the 4,680-token chunk that follows
    it, 4,680 queries; every query row of every head against the oracle.  Also
    checks that the layer call equals the LSE merge of the two attentions
    taken separately through the public calls."""
    K = _K()
    w = synth.workload("wan13b")
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    kc, vc = synth.make_chunk(w, "K"), synth.make_chunk(w, "V")
    T, H, d = xk.shape
    Tq = w.query_tokens
    # centres: the oracle's seeds (the first C tokens of every head)
    cents = [O.fit(x[: w.num_centroids], w.num_centroids, 0) for x in (xk, xv)]
    comps = [K.compress(K.Codec(H, d, w.num_centroids, bits, w.group_size), to_dev(x), 0, centroids=to_dev(c))
             for x, bits, c in ((xk, w.bits_k, cents[0]), (xv, w.bits_v, cents[1]))]
    qd, kcd, vcd = to_dev(q), to_dev(kc), to_dev(vc)
    ws = K.alloc_workspace(K.KVQ_OP_LAYER_ATTENTION, comps[0].codec, T, "cuda", num_queries=Tq)
    o = torch.empty((Tq, H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    K.kvq_layer_attention(qd, comps[0], comps[1], kcd, vcd, o, lse, ws)
    # the same result from the two public attentions and one merge
    ws_a = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=Tq)
    oh, lh = torch.empty_like(o), torch.empty_like(lse)
    oc, lc = torch.empty_like(o), torch.empty_like(lse)
    K.kvq_attention_lse(qd, comps[0], comps[1], oh, lh, workspace=ws_a)
    K.kvq_attention_dense_lse(qd, kcd, vcd, oc, lc, workspace=ws_a)
    om, lm = torch.empty_like(o), torch.empty_like(lse)
    K.kvq_lse_merge([oh, oc], [lh, lc], om, lm)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(om - o)).item() < 1e-4 and torch.max(torch.abs(lm - lse)).item() < 1e-4
    # every row of every head against the oracle
    dk = O.decode(*O.encode(xk, cents[0], w.bits_k, w.group_size), cents[0], w.bits_k, w.group_size)
    dv = O.decode(*O.encode(xv, cents[1], w.bits_v, w.group_size), cents[1], w.bits_v, w.group_size)
    o_ref, lse_ref = O.layer_attention(q, dk, dv, kc, vc)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "wan layer")
    _status_ok()
