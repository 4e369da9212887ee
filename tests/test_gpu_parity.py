"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs.

Bar: centroid indices, packed codes and {scale, zero} bits identical; fitted
centres identical; per-head reconstruction identical in binary32; attention
within relative Frobenius 1e-2 and max abs 3e-2 of the oracle, LSE within
1e-3.  The tiny and the Wan-1.3B-like workloads are checked on every
token-head, query row and head; the 14B-like layer and the sweep points on
sampled token-heads and query rows that the oracle computes one by one; small
edge shapes in full.
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


def _gpu_encode(codec, x_np, cent_np):
    K = _K()
    x = to_dev(x_np)
    cent = to_dev(cent_np)
    idx, codes, meta = K.alloc_encoded(codec, x_np.shape[0], x.device)
    K.kvq_encode(codec, x, cent, idx, codes, meta)
    return K.Compressed(codec, x_np.shape[0], cent, idx, codes, meta)


def _assert_encoded_equal(comp, H, T, d, bits, G, idx_ref, codes_ref, meta_ref, tokens=None, heads=None):
    idx = bits_u16(comp.idx).reshape(H, T)
    codes = u8(comp.codes).reshape(H, T, d * bits // 8)
    meta = f32_bits(comp.meta).reshape(H, T, d // G, 2)
    if heads is not None:
        idx, codes, meta = idx[heads], codes[heads], meta[heads]
    if tokens is not None:
        idx, codes, meta = idx[:, tokens], codes[:, tokens], meta[:, tokens]
    assert np.array_equal(idx, idx_ref), f"idx mismatch at {np.argwhere(idx != idx_ref)[:5]}"
    assert np.array_equal(codes, codes_ref), f"codes mismatch at {np.argwhere(codes != codes_ref)[:5]}"
    assert np.array_equal(meta, f32_bits(meta_ref)), "meta mismatch"


def _attention(q_np, kc, vc, t0=None, t1=None, o_dtype=torch.float32, split=False):
    K = _K()
    q = to_dev(q_np)
    Tq, H, d = q_np.shape
    o = torch.empty((Tq, H, d), dtype=o_dtype, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, kc.codec, kc.num_tokens, "cuda", num_queries=Tq) if split else None
    K.kvq_attention_lse(q, kc, vc, o, lse, t_begin=0 if t0 is None else t0, t_end=t1, workspace=ws)
    return o, lse


def _status_ok():
    K = _K()
    assert K.kvq_last_device_status() == K.KVQ_OK


def _sample_tokens(T, n, seed):
    rng = np.random.default_rng(seed)
    pick = set(range(min(T, 128))) | set(range(max(0, T - 128), T))
    pick |= set(rng.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(pick))


# ----------------------------------------------------------------------------
# tiny workload: every output in full
# ----------------------------------------------------------------------------

def test_tiny_end_to_end():
    K = _K()
    w = synth.workload("tiny")
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    T, H, d = xk.shape
    codec = K.Codec(H, d, w.num_centroids, w.bits_k, w.group_size)
    comps, decs = [], []
    for x in (xk, xv):
        cent_ref = O.fit(x, w.num_centroids, w.kmeans_iters)
        idx_ref, codes_ref, meta_ref = O.encode(x, cent_ref, w.bits_k, w.group_size)
        dec_ref = O.decode(idx_ref, codes_ref, meta_ref, cent_ref, w.bits_k, w.group_size)
        xd = to_dev(x)
        cent = torch.empty((H, w.num_centroids, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, xd, w.kmeans_iters, cent)
        assert np.array_equal(bits_u16(cent), cent_ref), "fitted centres differ"
        comp = _gpu_encode(codec, x, cent_ref)
        _assert_encoded_equal(comp, H, T, d, w.bits_k, w.group_size, idx_ref, codes_ref, meta_ref)
        dec = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, dec)
        assert np.array_equal(f32_bits(dec), f32_bits(dec_ref)), "decode differs"
        decb = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_decode(comp, decb)
        want_b = torch.from_numpy(dec_ref).to(torch.bfloat16)
        assert torch.equal(decb.cpu().view(torch.int16), want_b.view(torch.int16))
        comps.append(comp)
        decs.append(dec_ref)
    o_ref, lse_ref = O.attention(q, decs[0], decs[1])
    o, lse = _attention(q, comps[0], comps[1])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "tiny")
    o2, lse2 = _attention(q, comps[0], comps[1], split=True)
    assert_attention_close(o2.cpu().numpy(), lse2.cpu().numpy(), o_ref, lse_ref, "tiny split")
    # the bf16 output is the binary32 result rounded to nearest-even
    ob, lseb = _attention(q, comps[0], comps[1], o_dtype=torch.bfloat16)
    assert torch.equal(ob.cpu().view(torch.int16), o.cpu().to(torch.bfloat16).view(torch.int16))
    assert torch.equal(lseb.cpu(), lse.cpu())
    # split history + LSE merge
    cuts = [0, 300, 301, 777, T]
    o_parts, l_parts = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, lse = _attention(q, comps[0], comps[1], a, b)
        o_parts.append(o)
        l_parts.append(lse)
    om = torch.empty_like(o_parts[0])
    lm = torch.empty_like(l_parts[0])
    K.kvq_lse_merge(o_parts, l_parts, om, lm)
    assert_attention_close(om.cpu().numpy(), lm.cpu().numpy(), o_ref, lse_ref, "tiny merged")
    # merge against the oracle's merge of the GPU's own parts (tight)
    o2, l2 = O.lse_merge([p.cpu().numpy() for p in o_parts], [p.cpu().numpy() for p in l_parts])
    assert np.max(np.abs(om.cpu().numpy() - o2)) < 1e-5
    assert np.max(np.abs(lm.cpu().numpy() - l2)) < 1e-5
    _status_ok()


# ----------------------------------------------------------------------------
# Wan-1.3B-like layer at full size (the benchmarked launch configuration)
# ----------------------------------------------------------------------------

@pytest.fixture(scope="module")
def wan():
    w = synth.workload("wan13b")
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    seeds_k = O.fit(xk[: w.num_centroids], w.num_centroids, 0)
    seeds_v = O.fit(xv[: w.num_centroids], w.num_centroids, 0)
    return w, xk, xv, q, seeds_k, seeds_v


def test_wan_encode_decode_full_size(wan):
    """Every token-head of the Wan-1.3B-like history (12 heads x 32,760 tokens,
    K and V): idx, codes and {s, z} bit-exact, and the reconstruction bit-exact
    in binary32."""
    K = _K()
    w, xk, xv, q, seeds_k, seeds_v = wan
    T, H, d = xk.shape
    for x, cent, bits in ((xk, seeds_k, w.bits_k), (xv, seeds_v, w.bits_v)):
        codec = K.Codec(H, d, w.num_centroids, bits, w.group_size)
        comp = _gpu_encode(codec, x, cent)
        idx_r, codes_r, meta_r = O.encode(x, cent, bits, w.group_size)
        _assert_encoded_equal(comp, H, T, d, bits, w.group_size, idx_r, codes_r, meta_r)
        dec = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, dec)
        dref = O.decode(idx_r, codes_r, meta_r, cent, bits, w.group_size)
        assert np.array_equal(f32_bits(dec), f32_bits(dref)), "decode differs"
    _status_ok()


def test_wan_fit_full_size(wan):
    """Centres of all 12 heads after the benchmark's 2 k-means rounds, K and V,
    bit-exact."""
    K = _K()
    w, xk, xv, *_ = wan
    T, H, d = xk.shape
    for x, bits in ((xk, w.bits_k), (xv, w.bits_v)):
        codec = K.Codec(H, d, w.num_centroids, bits, w.group_size)
        cent = torch.empty((H, w.num_centroids, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, to_dev(x), w.kmeans_iters, cent)
        ref = O.fit(x, w.num_centroids, w.kmeans_iters)
        assert np.array_equal(bits_u16(cent), ref), f"centres differ in {np.sum(bits_u16(cent) != ref)} values"
    _status_ok()


def test_wan_attention_full_size(wan):
    """All 4,680 query rows of all 12 heads over the whole 32,760-token
    compressed history, unsplit and with the history split inside the call."""
    K = _K()
    w, xk, xv, q, seeds_k, seeds_v = wan
    T, H, d = xk.shape
    ck = _gpu_encode(K.Codec(H, d, w.num_centroids, w.bits_k, w.group_size), xk, seeds_k)
    cv = _gpu_encode(K.Codec(H, d, w.num_centroids, w.bits_v, w.group_size), xv, seeds_v)
    o, lse = _attention(q, ck, cv)
    o_s, lse_s = _attention(q, ck, cv, split=True)
    dk = O.decode(*O.encode(xk, seeds_k, w.bits_k, w.group_size), seeds_k, w.bits_k, w.group_size)
    dv = O.decode(*O.encode(xv, seeds_v, w.bits_v, w.group_size), seeds_v, w.bits_v, w.group_size)
    o_ref, lse_ref = O.attention(q, dk, dv)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "wan full")
    assert_attention_close(o_s.cpu().numpy(), lse_s.cpu().numpy(), o_ref, lse_ref, "wan full, split history")
    _status_ok()


# ----------------------------------------------------------------------------
# 14B-like layer: 40 heads, mixed k4v2, 8 history blocks merged by LSE
# ----------------------------------------------------------------------------

def test_14b_blocks_merged_sampled():
    K = _K()
    w = synth.workload("14b")
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    T, H, d = xk.shape
    sk = O.fit(xk[: w.num_centroids], w.num_centroids, 0)
    sv = O.fit(xv[: w.num_centroids], w.num_centroids, 0)
    ck = _gpu_encode(K.Codec(H, d, w.num_centroids, w.bits_k, w.group_size), xk, sk)
    cv = _gpu_encode(K.Codec(H, d, w.num_centroids, w.bits_v, w.group_size), xv, sv)
    nb = w.history_blocks
    edges = [T * i // nb for i in range(nb + 1)]
    parts = [_attention(q, ck, cv, a, b) for a, b in zip(edges[:-1], edges[1:])]
    om = torch.empty_like(parts[0][0])
    lm = torch.empty_like(parts[0][1])
    K.kvq_lse_merge([p[0] for p in parts], [p[1] for p in parts], om, lm)
    heads = [5, 38]
    rows = _sample_tokens(w.query_tokens, 128, 6)
    sub = lambda a: np.ascontiguousarray(a[:, heads])
    ek = O.encode(sub(xk), sk[heads], w.bits_k, w.group_size)
    ev = O.encode(sub(xv), sv[heads], w.bits_v, w.group_size)
    toks = _sample_tokens(T, 1024, 7)
    _assert_encoded_equal(ck, H, T, d, w.bits_k, w.group_size, ek[0][:, toks], ek[1][:, toks], ek[2][:, toks],
                          tokens=toks, heads=heads)
    dk = O.decode(*ek, sk[heads], w.bits_k, w.group_size)
    dv = O.decode(*ev, sv[heads], w.bits_v, w.group_size)
    o_ref, lse_ref = O.attention(sub(q), dk, dv, rows=rows)
    assert_attention_close(om.cpu().numpy()[rows][:, heads], lm.cpu().numpy()[heads][:, rows], o_ref, lse_ref,
                           "14b merged")
    # one block on its own
    b = 3
    ob_ref, lb_ref = O.attention(sub(q), dk[edges[b]:edges[b + 1]], dv[edges[b]:edges[b + 1]], rows=rows)
    assert_attention_close(parts[b][0].cpu().numpy()[rows][:, heads], parts[b][1].cpu().numpy()[heads][:, rows],
                           ob_ref, lb_ref, "14b block 3")
    _status_ok()


# ----------------------------------------------------------------------------
# sweep points (12 heads, AR(1) + outliers)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T,Tq,bk,bv,G,C", [(4096, 1560, 4, 2, 64, 64), (8192, 1560, 2, 4, 32, 1024),
                                             (4096, 4680, 4, 4, 16, 256)])
def test_sweep_point(T, Tq, bk, bv, G, C):
    K = _K()
    w = synth.sweep_point(T, Tq, bk, bv, G, C)
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    H, d = w.num_heads, w.head_dim
    heads = [0, 9]
    sub = lambda a: np.ascontiguousarray(a[:, heads])
    cks, decs = [], []
    for x, bits in ((xk, bk), (xv, bv)):
        codec = K.Codec(H, d, C, bits, G)
        cent = torch.empty((H, C, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, to_dev(x), 2, cent)
        cref = O.fit(sub(x), C, 2)
        assert np.array_equal(bits_u16(cent)[heads], cref)
        comp = _gpu_encode(codec, x, bits_u16(cent))
        e = O.encode(sub(x), cref, bits, G)
        _assert_encoded_equal(comp, H, T, d, bits, G, *e, heads=heads)
        cks.append(comp)
        decs.append(O.decode(*e, cref, bits, G))
    o, lse = _attention(q, cks[0], cks[1])
    rows = _sample_tokens(Tq, 256, 8)
    o_ref, lse_ref = O.attention(sub(q), decs[0], decs[1], rows=rows)
    assert_attention_close(o.cpu().numpy()[rows][:, heads], lse.cpu().numpy()[heads][:, rows], o_ref, lse_ref,
                           w.name)
    _status_ok()


# ----------------------------------------------------------------------------
# edge cases: ragged tails, tiny sizes, degenerate codecs, ranges
# ----------------------------------------------------------------------------

def _bf16_bits(a):
    return synth.bf16_bits_from_f64(np.asarray(a, np.float64))


@pytest.mark.parametrize("d,T,Tq,C,bits,G", [(128, 300, 130, 5, 4, 16), (64, 1, 1, 1, 2, 16),
                                              (64, 129, 257, 129, 2, 64), (128, 1000, 7, 1, 2, 32),
                                              (128, 255, 128, 64, 4, 64)])
def test_edge_shapes_full(d, T, Tq, C, bits, G):
    K = _K()
    rng = np.random.default_rng(T * 7 + d)
    H = 3
    xk = _bf16_bits(rng.normal(size=(T, H, d)) * rng.uniform(0.5, 3, size=(1, H, d)))
    xv = _bf16_bits(rng.normal(size=(T, H, d)))
    q = _bf16_bits(rng.normal(size=(Tq, H, d)))
    codec = K.Codec(H, d, C, bits, G)
    comps, decs = [], []
    for x in (xk, xv):
        cent_ref = O.fit(x, C, 2)
        cent = torch.empty((H, C, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, to_dev(x), 2, cent)
        assert np.array_equal(bits_u16(cent), cent_ref)
        e = O.encode(x, cent_ref, bits, G)
        comp = _gpu_encode(codec, x, cent_ref)
        _assert_encoded_equal(comp, H, T, d, bits, G, *e)
        dec = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, dec)
        dref = O.decode(*e, cent_ref, bits, G)
        assert np.array_equal(f32_bits(dec), f32_bits(dref))
        comps.append(comp)
        decs.append(dref)
    o, lse = _attention(q, comps[0], comps[1])
    o_ref, lse_ref = O.attention(q, decs[0], decs[1])
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "edge full")
    # an unaligned sub-range and an empty range
    t0, t1 = T // 3, T - T // 5
    if t1 > t0:
        o, lse = _attention(q, comps[0], comps[1], t0, t1)
        o_ref, lse_ref = O.attention(q, decs[0][t0:t1], decs[1][t0:t1])
        assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "edge range")
    o, lse = _attention(q, comps[0], comps[1], T // 2, T // 2)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    _status_ok()


def test_identical_tokens_and_constant_groups():
    K = _K()
    H, d, T, C = 2, 128, 200, 4
    rng = np.random.default_rng(31)
    tok = _bf16_bits(rng.normal(size=(H, d)))
    x = np.broadcast_to(tok[None], (T, H, d)).copy()
    # tokens 100.. differ from the first token only in channels 64..127, so
    # every centre equals the token in channels 0..63 and the residual of
    # those channels is a constant zero group whichever centre a token joins
    x[100:, :, 64:] = _bf16_bits(rng.normal(size=(T - 100, H, 64)))
    for bits, G in ((2, 16), (4, 64)):
        codec = K.Codec(H, d, C, bits, G)
        cent_ref = O.fit(x, C, 2)
        e = O.encode(x, cent_ref, bits, G)
        comp = _gpu_encode(codec, x, cent_ref)
        _assert_encoded_equal(comp, H, T, d, bits, G, *e)
        assert np.all(e[1][:, :, : 64 * bits // 8] == 0) and np.all(e[2][:, :, : 64 // G] == 0)
    _status_ok()


def test_encode_ties_and_near_ties():
    """Duplicated centres (exact ties) and tokens half-way between two centres:
    the tensor-core filter's window then holds several candidates and the
    specified distance decides, lowest index first."""
    K = _K()
    rng = np.random.default_rng(41)
    H, d, C, T = 2, 128, 64, 700
    base = rng.integers(-4, 5, size=(H, C // 2, d)).astype(np.float64)
    cent = _bf16_bits(np.concatenate([base, base], axis=1))  # centre j == centre j + 32
    cf = synth.bf16_bits_to_f32(cent).astype(np.float64)
    x = rng.normal(size=(T, H, d)) * 2
    for t in range(0, T, 3):  # midpoints of centre pairs (exact in bf16: half-integers)
        for h in range(H):
            a, b = rng.choice(C // 2, size=2, replace=False)
            x[t, h] = 0.5 * (cf[h, a] + cf[h, b])
    for t in range(1, T, 7):  # exactly on a centre
        for h in range(H):
            x[t, h] = cf[h, rng.integers(C)]
    x = _bf16_bits(x)
    for bits, G in ((2, 16), (4, 32)):
        codec = K.Codec(H, d, C, bits, G)
        e = O.encode(x, cent, bits, G)
        comp = _gpu_encode(codec, x, cent)
        _assert_encoded_equal(comp, H, T, d, bits, G, *e)
        assert np.all(e[0] < C // 2)  # ties resolved to the lower duplicate
    _status_ok()


def test_fit_token_order_sums_with_inexact_binary64():
    """Values spanning ~33 decades make the binary64 centre sums inexact; the
    fit still matches the oracle bit for bit because both sum every centre's
    tokens sequentially in token order."""
    K = _K()
    rng = np.random.default_rng(43)
    T, H, d, C = 3000, 2, 128, 16
    mag = 10.0 ** rng.uniform(-30, 3, size=(T, H, d))
    x = _bf16_bits(rng.normal(size=(T, H, d)) * mag)
    for it in (1, 3):
        codec = K.Codec(H, d, C, 2, 16)
        cent = torch.empty((H, C, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, to_dev(x), it, cent)
        assert np.array_equal(bits_u16(cent), O.fit(x, C, it))
    _status_ok()


@pytest.mark.parametrize("d,T,H,C,it", [(128, 2051, 3, 37, 2), (64, 777, 2, 64, 1)])
def test_fit_float32_history(d, T, H, C, it):
    """kvq_fit_centroids over a float32 history (the binary32 row gathers of
    the centre sums; L from 24-bit significands) bit-exact against the oracle,
    a ragged token count included."""
    K = _K()
    rng = np.random.default_rng(d * 1000 + T)
    x = (rng.normal(size=(T, H, d)) * rng.uniform(0.2, 5, size=(1, H, d))).astype(np.float32)
    x[::97] *= np.float32(2.0 ** -20)     # a spread of exponents in every head
    codec = K.Codec(H, d, C, 2, 16)
    cent = torch.empty((H, C, d), dtype=torch.bfloat16, device="cuda")
    K.kvq_fit_centroids(codec, to_dev(x), it, cent)
    assert np.array_equal(bits_u16(cent), O.fit(x, C, it))
    _status_ok()
