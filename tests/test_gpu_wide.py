"""Wider GPU parity at the full sizes of the 14B-like layer, the sweep and
the joint workload.

* 14B-like layer (40 heads x 128, 93,600 history tokens, C = 512, K4V2,
  G = 32, 8 history blocks): idx, codes and {s, z} of K and V bit-exact on a
  seeded 1/16 of the 128-token tiles of every one of the 40 heads (always
  the first and the tail tile); the LSE merge of the 8 block attentions on
  512 query rows of every head against the oracle's attention over the
  oracle's own reconstruction of the whole history of that head; the
  centres of the full-size fit (2 rounds over all 93,600 tokens) bit-exact
  on three heads.
* sweep: points that together cover every (b_K, b_V), every G, every C and
  a 131,072-token history.
* joint workload: the decoder at full size (32,760 tokens, both branches,
  K4V4 rank 192) on sampled tokens, within the decoder's derived bound.
* the next rows at the sizes the benchmark times them: QSAC encode of the
  whole Wan-like K history (sampled tiles, bit-exact), PSAC attention over the
  whole Wan-like history in 2 blocks merged by LSE (512 rows per head), and
  NanoKV-Fast on the whole joint workload (512 rows per head).
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


def _gpu_encode(codec, x, cent_np):
    K = _K()
    T = x.shape[0]
    cent = to_dev(cent_np)
    idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
    K.kvq_encode(codec, x, cent, idx, codes, meta)
    return K.Compressed(codec, T, cent, idx, codes, meta)


def _tiles_sample(T, frac, seed):
    """Token indices of a seeded `frac` of the 128-token tiles, always with the
    first and the tail tile."""
    ntiles = (T + 127) // 128
    rng = np.random.default_rng(seed)
    k = max(1, int(round(ntiles * frac)))
    tiles = set(rng.choice(ntiles, size=k, replace=False).tolist()) | {0, ntiles - 1}
    return np.concatenate([np.arange(t * 128, min(T, t * 128 + 128)) for t in sorted(tiles)])


def _rows_sample(n, k, seed):
    """k query rows (all of them when n <= k): the first and last 64 and a
    seeded choice of the rest."""
    if n <= k:
        return np.arange(n)
    ends = set(range(64)) | set(range(n - 64, n))
    rest = np.array(sorted(set(range(n)) - ends))
    rng = np.random.default_rng(seed)
    pick = ends | set(rng.choice(rest, size=k - len(ends), replace=False).tolist())
    return np.array(sorted(pick))


@pytest.fixture(scope="module")
def w14():
    w = synth.workload("14b")
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    return w, xk, xv, q


def test_14b_codes_every_head_and_merged_attention(w14):
    K = _K()
    w, xk, xv, q = w14
    T, H, d = xk.shape
    C, G = w.num_centroids, w.group_size
    seeds = [O.fit(x[:C], C, 0) for x in (xk, xv)]
    comps = []
    for x, cent, bits in ((xk, seeds[0], w.bits_k), (xv, seeds[1], w.bits_v)):
        codec = K.Codec(H, d, C, bits, G)
        comps.append(_gpu_encode(codec, to_dev(x), cent))
    # (1) codes and {s, z} on 1/16 of the tiles of every head
    toks = _tiles_sample(T, 1.0 / 16, 11)
    for comp, x, cent, bits in zip(comps, (xk, xv), seeds, (w.bits_k, w.bits_v)):
        idx_r, codes_r, meta_r = O.encode(np.ascontiguousarray(x[toks]), cent, bits, G)
        idx = bits_u16(comp.idx).reshape(H, T)[:, toks]
        codes = u8(comp.codes).reshape(H, T, d * bits // 8)[:, toks]
        meta = f32_bits(comp.meta).reshape(H, T, d // G, 2)[:, toks]
        assert np.array_equal(idx, idx_r), f"idx mismatch at {np.argwhere(idx != idx_r)[:5]}"
        assert np.array_equal(codes, codes_r), f"codes mismatch at {np.argwhere(codes != codes_r)[:5]}"
        assert np.array_equal(meta, f32_bits(meta_r)), "meta mismatch"
    # (2) the 8 history blocks, merged by LSE, on 512 query rows of every head
    nb = w.history_blocks
    edges = [T * i // nb for i in range(nb + 1)]
    qd = to_dev(q)
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=q.shape[0])
    parts = []
    for a, b in zip(edges[:-1], edges[1:]):
        o = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
        K.kvq_attention_lse(qd, comps[0], comps[1], o, lse, t_begin=a, t_end=b, workspace=ws)
        parts.append((o, lse))
    om = torch.empty_like(parts[0][0])
    lm = torch.empty_like(parts[0][1])
    K.kvq_lse_merge([p[0] for p in parts], [p[1] for p in parts], om, lm)
    assert K.kvq_last_device_status() == K.KVQ_OK
    om, lm = om.cpu().numpy(), lm.cpu().numpy()
    rows = _rows_sample(q.shape[0], 512, 12)
    for h0 in range(0, H, 8):  # eight heads at a time: the oracle runs one thread per head
        hs = slice(h0, min(H, h0 + 8))
        dec = []
        for x, cent, bits in ((xk, seeds[0], w.bits_k), (xv, seeds[1], w.bits_v)):
            e = O.encode(np.ascontiguousarray(x[:, hs]), cent[hs], bits, G)
            dec.append(O.decode(*e, cent[hs], bits, G))
        o_ref, lse_ref = O.attention(np.ascontiguousarray(q[:, hs]), dec[0], dec[1], rows=rows)
        assert_attention_close(om[rows][:, hs], lm[hs][:, rows], o_ref, lse_ref, f"14b heads {h0}..")


def test_14b_fit_full_size(w14):
    """kvq_fit_centroids over the whole 93,600-token history of all 40 heads
    (C = 512, 2 rounds), bit-exact against the oracle on three heads."""
    K = _K()
    w, xk, xv, q = w14
    T, H, d = xk.shape
    heads = [0, 17, 39]
    codec = K.Codec(H, d, w.num_centroids, w.bits_k, w.group_size)
    cent = torch.empty((H, w.num_centroids, d), dtype=torch.bfloat16, device="cuda")
    K.kvq_fit_centroids(codec, to_dev(xk), w.kmeans_iters, cent)
    got = bits_u16(cent)[heads]
    ref = O.fit(np.ascontiguousarray(xk[:, heads]), w.num_centroids, w.kmeans_iters)
    assert np.array_equal(got, ref), f"centres differ in {np.sum(got != ref)} values"
    assert K.kvq_last_device_status() == K.KVQ_OK


@pytest.mark.parametrize("T,Tq,bk,bv,G,C", [(131072, 1560, 2, 2, 16, 64), (16384, 4680, 2, 2, 64, 256),
                                             (32768, 1560, 4, 2, 32, 1024)])
def test_sweep_cover(T, Tq, bk, bv, G, C):
    """Sweep points beside those of test_gpu_parity: with them every (b_K, b_V),
    G and C appears, and the longest history (131,072 tokens)."""
    K = _K()
    w = synth.sweep_point(T, Tq, bk, bv, G, C)
    xk, xv, q = synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)
    H, d = w.num_heads, w.head_dim
    heads = [2, 11]
    sub = lambda a: np.ascontiguousarray(a[:, heads])
    comps, decs = [], []
    for x, bits in ((xk, bk), (xv, bv)):
        codec = K.Codec(H, d, C, bits, G)
        xd = to_dev(x)
        cent = torch.empty((H, C, d), dtype=torch.bfloat16, device="cuda")
        K.kvq_fit_centroids(codec, xd, 2, cent)
        cref = O.fit(sub(x), C, 2)
        assert np.array_equal(bits_u16(cent)[heads], cref), "fitted centres differ"
        comp = _gpu_encode(codec, xd, bits_u16(cent))
        idx_r, codes_r, meta_r = O.encode(sub(x), cref, bits, G)
        assert np.array_equal(bits_u16(comp.idx).reshape(H, T)[heads], idx_r)
        assert np.array_equal(u8(comp.codes).reshape(H, T, d * bits // 8)[heads], codes_r)
        assert np.array_equal(f32_bits(comp.meta).reshape(H, T, d // G, 2)[heads], f32_bits(meta_r))
        comps.append(comp)
        decs.append(O.decode(idx_r, codes_r, meta_r, cref, bits, G))
    o = torch.empty((Tq, H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=Tq)
    K.kvq_attention_lse(to_dev(q), comps[0], comps[1], o, lse, workspace=ws)
    rows = _rows_sample(Tq, 384, 13)
    o_ref, lse_ref = O.attention(sub(q), decs[0], decs[1], rows=rows)
    assert_attention_close(o.cpu().numpy()[rows][:, heads], lse.cpu().numpy()[heads][:, rows], o_ref, lse_ref,
                           w.name)
    assert K.kvq_last_device_status() == K.KVQ_OK


def test_joint_decode_full_size_sampled():
    """The joint workload's decoder at full size (32,760 tokens, 12 x 128, rank
    192, INT4 group 32, W_dec = W_enc^T), K and V branches: the oracle's own
    codes of every token are decoded on the GPU; sampled tokens are compared
    with the oracle's decoder within 2^-15 sum_n |c^_n w_ni| (c^ carried as a
    bf16 high part plus a bf16 remainder) plus binary32 rounding."""
    K = _K()
    w = synth.workload("joint")
    H, d, r, G = w.num_heads, w.head_dim, w.joint_rank, w.joint_group
    w_enc = synth.make_orthonormal_encoder(w)
    w_dec = np.ascontiguousarray(w_enc.T)
    wd = _widen(w_dec)
    for which, bits in (("K", w.bits_k), ("V", w.bits_v)):
        x = synth.make_history(w, which)
        T = x.shape[0]
        cent = O.fit(x[: w.num_centroids], w.num_centroids, 0)
        idx_r, codes_r, meta_r, coef_r = O.joint_encode(x, cent, w_enc, bits, G)
        codec = K.Codec(H, d, w.num_centroids, bits, G, r)
        comp = K.Compressed(codec, T, to_dev(cent), to_dev(idx_r.view(np.int16)), to_dev(codes_r),
                            to_dev(meta_r), w_dec=to_dev(w_dec))
        out = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, out)
        torch.cuda.synchronize()
        assert K.kvq_last_device_status() == K.KVQ_OK
        toks = _tiles_sample(T, 1.0 / 16, 14 + bits)
        ref = O.joint_decode(idx_r[:, toks], codes_r[toks], meta_r[toks], cent, w_dec, bits, G)
        s = np.repeat(meta_r[toks][:, :, 0], G, axis=1).astype(np.float64)
        S = (np.abs(coef_r[toks]) + s) @ np.abs(wd)
        bound = ((2.0 ** -15 + (r + 2) * 2.0 ** -24) * S).reshape(len(toks), H, d) + 2.0 ** -23 * np.abs(ref)
        err = np.abs(out.cpu().numpy()[toks].astype(np.float64) - ref)
        assert np.all(err <= bound), f"{which}: decode error {np.max(err / bound):.2f} x bound"


def _widen(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


# ---------------------------------------------------------------------------
# the next rows at the sizes the benchmark times them
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def wan_full():
    w = synth.workload("wan13b")
    return w, synth.make_history(w, "K"), synth.make_history(w, "V"), synth.make_queries(w)


def test_qsac_full_size_sampled(wan_full):
    """QSAC encode (M = 4) of the whole Wan-like K history (32,760 x 12,
    C = 256, INT2 G16, weights from the chunk's queries), bit-exact on a
    seeded 1/16 of the tiles of every head."""
    K = _K()
    w, xk, _, q = wan_full
    T, H, d = xk.shape
    C, G = w.num_centroids, w.group_size
    cent = O.fit(xk[:C], C, 0)
    wts = O.qsac_weights(O.query_moments(q), H, d)
    codec = K.Codec(H, d, C, w.bits_k, G)
    idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
    K.kvq_encode_qsac(codec, to_dev(xk), to_dev(cent), to_dev(wts), idx, codes, meta, M=4)
    assert K.kvq_last_device_status() == K.KVQ_OK
    toks = _tiles_sample(T, 1.0 / 16, 21)
    idx_r, codes_r, meta_r = O.qsac_encode(np.ascontiguousarray(xk[toks]), cent, wts, w.bits_k, G, 4)
    assert np.array_equal(bits_u16(idx).reshape(H, T)[:, toks], idx_r)
    assert np.array_equal(u8(codes).reshape(H, T, d * w.bits_k // 8)[:, toks], codes_r)
    assert np.array_equal(f32_bits(meta).reshape(H, T, d // G, 2)[:, toks], f32_bits(meta_r))


def test_psac_attention_full_size_sampled(wan_full):
    """PSAC attention over the whole Wan-like history in the benchmark's 2
    blocks (split calls, merged by LSE), fed the oracle's coefficients, on 512
    query rows of every head."""
    K = _K()
    w, xk, xv, q = wan_full
    T, H, d = xk.shape
    C, G = w.num_centroids, w.group_size
    comps, decs = [], []
    for x, bits in ((xk, w.bits_k), (xv, w.bits_v)):
        cent = O.fit(x[:C], C, 0)
        codec = K.Codec(H, d, C, bits, G)
        comps.append(_gpu_encode(codec, to_dev(x), cent))
        decs.append(O.decode(*O.encode(x, cent, bits, G), cent, bits, G))
    U = O.psac_basis(O.query_moments(q), 8).astype(np.float32)
    coef = O.psac_coefficients(xk, decs[0], U.astype(np.float64))
    coef_d = to_dev(np.ascontiguousarray(coef.transpose(1, 0, 2)))
    qd, Ud = to_dev(q), to_dev(U)
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, comps[0].codec, T, "cuda", num_queries=q.shape[0])
    edges = [0, T // 2, T]
    parts = []
    for a, b in zip(edges[:-1], edges[1:]):
        o = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
        K.kvq_attention_psac_lse(qd, comps[0], comps[1], Ud, coef_d, o, lse, t_begin=a, t_end=b, workspace=ws)
        parts.append((o, lse))
    om, lm = torch.empty_like(parts[0][0]), torch.empty_like(parts[0][1])
    K.kvq_lse_merge([p[0] for p in parts], [p[1] for p in parts], om, lm)
    assert K.kvq_last_device_status() == K.KVQ_OK
    rows = _rows_sample(q.shape[0], 512, 22)
    o_ref, lse_ref = O.attention_psac(q, decs[0], decs[1], U.astype(np.float64), coef, rows=rows)
    assert_attention_close(om.cpu().numpy()[rows], lm.cpu().numpy()[:, rows], o_ref, lse_ref, "psac full size")


def test_fast_attention_full_size_sampled():
    """NanoKV-Fast on the whole joint workload (32,760 keys, 12 heads, 4,680
    queries, d_low = 64): the GPU decodes both branches into the low space,
    then attends there; 512 query rows of every head against the oracle's
    low-space decode and fast_attention."""
    K = _K()
    w = synth.workload("joint")
    H, d, r, G, C = w.num_heads, w.head_dim, w.joint_rank, w.joint_group, w.num_centroids
    dl = 64
    w_enc = synth.make_orthonormal_encoder(w)
    w_dec = np.ascontiguousarray(w_enc.T)
    q = synth.make_queries(w)
    lows, lows_ref, Ps = [], [], []
    for which, bits in (("K", w.bits_k), ("V", w.bits_v)):
        x = synth.make_history(w, which)
        T = x.shape[0]
        cent = O.fit(x[:C], C, 0)
        idx, codes, meta, _ = O.joint_encode(x, cent, w_enc, bits, G)
        P, W_low, c_low = O.fast_maps_analytical(w_dec, cent, dl)
        Pb, Wb, cb = O.bf16_bits(P), O.bf16_bits(W_low), O.bf16_bits(c_low)
        lows_ref.append(O.bf16_bits(O.joint_decode(idx, codes, meta, cb, Wb, bits, G)))
        comp = K.Compressed(K.Codec(H, dl, C, bits, G, r), T, to_dev(cb), to_dev(idx.view(np.int16)),
                            to_dev(codes), to_dev(meta), w_dec=to_dev(Wb))
        out = torch.empty((T, H, dl), dtype=torch.bfloat16, device="cuda")
        K.kvq_decode(comp, out)
        lows.append(out)
        Ps.append(Pb)
    R = np.ascontiguousarray(np.transpose(Ps[1], (0, 2, 1)))
    o = torch.empty((q.shape[0], H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    K.kvq_fast_attention_lse(to_dev(q), lows[0], lows[1], to_dev(Ps[0]), to_dev(R), o, lse,
                             K.fast_attention_workspace(H, d, dl, q.shape[0], "cuda"))
    assert K.kvq_last_device_status() == K.KVQ_OK
    rows = _rows_sample(q.shape[0], 512, 23)
    o_ref, lse_ref = O.fast_attention(q, lows_ref[0], lows_ref[1], Ps[0], R, rows=rows)
    assert_attention_close(o.cpu().numpy()[rows], lse.cpu().numpy()[:, rows], o_ref, lse_ref, "fast full size")
