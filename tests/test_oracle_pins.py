"""Pins for the CPU oracle: each check ties an oracle function to something
other than itself -- hand-worked examples of the pages' formulas, exact
rational arithmetic, closed forms, invariants, and library routines."""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16(a):
    """float -> bf16 bits via torch (an implementation independent of the oracle)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# distance
# ----------------------------------------------------------------------------

def test_distance_channel_order_golden():
    for case in _golden("distance_order.json")["cases"]:
        got = O.distance(np.array(case["x"], np.float32), np.array(case["mu"], np.float32))
        assert got == np.float32(case["spec"])
        exact = sum((Fraction(a) - Fraction(b)) ** 2 for a, b in zip(case["x"], case["mu"]))
        assert float(exact) == case["exact"]


def test_distance_within_rounding_bound_of_exact():
    rng = np.random.default_rng(1)
    u = 2.0 ** -24
    for _ in range(300):
        d = int(rng.integers(1, 130))
        x = _widen(_bf16(rng.normal(size=d) * rng.uniform(0.1, 10)))
        mu = _widen(_bf16(rng.normal(size=d) * rng.uniform(0.1, 10)))
        exact = sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(x, mu))
        got = Fraction(O.distance(x, mu))
        k = d + 2
        gamma = Fraction(k) * Fraction(u) / (1 - Fraction(k) * Fraction(u))
        assert abs(got - exact) <= gamma * exact


# ----------------------------------------------------------------------------
# assignment
# ----------------------------------------------------------------------------

def test_assign_matches_exact_rational_argmin():
    rng = np.random.default_rng(2)
    checked = 0
    for trial in range(40):
        T, H, d, C = int(rng.integers(1, 64)), int(rng.integers(1, 3)), int(rng.integers(1, 9)), int(rng.integers(1, 9))
        x = _bf16(rng.normal(size=(T, H, d)))
        cent = _bf16(rng.normal(size=(H, C, d)))
        idx = O.assign(x, cent)
        xf, cf = _widen(x), _widen(cent)
        for h in range(H):
            for t in range(T):
                ds = [sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(xf[t, h], cf[h, j]))
                      for j in range(C)]
                best = min(range(C), key=lambda j: (ds[j], j))
                others = [ds[j] for j in range(C) if j != best]
                if others and min(others) - ds[best] <= Fraction(1, 10 ** 5) * (ds[best] + 1):
                    continue  # near tie: the binary32 specification may legitimately differ
                assert idx[h, t] == best
                checked += 1
    assert checked > 500


def test_assign_ties_go_to_lowest_index():
    # duplicated centres and exactly equidistant centres
    x = _bf16(np.array([[[0.0, 0.0]], [[1.0, 1.0]]], np.float32))  # T=2, H=1, d=2
    cent = _bf16(np.array([[[1.0, 0.0], [0.0, 1.0], [1.0, 0.0]]], np.float32))
    idx = O.assign(x, cent)
    assert idx.tolist() == [[0, 0]]
    cent2 = _bf16(np.array([[[5.0, 5.0], [0.0, 1.0], [1.0, 0.0]]], np.float32))
    assert O.assign(x, cent2).tolist() == [[1, 1]]


# ----------------------------------------------------------------------------
# Eq. 1 quantisation and packing
# ----------------------------------------------------------------------------

def test_eq1_worked_examples():
    for g in _golden("eq1_worked_examples.json")["groups"]:
        s, z, q = O.quant_group(np.array(g["r"], np.float32), g["bits"])
        assert s == g["s"] and z == g["z"], g
        assert math.copysign(1.0, z) == math.copysign(1.0, g["z"]), g
        assert q.tolist() == g["q"], g
        dec = [O.dequant(int(c), s, z) for c in q]
        assert dec == g["decoded"], g
        assert O.pack(q, g["bits"]).tolist() == g["packed"], g


def test_quant_error_bound_and_nearest_level():
    rng = np.random.default_rng(3)
    for _ in range(400):
        bits = int(rng.choice([2, 4]))
        G = int(rng.choice([4, 16, 32, 64]))
        r = (rng.standard_t(3, size=G) * rng.uniform(1e-3, 50)).astype(np.float32)
        s, z, q = O.quant_group(r, bits)
        qmax = (1 << bits) - 1
        assert q.min() >= 0 and q.max() <= qmax
        dec = np.array([O.dequant(int(c), s, z) for c in q], np.float64)
        err = np.abs(dec - r.astype(np.float64))
        # rounding to the nearest level leaves at most half a step, plus the
        # binary32 error of forming r*inv, z and (q - z)*s
        slack = 4 * np.finfo(np.float32).eps * (np.abs(r).max() + s * (qmax + abs(z)))
        assert np.all(err <= s / 2 + slack)
        # every code is (one of) the nearest representable level(s)
        levels = (np.arange(qmax + 1) - z) * np.float64(s)
        best = np.min(np.abs(levels[None, :] - r.astype(np.float64)[:, None]), axis=1)
        assert np.all(err <= best + slack)
        # the group's extremes land on the end codes (generic data)
        if np.ptp(r) > 0:
            assert q[np.argmin(r)] == 0 and q[np.argmax(r)] == qmax


def test_pack_layout_and_roundtrip():
    assert O.pack(np.array([0, 1, 2, 3], np.uint8), 2).tolist() == [0xE4]
    assert O.pack(np.array([3, 10], np.uint8), 4).tolist() == [0xA3]
    rng = np.random.default_rng(4)
    for bits in (2, 4):
        q = rng.integers(0, 1 << bits, size=128).astype(np.uint8)
        b = O.pack(q, bits)
        assert b.shape == (128 * bits // 8,)
        assert np.array_equal(O.unpack(b, 128, bits), q)
        # independent unpack with numpy bit arithmetic
        per = 8 // bits
        manual = np.array([(b[c // per] >> ((c % per) * bits)) & ((1 << bits) - 1) for c in range(128)])
        assert np.array_equal(manual, q)


# ----------------------------------------------------------------------------
# storage accounting vs figures printed on the pages
# ----------------------------------------------------------------------------

def test_storage_ratios_printed_on_pages():
    g = _golden("storage_ratios.json")
    for row in g["rtn"]:
        assert round(O.compression_ratio(row["bits"], row["group"], row["meta_bits"]), 2) == row["ratio"]
    for row in g["bits_per_value"]:
        assert O.bits_per_value(row["bits"], row["group"], row["meta_bits"]) == row["value"]
    for row in g["joint_nominal"]:
        assert O.joint_nominal_ratio(row["heads"] * row["head_dim"], row["rank"]) == row["ratio"]
    # the joint workload: 12 heads x 128 channels, rank 192 -> 32x nominal
    assert O.joint_nominal_ratio(1536, 192) == 32
    # per token-head bytes of the stored format: 128 ch, INT2, group 16:
    # 32 B codes + 8 groups x 8 B {s, z} + 2 B index
    assert O.stored_bytes_per_token_head(128, 2, 16) == 98


# ----------------------------------------------------------------------------
# encode / decode
# ----------------------------------------------------------------------------

def test_identical_tokens_collapse_to_centre():
    rng = np.random.default_rng(5)
    H, d, T, C = 2, 64, 40, 4
    tok = _bf16(rng.normal(size=(H, d)))
    x = np.broadcast_to(tok[None], (T, H, d)).copy()
    cent = O.fit(x, C, 3)
    for h in range(H):
        for j in range(C):
            assert np.array_equal(cent[h, j], tok[h])
    idx, codes, meta = O.encode(x, cent, 2, 32)
    assert np.all(idx == 0)
    assert np.all(codes == 0)
    assert np.all(meta == 0.0)
    dec = O.decode(idx, codes, meta, cent, 2, 32)
    assert np.array_equal(dec, np.broadcast_to(_widen(tok)[None], (T, H, d)))


def test_zero_centre_reduces_to_plain_groupwise_rtn():
    rng = np.random.default_rng(6)
    T, H, d, G = 33, 3, 64, 16
    x = _bf16(rng.normal(size=(T, H, d)) * 3)
    cent = np.zeros((H, 1, d), np.uint16)
    idx, codes, meta = O.encode(x, cent, 4, G)
    assert np.all(idx == 0)
    xf = _widen(x)
    for h in range(H):
        c2, m2 = O.quant_rows(np.ascontiguousarray(xf[:, h, :]), 4, G)
        assert np.array_equal(codes[h], c2)
        assert np.array_equal(meta[h], m2)


def test_encode_decode_error_bound_and_residual_form():
    rng = np.random.default_rng(7)
    T, H, d, C, G = 200, 2, 64, 8, 16
    x = _bf16(rng.normal(size=(T, H, d)) * 2)
    cent = O.fit(x, C, 2)
    for bits in (2, 4):
        idx, codes, meta = O.encode(x, cent, bits, G)
        assert np.array_equal(idx, O.assign(x, cent))
        dec = O.decode(idx, codes, meta, cent, bits, G)
        xf = _widen(x).astype(np.float64)
        s = np.repeat(meta[..., 0], G, axis=2)  # [H][T][d]
        s = np.transpose(s, (1, 0, 2))
        err = np.abs(dec - xf)
        assert np.all(err <= s / 2 + 1e-5 * (np.abs(xf) + 1))
        # the decoded vector is centre + dequantised residual: removing the
        # centre leaves a value on the group's quantisation grid
        cf = _widen(cent).astype(np.float64)
        mu = np.stack([cf[h][idx[h]] for h in range(H)], axis=1)  # [T][H][d]
        z = np.transpose(np.repeat(meta[..., 1], G, axis=2), (1, 0, 2))
        with np.errstate(divide="ignore", invalid="ignore"):
            lvl = np.where(s > 0, (dec - mu) / s + z, 0.0)
        assert np.all(np.abs(lvl - np.round(lvl)) < 1e-3)
        assert np.all((np.round(lvl) >= -1e-9) & (np.round(lvl) <= (1 << bits) - 1))


def test_decode_uses_each_stored_field():
    """Hand-built encoded form: decode = centre + (q - z) s per group."""
    H, T, d, C, G, bits = 1, 2, 8, 2, 4, 2
    cent = _bf16(np.array([[[1, 2, 3, 4, 5, 6, 7, 8], [-1, -1, -1, -1, 0.5, 0.5, 0.5, 0.5]]], np.float32))
    idx = np.array([[1, 0]], np.uint16)
    q = np.array([[0, 1, 2, 3, 3, 2, 1, 0], [1, 1, 1, 1, 0, 0, 0, 0]], np.uint8)
    codes = np.stack([O.pack(q[t], bits) for t in range(T)])[None]
    meta = np.array([[[[0.5, 1.0], [2.0, 0.0]], [[0.25, 2.0], [1.0, -1.0]]]], np.float32)
    dec = O.decode(idx, codes, meta, cent, bits, G)
    want_t0 = [-1 + (0 - 1) * 0.5, -1 + 0, -1 + 0.5, -1 + 1.0, 0.5 + 6, 0.5 + 4, 0.5 + 2, 0.5 + 0]
    want_t1 = [1 + (1 - 2) * 0.25, 2 - 0.25, 3 - 0.25, 4 - 0.25, 5 + 1, 6 + 1, 7 + 1, 8 + 1]
    assert dec[0, 0].tolist() == want_t0
    assert dec[1, 0].tolist() == want_t1


# ----------------------------------------------------------------------------
# k-means fitting
# ----------------------------------------------------------------------------

def test_fit_seeds_from_first_tokens():
    rng = np.random.default_rng(8)
    x = rng.normal(size=(50, 2, 16)).astype(np.float32)
    cent = O.fit(x, 5, 0)
    for h in range(2):
        assert np.array_equal(cent[h], _bf16(x[:5, h, :]))


def test_fit_recovers_planted_centres_with_exact_update():
    rng = np.random.default_rng(9)
    H, d, C, per = 2, 32, 6, 40
    planted = (rng.integers(-8, 9, size=(H, C, d)) * 4).astype(np.float64)
    members = []
    for j in range(C):
        members.append(planted[:, j, :][None] + rng.normal(0, 0.05, size=(per, H, d)))
    # first C tokens: one per blob, so the seeds land in distinct blobs
    first = np.stack([m[0] for m in members])
    rest = np.concatenate([m[1:] for m in members])
    order = rng.permutation(rest.shape[0])
    x = _bf16(np.concatenate([first, rest[order]]).astype(np.float32))
    blob = np.concatenate([np.arange(C), np.repeat(np.arange(C), per - 1)[order]])
    cent = O.fit(x, C, 1)
    xf = _widen(x).astype(np.float64)
    for h in range(H):
        for j in range(C):
            mean = xf[blob == j, h, :].mean(axis=0)
            assert np.array_equal(cent[h, j], _bf16(mean.astype(np.float32)))


def test_fit_inertia_non_increasing_up_to_centre_rounding():
    rng = np.random.default_rng(10)
    x = _bf16(rng.normal(size=(400, 2, 32)))
    iters = 5
    cent, inertia = O.fit(x, 12, iters, return_inertia=True)
    xmax = float(np.abs(_widen(x)).max())
    # rounding a mean to bf16 moves it by <= 2^-8 relative per channel; by the
    # parallel-axis identity that can add at most sum_j n_j |mu_j - mean_j|^2
    bound = 400 * 32 * (2.0 ** -8 * xmax) ** 2
    for h in range(2):
        for i in range(iters):
            assert inertia[h, i + 1] <= inertia[h, i] + bound
        assert inertia[h, -1] < inertia[h, 0]


def test_fit_c_equals_t_each_point_is_its_centre():
    rng = np.random.default_rng(11)
    T = 24
    x = _bf16(rng.normal(size=(T, 1, 8)))
    cent, inertia = O.fit(x, T, 3, return_inertia=True)
    assert np.array_equal(cent[0], x[:, 0, :])
    assert inertia[0, -1] == 0.0


def test_fit_empty_cluster_keeps_centre():
    # tokens 0 and 1 identical -> seeds 0 and 1 coincide and, by the
    # lowest-index tie rule, centre 1 receives no token in the first round
    x = np.array([[[1.0, 1.0]], [[1.0, 1.0]], [[5.0, 5.0]], [[1.5, 1.0]], [[5.5, 5.0]]], np.float32)
    cent = O.fit(x, 3, 1)
    assert _widen(cent[0, 1]).tolist() == [1.0, 1.0]          # empty: kept
    assert _widen(cent[0, 0]).tolist() == [1.1640625, 1.0]    # bf16(3.5/3)
    assert _widen(cent[0, 2]).tolist() == [5.25, 5.0]
    # second round: tokens 0 and 1 now sit exactly on centre 1
    cent = O.fit(x, 3, 2)
    assert _widen(cent[0, 0]).tolist() == [1.5, 1.0]
    assert _widen(cent[0, 1]).tolist() == [1.0, 1.0]
    assert _widen(cent[0, 2]).tolist() == [5.25, 5.0]


# ----------------------------------------------------------------------------
# joint head-channel path
# ----------------------------------------------------------------------------

def test_joint_identity_encoder_is_channel_quantisation():
    rng = np.random.default_rng(12)
    T, H, d, C, r, G = 20, 3, 64, 4, 96, 32
    x = _bf16(rng.normal(size=(T, H, d)))
    cent = O.fit(x, C, 1)
    w = np.zeros((H * d, r), np.float32)
    w[np.arange(r), np.arange(r)] = 1.0
    idx, codes, meta, coef = O.joint_encode(x, cent, _bf16(w), 4, G)
    assert np.array_equal(idx, O.assign(x, cent))
    xf, cf = _widen(x), _widen(cent)
    res = np.stack([xf[:, h, :] - cf[h][idx[h]] for h in range(H)], axis=1).reshape(T, H * d)
    want = _widen(_bf16(res[:, :r]))
    assert np.array_equal(coef, want)
    c2, m2 = O.quant_rows(coef, 4, G)
    assert np.array_equal(codes, c2) and np.array_equal(meta, m2)


def test_joint_decode_is_projection_when_coefficients_are_on_grid():
    rng = np.random.default_rng(13)
    T, H, d, C, r, G = 10, 2, 64, 3, 64, 32
    cent = _bf16(rng.normal(size=(H, C, d)))
    idx = rng.integers(0, C, size=(H, T)).astype(np.uint16)
    coef = rng.integers(-7, 8, size=(T, r)).astype(np.float32)
    for t in range(T):  # force a full 15-step span in every group -> s = 1
        for g in range(r // G):
            coef[t, g * G] = -7.0
            coef[t, g * G + 1] = 8.0
    codes, meta = O.quant_rows(coef, 4, G)
    assert np.all(meta[..., 0] == 1.0)
    rng2 = np.random.default_rng(14)
    q_, _ = np.linalg.qr(rng2.normal(size=(H * d, r)))
    w_dec = _bf16(q_.T)
    out = O.joint_decode(idx, codes, meta, cent, w_dec, 4, G)
    proj = coef.astype(np.float64) @ _widen(w_dec).astype(np.float64)  # [T][H*d]
    cf = _widen(cent).astype(np.float64)
    want = np.stack([cf[h][idx[h]] for h in range(H)], axis=1) + proj.reshape(T, H, d)
    assert np.max(np.abs(out - want)) < 1e-5 * (np.abs(want).max() + 1)


# ----------------------------------------------------------------------------
# attention and log-sum-exp merging
# ----------------------------------------------------------------------------

def test_attention_single_key_returns_its_value():
    rng = np.random.default_rng(15)
    q = _bf16(rng.normal(size=(5, 2, 64)))
    k = rng.normal(size=(1, 2, 64)).astype(np.float32)
    v = rng.normal(size=(1, 2, 64)).astype(np.float32)
    o, lse = O.attention(q, k, v)
    qf = _widen(q).astype(np.float64)
    for h in range(2):
        assert np.allclose(o[:, h, :], v[0, h][None], rtol=0, atol=1e-15)
        want = qf[:, h, :] @ k[0, h].astype(np.float64) / 8.0
        assert np.allclose(lse[h], want, rtol=1e-14, atol=1e-14)


def test_attention_identical_keys_mean_value_and_log_n():
    rng = np.random.default_rng(16)
    n = 7
    q = _bf16(rng.normal(size=(3, 1, 64)))
    k = np.broadcast_to(rng.normal(size=(1, 1, 64)).astype(np.float32), (n, 1, 64)).copy()
    v = rng.normal(size=(n, 1, 64)).astype(np.float32)
    o, lse = O.attention(q, k, v)
    s = _widen(q)[:, 0, :].astype(np.float64) @ k[0, 0].astype(np.float64) / 8.0
    assert np.allclose(o[:, 0, :], v[:, 0, :].astype(np.float64).mean(axis=0)[None], atol=1e-14)
    assert np.allclose(lse[0], s + math.log(n), atol=1e-13)


def test_attention_two_keys_logistic():
    rng = np.random.default_rng(17)
    q = _bf16(rng.normal(size=(4, 1, 64)))
    k = rng.normal(size=(2, 1, 64)).astype(np.float32)
    v = rng.normal(size=(2, 1, 64)).astype(np.float32)
    o, lse = O.attention(q, k, v)
    qf = _widen(q).astype(np.float64)
    for i in range(4):
        s1 = float(qf[i, 0] @ k[0, 0].astype(np.float64)) / 8.0
        s2 = float(qf[i, 0] @ k[1, 0].astype(np.float64)) / 8.0
        w1 = 1.0 / (1.0 + math.exp(s2 - s1))
        want = w1 * v[0, 0].astype(np.float64) + (1 - w1) * v[1, 0].astype(np.float64)
        assert np.allclose(o[i, 0], want, atol=1e-14)
        assert abs(lse[0, i] - (max(s1, s2) + math.log1p(math.exp(-abs(s1 - s2))))) < 1e-13


def test_attention_matches_library_sdpa_and_logsumexp():
    from scipy.special import logsumexp

    rng = np.random.default_rng(18)
    Tq, T, H, d = 37, 300, 3, 64
    q = _bf16(rng.normal(size=(Tq, H, d)))
    k = rng.normal(size=(T, H, d)).astype(np.float32)
    v = rng.normal(size=(T, H, d)).astype(np.float32)
    o, lse = O.attention(q, k, v)
    qt = torch.from_numpy(_widen(q).astype(np.float64)).permute(1, 0, 2)
    kt = torch.from_numpy(k.astype(np.float64)).permute(1, 0, 2)
    vt = torch.from_numpy(v.astype(np.float64)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(1, 0, 2).numpy()
    assert np.max(np.abs(o - ref)) < 1e-12
    s = np.einsum("qhd,khd->hqk", _widen(q).astype(np.float64), k.astype(np.float64)) / math.sqrt(d)
    assert np.max(np.abs(lse - logsumexp(s, axis=2))) < 1e-12


def test_merge_of_split_history_equals_unsplit():
    rng = np.random.default_rng(19)
    Tq, T, H, d = 20, 333, 2, 64
    q = _bf16(rng.normal(size=(Tq, H, d)))
    k = (rng.normal(size=(T, H, d)) * 2).astype(np.float32)
    v = rng.normal(size=(T, H, d)).astype(np.float32)
    o_full, lse_full = O.attention(q, k, v)
    cuts = [0, 1, 100, 101, 250, T]
    parts = [O.attention(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = O.lse_merge([p[0] for p in parts], [p[1] for p in parts])
    assert np.max(np.abs(o - o_full)) < 1e-12
    assert np.max(np.abs(lse - lse_full)) < 1e-12


def test_merge_with_empty_parts():
    rng = np.random.default_rng(20)
    o1 = rng.normal(size=(5, 2, 8))
    l1 = rng.normal(size=(2, 5))
    o_empty, l_empty = O.attention(_bf16(rng.normal(size=(5, 2, 8))), np.zeros((0, 2, 8), np.float32),
                                   np.zeros((0, 2, 8), np.float32))
    assert np.all(l_empty == -np.inf) and np.all(o_empty == 0)
    o, l = O.lse_merge([o1, o_empty], [l1, l_empty])
    assert np.allclose(o, o1, atol=1e-15) and np.allclose(l, l1, atol=1e-15)
    o, l = O.lse_merge([o_empty, o_empty], [l_empty, l_empty])
    assert np.all(l == -np.inf) and np.all(o == 0)


# ----------------------------------------------------------------------------
# full-layer attention: compressed history + uncompressed current chunk
# ----------------------------------------------------------------------------

def test_layer_attention_matches_library_sdpa_over_all_keys():
    """One softmax over history and chunk keys: torch's SDPA over the union
    (chunk keys first, history after -- a different order from the oracle's)
    and scipy's logsumexp of the logits."""
    from scipy.special import logsumexp

    rng = np.random.default_rng(21)
    Tq, T, Tc, H, d = 29, 211, 45, 3, 64
    q = _bf16(rng.normal(size=(Tq, H, d)))
    kh = (rng.normal(size=(T, H, d)) * 1.5).astype(np.float32)
    vh = rng.normal(size=(T, H, d)).astype(np.float32)
    kc = _bf16(rng.normal(size=(Tc, H, d)) * 1.5)
    vc = _bf16(rng.normal(size=(Tc, H, d)))
    o, lse = O.layer_attention(q, kh, vh, kc, vc)
    kall = np.concatenate([_widen(kc), kh]).astype(np.float64)
    vall = np.concatenate([_widen(vc), vh]).astype(np.float64)
    qt = torch.from_numpy(_widen(q).astype(np.float64)).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(kall).permute(1, 0, 2), torch.from_numpy(vall).permute(1, 0, 2)).permute(1, 0, 2)
    assert np.max(np.abs(o - ref.numpy())) < 1e-12
    s = np.einsum("qhd,khd->hqk", _widen(q).astype(np.float64), kall) / math.sqrt(d)
    assert np.max(np.abs(lse - logsumexp(s, axis=2))) < 1e-12


def test_layer_attention_reads_chunk_as_bf16_and_handles_empty_sets():
    rng = np.random.default_rng(22)
    Tq, T, Tc, H, d = 9, 40, 17, 2, 64
    q = _bf16(rng.normal(size=(Tq, H, d)))
    kh = rng.normal(size=(T, H, d)).astype(np.float32)
    vh = rng.normal(size=(T, H, d)).astype(np.float32)
    kc = _bf16(rng.normal(size=(Tc, H, d)))
    vc = _bf16(rng.normal(size=(Tc, H, d)))
    # bf16 bits and the same values as float32 give the same result
    o1, l1 = O.layer_attention(q, kh, vh, kc, vc)
    o2, l2 = O.layer_attention(q, kh, vh, _widen(kc), _widen(vc))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # empty chunk: the history alone; empty history: the chunk alone
    none = np.zeros((0, H, d), np.float32)
    oh, lh = O.layer_attention(q, kh, vh, none, none)
    oa, la = O.attention(q, kh, vh)
    assert np.array_equal(oh, oa) and np.array_equal(lh, la)
    oc, lc = O.layer_attention(q, none, none, kc, vc)
    s = np.einsum("qhd,khd->hqk", _widen(q).astype(np.float64), _widen(kc).astype(np.float64)) / 8.0
    m = s.max(axis=2, keepdims=True)
    assert np.allclose(lc, (m + np.log(np.exp(s - m).sum(axis=2, keepdims=True)))[..., 0], atol=1e-13)
    # both empty: O = 0, lse = -inf
    oz, lz = O.layer_attention(q, none, none, none, none)
    assert np.all(oz == 0) and np.all(lz == -np.inf)


def test_layer_attention_is_the_merge_of_history_and_chunk():
    """Splitting the keys into the history part and the chunk part and
    merging by LSE gives the layer result (the identity the GPU path uses)."""
    rng = np.random.default_rng(23)
    Tq, T, Tc, H, d = 12, 130, 33, 2, 128
    q = _bf16(rng.normal(size=(Tq, H, d)))
    kh = (rng.normal(size=(T, H, d)) * 2).astype(np.float32)
    vh = rng.normal(size=(T, H, d)).astype(np.float32)
    kc = _bf16(rng.normal(size=(Tc, H, d)) * 2)
    vc = _bf16(rng.normal(size=(Tc, H, d)))
    o, lse = O.layer_attention(q, kh, vh, kc, vc)
    ph = O.attention(q, kh, vh)
    pc = O.attention(q, kc, vc)
    om, lm = O.lse_merge([ph[0], pc[0]], [ph[1], pc[1]])
    assert np.max(np.abs(o - om)) < 1e-12 and np.max(np.abs(lse - lm)) < 1e-12


# ----------------------------------------------------------------------------
# QuantWM: query-sensitive centre selection (QSAC), principal-subspace logit
# correction (PSAC)
# ----------------------------------------------------------------------------

def test_qsac_worked_example():
    g = _golden("qsac_worked_example.json")
    x = np.array(g["x"], np.float32)
    cent = _bf16(np.array(g["centres"], np.float32))[None]          # [1][C][d]
    G = g["group"]
    for case in g["cases"]:
        w = np.array(case["w"], np.float32)
        mus = _widen(cent[0])
        assert [O.weighted_distance(x, mu, w) for mu in mus] == case["distance"]
        assert [O.qsac_score(x - mu, w, G) for mu in mus] == case["score"]
        for M, want in case["choice"].items():
            idx, cand = O.qsac_assign(x[None, None], cent, w[None], G, int(M), return_candidates=True)
            assert int(idx[0, 0]) == want, (case["note"], M)
            ranked = [int(c) for c in cand[0, 0] if c >= 0]
            assert ranked == [j for j in np.argsort(case["rank"])][: min(int(M), 3)]


def test_qsac_unit_weights_one_candidate_is_plain_nearest_centre():
    """w = 1 and M = 1 reduce QSAC to the plain nearest-centre encode."""
    rng = np.random.default_rng(31)
    x = _bf16(rng.normal(size=(400, 3, 64)) * rng.uniform(0.5, 2, size=(1, 3, 64)))
    cent = O.fit(x[:32], 32, 0)
    w = O.qsac_weights(None, 3, 64)
    assert np.array_equal(O.qsac_assign(x, cent, w, 16, 1), O.assign(x, cent))
    for a, b in zip(O.qsac_encode(x, cent, w, 2, 16, 1), O.encode(x, cent, 2, 16)):
        assert np.array_equal(a, b)


def test_qsac_against_exact_rational_selection():
    """Candidates and choice against exact rational arithmetic (tiny random
    problems; cases whose exact values come within 1e-4 relative of a tie are
    skipped, since binary32 may then order them either way)."""
    rng = np.random.default_rng(32)
    checked = 0
    for trial in range(40):
        d, G, C, M = 8, 4, 6, 3
        x = rng.normal(size=d).astype(np.float32)
        mus = _widen(_bf16(rng.normal(size=(C, d))))
        w = rng.uniform(0.1, 4.0, size=d).astype(np.float32)
        X = [Fraction(float(v)) for v in x]
        W = [Fraction(float(v)) for v in w]
        D = [sum(W[c] * (X[c] - Fraction(float(mu[c]))) ** 2 for c in range(d)) for mu in mus]
        order = sorted(range(C), key=lambda j: (D[j], j))
        gaps = [abs(D[order[k + 1]] - D[order[k]]) / max(D[order[k]], Fraction(1, 10 ** 9)) for k in range(M)]
        if min(gaps) < Fraction(1, 10 ** 4):
            continue
        S = {}
        for j in order[:M]:
            r = [X[c] - Fraction(float(mus[j][c])) for c in range(d)]
            S[j] = sum(sum(W[g * G:(g + 1) * G]) * (max(r[g * G:(g + 1) * G]) - min(r[g * G:(g + 1) * G])) ** 2
                       for g in range(d // G))
        best = min(order[:M], key=lambda j: (S[j], order.index(j)))
        others = [S[j] for j in order[:M] if j != best]
        if others and min(abs(s - S[best]) for s in others) < Fraction(1, 10 ** 4) * max(S[best], Fraction(1)):
            continue
        idx, cand = O.qsac_assign(x[None, None], _bf16(mus)[None], w[None], G, M, return_candidates=True)
        assert [int(c) for c in cand[0, 0]] == order[:M]
        assert int(idx[0, 0]) == best
        checked += 1
    assert checked >= 25


def test_qsac_power_of_two_weight_scaling_keeps_the_choice():
    rng = np.random.default_rng(33)
    x = _bf16(rng.normal(size=(200, 2, 32)))
    cent = O.fit(x[:16], 16, 0)
    w = rng.uniform(0.2, 3.0, size=(2, 32)).astype(np.float32)
    base = O.qsac_assign(x, cent, w, 16, 4)
    for k in (-3, 5):
        assert np.array_equal(O.qsac_assign(x, cent, (w * np.float32(2.0 ** k)).astype(np.float32), 16, 4), base)


def test_query_moments_and_weights_closed_form():
    """Queries along coordinate axes: M_h is diagonal with the mean squares;
    the QSAC weights are that diagonal; no statistics gives unit weights."""
    n, H, d = 6, 2, 4
    q = np.zeros((n, H, d), np.float32)
    for t in range(n):
        q[t, :, t % d] = t + 1.0
    M = O.query_moments(q)
    want = np.zeros((H, d))
    for t in range(n):
        want[:, t % d] += (t + 1.0) ** 2 / n
    assert np.allclose(M, np.stack([np.diag(want[h]) for h in range(H)]), atol=0, rtol=1e-15)
    assert np.array_equal(O.qsac_weights(M, H, d), want.astype(np.float32))
    assert np.array_equal(O.qsac_weights(None, H, d), np.ones((H, d), np.float32))


def _psac_case(seed, r):
    rng = np.random.default_rng(seed)
    Tq, T, H, d = 12, 80, 2, 16
    q_hist = _bf16(rng.normal(size=(300, H, d)) * np.linspace(3, 0.2, d)[None, None])
    q = _bf16(rng.normal(size=(Tq, H, d)))
    k = _bf16(rng.normal(size=(T, H, d)))
    k_hat = (_widen(k) + rng.normal(size=(T, H, d)).astype(np.float32) * 0.1).astype(np.float32)
    v = rng.normal(size=(T, H, d)).astype(np.float32)
    M = O.query_moments(q_hist)
    U = O.psac_basis(M, r)
    return q, k, k_hat, v, M, U


def test_psac_basis_is_the_principal_query_subspace():
    q, k, k_hat, v, M, U = _psac_case(34, 5)
    for h in range(M.shape[0]):
        assert np.allclose(U[h].T @ U[h], np.eye(5), atol=1e-12)
        lam = np.einsum("dr,de,er->r", U[h], M[h], U[h])
        assert np.all(np.diff(lam) <= 1e-12)                          # decreasing
        assert np.allclose(M[h] @ U[h], U[h] * lam[None], atol=1e-10)  # eigenvectors
        top = np.sort(np.linalg.eigvalsh(M[h]))[::-1][:5]
        assert np.allclose(lam, top, rtol=1e-12)
        assert np.all(U[h][np.argmax(np.abs(U[h]), axis=0), np.arange(5)] > 0)


def test_psac_full_rank_restores_the_exact_logits():
    """r = d: k^ + U U^T (k - k^) = k, so the corrected attention is the
    attention over the original keys (up to the binary32 storage of C)."""
    q, k, k_hat, v, M, U = _psac_case(35, 16)
    coef = O.psac_coefficients(k, k_hat, U)
    o, lse = O.attention_psac(q, k_hat, v, U, coef)
    o_ref, lse_ref = O.attention(q, k, v)
    assert np.max(np.abs(o - o_ref)) < 1e-5 and np.max(np.abs(lse - lse_ref)) < 1e-5


def test_psac_rank_zero_and_queries_in_the_subspace():
    """r = 0 leaves the plain attention over k^; a query inside span(U_r) sees
    its exact logits q . k, whatever the error outside that span."""
    q, k, k_hat, v, M, U = _psac_case(36, 4)
    Tq, H, d = q.shape
    o0, l0 = O.attention_psac(q, k_hat, v, U[:, :, :0], O.psac_coefficients(k, k_hat, U[:, :, :0]))
    oa, la = O.attention(q, k_hat, v)
    assert np.array_equal(o0, oa) and np.array_equal(l0, la)
    a = np.random.default_rng(37).normal(size=(Tq, H, 4))
    q_in = np.einsum("hdr,thr->thd", U, a)                              # queries in span(U_r), float64
    coef = O.psac_coefficients(k, k_hat, U)
    o, lse = O.attention_psac(q_in, k_hat, v, U, coef)
    o_ref, lse_ref = O.attention(q_in, k, v)
    assert np.max(np.abs(lse - lse_ref)) < 1e-5 and np.max(np.abs(o - o_ref)) < 1e-5


def test_qsac_ties_follow_index_order():
    """Three centres at the same weighted distance and with the same score:
    they rank by index and the lowest index is chosen."""
    x = np.zeros((1, 1, 4), np.float32)
    cent = _bf16(np.eye(4, dtype=np.float32)[:3])[None]
    w = np.ones((1, 4), np.float32)
    idx, cand = O.qsac_assign(x, cent, w, 2, 3, return_candidates=True)
    assert [int(c) for c in cand[0, 0]] == [0, 1, 2] and int(idx[0, 0]) == 0
    idx, cand = O.qsac_assign(x, cent[:, ::-1].copy(), w, 2, 2, return_candidates=True)
    assert [int(c) for c in cand[0, 0]] == [0, 1] and int(idx[0, 0]) == 0

# ----------------------------------------------------------------------------
# compact 16-bit {s, z} (TempoKV, Table 1: b + 1 bits per value at G = 32)
# ----------------------------------------------------------------------------

def test_bf16_round_matches_torch_and_hand_cases():
    """binary32 -> bf16 (centres, joint residual): torch's conversion is an
    independent round-to-nearest-even implementation; they agree on random
    values over the whole exponent range, on exact ties, subnormals and on
    overflow to infinity.  Hand cases: 1 + 2^-8 is a tie and goes to the even
    neighbour 1.0 (0x3f80); 1 + 3 2^-8 goes up to 1 + 2^-6 (0x3f82); -0 keeps
    its sign; a NaN stays a NaN."""
    rng = np.random.default_rng(67)
    mant = rng.integers(0, 1 << 23, size=6000, dtype=np.uint32)
    expo = rng.integers(0, 255, size=6000, dtype=np.uint32)
    sign = rng.integers(0, 2, size=6000, dtype=np.uint32)
    u = (sign << 31) | (expo << 23) | mant
    ties = (rng.integers(0, 1 << 16, size=2000, dtype=np.uint32) << 16) | np.uint32(0x8000)
    ties = ties[((ties >> 23) & 0xFF) != 0xFF]
    vals = np.concatenate([u, ties]).view(np.float32)
    want = torch.from_numpy(vals.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.bf16_round(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want), f"differs at {vals[got != want][:5]}"
    assert O.bf16_round(1.0 + 2.0 ** -8) == 0x3F80
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert O.bf16_round(-0.0) == 0x8000
    assert O.bf16_round(3.4e38) == 0x7F80                      # rounds past the largest bf16
    nan = O.bf16_round(float("nan"))
    assert (nan & 0x7F80) == 0x7F80 and (nan & 0x007F) != 0


def test_f16_round_golden():
    g = _golden("eq1_f16_worked_examples.json")
    for case in g["round"]:
        assert O.f16_round(case["f"]) == case["h"], case["note"]


def test_f16_round_matches_numpy_in_range():
    """numpy's float16 conversion (round to nearest even, gradual underflow)
    is an independent implementation; they agree wherever numpy does not
    overflow, and numpy's widening agrees on every finite pattern."""
    rng = np.random.default_rng(61)
    vals = np.concatenate([
        rng.normal(size=4000) * 10.0 ** rng.uniform(-9, 4.8, size=4000),
        (rng.integers(0, 4096, size=2000) + rng.choice([0.25, 0.5, 0.75], size=2000)) * 2.0 ** -24,
        rng.uniform(-65519, 65519, size=2000),
    ]).astype(np.float32)
    vals = vals[np.abs(vals) < 65520.0]  # numpy rounds these to infinity; the oracle saturates
    want = vals.astype(np.float16).view(np.uint16)
    got = np.array([O.f16_round(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want), f"differs at {vals[got != want][:5]}"
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    fin = np.isfinite(bits.view(np.float16))
    widened = np.array([O.f16_widen(int(b)) for b in bits[fin]], np.float32)
    assert np.array_equal(widened.view(np.uint32), bits[fin].view(np.float16).astype(np.float32).view(np.uint32))


def test_eq1_f16_worked_examples():
    g = _golden("eq1_f16_worked_examples.json")
    for case in g["groups"]:
        s16, z16, q = O.quant_group16(np.array(case["r"], np.float32), case["bits"])
        assert (s16, z16) == (case["s16"], case["z16"]), case["note"]
        assert q.tolist() == case["q"], case["note"]
        dec = [O.dequant(int(qq), O.f16_widen(s16), O.f16_widen(z16)) for qq in q]
        assert dec == case["decoded"], case["note"]


def test_eq1_f16_error_bound():
    """For groups whose zero point is stored exactly (min <= 0 <= max keeps it
    in [0, 2^b - 1]), every residual decodes within s16/2 + (2^b - 1)|s - s16|
    (the grid of the rounded scale may stop short of max) plus binary32
    rounding."""
    rng = np.random.default_rng(62)
    for trial in range(400):
        bits = (2, 4)[trial % 2]
        G = (16, 32, 64)[trial % 3]
        r = (rng.normal(size=G) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        r[0], r[1] = -abs(r[0]), abs(r[1])
        s16, z16, q = O.quant_group16(r, bits)
        s_exact = (np.float32(r.max()) - np.float32(r.min())) / np.float32((1 << bits) - 1)
        sf, zf = O.f16_widen(s16), O.f16_widen(z16)
        assert zf == np.rint(zf) and 0 <= zf <= (1 << bits) - 1
        dec = np.array([O.dequant(int(qq), sf, zf) for qq in q], np.float64)
        bound = sf / 2 + ((1 << bits) - 1) * abs(float(s_exact) - sf) + 4 * np.spacing(np.abs(r).max())
        assert np.all(np.abs(dec - r.astype(np.float64)) <= bound)


def test_eq1_f16_equals_binary32_codec_when_scale_is_a_half():
    """Groups whose binary32 scale is itself a binary16 value and whose zero
    point is small: the compact codec stores the same s and z and the same
    codes as the binary32 one."""
    rng = np.random.default_rng(63)
    for trial in range(200):
        bits = (2, 4)[trial % 2]
        qmax = (1 << bits) - 1
        s = np.float32(np.float16(2.0 ** rng.integers(-8, 4) * rng.integers(1, 1024) / 512.0))
        mn = -np.float32(rng.integers(0, qmax + 1)) * s
        r = (mn + rng.integers(0, qmax * 4 + 1, size=32).astype(np.float32) * s / np.float32(4.0)).astype(np.float32)
        r[0], r[1] = mn, mn + np.float32(qmax) * s
        if np.float32(r.max() - r.min()) / np.float32(qmax) != s:
            continue
        s32, z32, q32 = O.quant_group(r, bits)
        s16, z16, q16 = O.quant_group16(r, bits)
        assert O.f16_widen(s16) == s32 and O.f16_widen(z16) == z32
        assert np.array_equal(q16, q32)


def test_encode16_decode16_storage_and_bound():
    """The compact codec on a history: the same centre indices as the binary32
    codec, half the metadata bytes (4 per group against 8), and every value
    decoded within the per-group bound of the compact quantiser."""
    rng = np.random.default_rng(64)
    T, H, d, C = 300, 2, 64, 8
    x = synth.bf16_bits_from_f64(rng.normal(size=(T, H, d)) * rng.uniform(0.5, 3, size=(1, H, d)))
    cent = O.fit(x, C, 2)
    for bits, G in ((2, 16), (4, 32)):
        idx, codes, meta = O.encode(x, cent, bits, G)
        idx16, codes16, meta16 = O.encode16(x, cent, bits, G)
        assert np.array_equal(idx16, idx)
        assert meta16.nbytes * 2 == meta.nbytes
        dec = O.decode16(idx16, codes16, meta16, cent, bits, G).astype(np.float64)
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)
        s32 = meta[..., 0].astype(np.float64)
        s16 = np.vectorize(O.f16_widen)(meta16[..., 0]).astype(np.float64)
        z16 = np.vectorize(O.f16_widen)(meta16[..., 1])
        exact_z = (z16 == np.rint(z16)) & (np.abs(z16) <= 2048)
        bound = s16 / 2 + ((1 << bits) - 1) * np.abs(s32 - s16) + 1e-6 * (1 + np.abs(xf).max())
        err = np.abs(dec - xf).transpose(1, 0, 2).reshape(H, T, d // G, G).max(axis=3)
        assert np.all(err[exact_z] <= bound[exact_z])


# ----------------------------------------------------------------------------
# NanoKV-Fast: mixed-dimensional attention (NanoKV page, Fig. 4(d), Tables 6,
# 8, 9, 11)
# ----------------------------------------------------------------------------

def test_bf16_bits_rounds_to_nearest_even():
    """Against torch's float32 -> bf16 conversion (random values, every
    binade's ties, subnormals, overflow) and hand-worked float64 cases that
    float32 cannot hold: a value just above a tie rounds up, exact ties go to
    the even neighbour."""
    rng = np.random.default_rng(5)
    with np.errstate(over="ignore"):   # a few products overflow binary32: infinities are wanted
        a = (rng.standard_normal(20000) * np.exp2(rng.integers(-140, 128, 20000))).astype(np.float32)
    ties = (np.float32(1.0) + np.float32(2.0 ** -8) * np.arange(1, 64, 2, dtype=np.float32)).astype(np.float32)
    a = np.concatenate([a, ties, -ties, np.float32([0.0, -0.0, 3.0e38, 3.4e38, -3.4e38, 1e-40, 2.0 ** -133])])
    with np.errstate(over="ignore"):
        assert np.array_equal(O.bf16_bits(a), _bf16(a))
    assert O.bf16_bits(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81   # above the tie: up
    assert O.bf16_bits(np.array([1 + 2.0 ** -8]))[0] == 0x3F80                # tie: even (down)
    assert O.bf16_bits(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82            # tie: even (up)
    assert O.bf16_bits(np.array([-(1 + 2.0 ** -8 - 2.0 ** -45)]))[0] == 0xBF80
    assert O.bf16_bits(np.array([3 * 2.0 ** -134]))[0] == 0x0002              # subnormal tie: even


def _fast_case(seed, T=37, Tq=11, H=2, d=64):
    rng = np.random.default_rng(seed)
    q = _bf16(rng.standard_normal((Tq, H, d)) * 0.5)
    k = _bf16(rng.standard_normal((T, H, d)))
    v = _bf16(rng.standard_normal((T, H, d)))
    return q, k, v


def test_fast_attention_identity_maps_are_full_attention():
    """d_low = d with identity maps: the reduction and restoration change
    nothing, so the result is exactly ``attention`` over the same keys."""
    q, k, v = _fast_case(1)
    H, d = q.shape[1], q.shape[2]
    I = np.broadcast_to(np.eye(d), (H, d, d))
    o, lse = O.fast_attention(q, k, v, _bf16(I), _bf16(I))
    o_ref, lse_ref = O.attention(q, k, v)
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def test_fast_attention_channel_selection_is_brute_force():
    """P_h picks d_low channels (entries +-2, exact in bf16), R_h puts them
    back scaled by 1/2: the low-space logits are 2 q_c k'_c summed over the
    picked channels, the softmax scale is that of the FULL head dimension, and
    the output lands on the picked channels only -- checked against a direct
    loop over keys."""
    q, k, v = _fast_case(2, T=19, Tq=5, d=64)
    Tq, H, d = q.shape
    dl = 16
    rng = np.random.default_rng(3)
    P = np.zeros((H, d, dl))
    R = np.zeros((H, dl, d))
    picks = []
    for h in range(H):
        sel = rng.choice(d, dl, replace=False)
        sgn = rng.choice([-1.0, 1.0], dl)
        P[h, sel, np.arange(dl)] = 2.0 * sgn
        R[h, np.arange(dl), sel] = 0.5 * sgn
        picks.append((sel, sgn))
    k_low = np.zeros((k.shape[0], H, dl), np.float32)
    v_low = np.zeros((v.shape[0], H, dl), np.float32)
    kf, vf, qf = _widen(k), _widen(v), _widen(q).astype(np.float64)
    for h, (sel, sgn) in enumerate(picks):
        k_low[:, h] = kf[:, h][:, sel]
        v_low[:, h] = vf[:, h][:, sel]
    o, lse = O.fast_attention(q, _bf16(k_low), _bf16(v_low), _bf16(P), _bf16(R))
    for i in range(Tq):
        for h, (sel, sgn) in enumerate(picks):
            s = np.array([sum(2.0 * sgn[j] * qf[i, h, sel[j]] * k_low[t, h, j] for j in range(dl))
                          for t in range(k.shape[0])]) / math.sqrt(d)
            m = s.max()
            p = np.exp(s - m)
            want = np.zeros(d)
            for j in range(dl):
                want[sel[j]] = 0.5 * sgn[j] * float(np.dot(p, v_low[:, h, j])) / p.sum()
            assert np.allclose(o[i, h], want, rtol=1e-12, atol=1e-12)
            assert abs(lse[h, i] - (m + math.log(p.sum()))) < 1e-12


def test_fast_attention_in_the_span_equals_full_attention():
    """With orthonormal maps whose entries are exact in bf16 (Hadamard columns
    / 8, d = 64) and queries, keys and values inside their span, the reduced
    attention IS the full attention: q P P^T k = q k."""
    Tq, T, H, d, dl = 6, 29, 2, 64, 16
    Hd = np.array([[1.0]])
    while Hd.shape[0] < d:
        Hd = np.block([[Hd, Hd], [Hd, -Hd]])
    P = np.stack([Hd[:, 3:3 + dl] / 8.0, Hd[:, 40:40 + dl] / 8.0])      # [H][d][dl], orthonormal columns
    rng = np.random.default_rng(4)
    small = lambda *s: rng.integers(-4, 5, s).astype(np.float64) / 4.0
    q_low, k_low, v_low = small(Tq, H, dl), small(T, H, dl), small(T, H, dl)
    q = np.einsum("thl,hdl->thd", q_low, P)        # in the span; exact dyadic values
    k = np.einsum("thl,hdl->thd", k_low, P)
    v = np.einsum("thl,hdl->thd", v_low, P)
    assert np.array_equal(_widen(_bf16(q)).astype(np.float64), q)   # q itself is a bf16 tensor
    o, lse = O.fast_attention(_bf16(q), k_low.astype(np.float32), v_low.astype(np.float32), _bf16(P),
                              _bf16(np.transpose(P, (0, 2, 1))))
    o_ref, lse_ref = O.attention(q, k, v)
    assert np.allclose(o, o_ref, rtol=0, atol=1e-12) and np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_fast_maps_analytical_properties():
    """Per head: P_h has orthonormal columns ordered by descending singular
    value of the decoder slice; W_low = W_h P_h and c_low = mu_h P_h; when the
    slice has rank <= d_low the folded decoder loses nothing, W_low P_h^T =
    W_h, and the leading vector carries the largest singular value."""
    rng = np.random.default_rng(6)
    r, H, d, C, dl = 24, 2, 64, 5, 16
    base = _bf16(rng.standard_normal((10, H * d)) / 8.0)
    w_dec = base[rng.integers(0, 10, r)]             # 24 rows copied from 10: rank <= 10 < dl, exactly
    cent = _bf16(rng.standard_normal((H, C, d)))
    P, W_low, c_low = O.fast_maps_analytical(w_dec, cent, dl)
    W = _widen(w_dec).astype(np.float64)
    for h in range(H):
        Wh = W[:, h * d:(h + 1) * d]
        assert np.allclose(P[h].T @ P[h], np.eye(dl), atol=1e-12)
        assert np.allclose(W_low[:, h * dl:(h + 1) * dl], Wh @ P[h], atol=1e-12)
        assert np.allclose(c_low[h], _widen(cent[h]).astype(np.float64) @ P[h], atol=1e-12)
        assert np.allclose(W_low[:, h * dl:(h + 1) * dl] @ P[h].T, Wh, atol=1e-9)
        gains = np.linalg.norm(Wh @ P[h], axis=0)
        assert np.all(np.diff(gains[:10]) <= 1e-9) and abs(gains[0] - np.linalg.norm(Wh, 2)) < 1e-9
        assert np.all(P[h][np.argmax(np.abs(P[h]), axis=0), np.arange(dl)] > 0)


def test_fast_mac_accounting_against_tables_6_9_11():
    """Table 6's head-layer counts add up to Table 9's layers x heads; with
    every head-layer attending its whole history at its deployed dim the
    history MACs fall to sum count d_h / (sum count 128), a bound Table 11's
    saving (which routes some history at full dimension, Table 7) stays
    under; and Table 11's overall saving is the product of its two columns."""
    for m in _golden("nanokv_fast_tables.json")["models"]:
        dims = {int(k): v for k, v in m["dims"].items()}
        assert sum(dims.values()) == m["layers"] * m["heads"]
        ratio = O.fast_history_mac_ratio(dims, m["head_dim"])
        assert m["history_saved_pct"] <= 100.0 * (1.0 - ratio)
        assert abs(m["historical_share_pct"] * m["history_saved_pct"] / 100.0 - m["all_saved_pct"]) < 0.006
    hy32 = _golden("nanokv_fast_tables.json")["models"][1]
    assert O.fast_history_mac_ratio({int(k): v for k, v in hy32["dims"].items()}) == 0.5
    assert O.fast_history_mac_ratio({64: 3}) == 0.5 and O.fast_history_mac_ratio({128: 1}) == 1.0


def test_fast_reduce_queries_rounds_the_exact_sum_once():
    """q_h P_h is formed exactly and rounded to bf16 once, to nearest even:
    with q = (1, 2^-8) the columns (1, 1), (1, 3), (1, 1 + 2^-7) and (-1, -1)
    give 1 + 2^-8 (a tie: down to 1), 1 + 3 2^-8 (a tie: up), 1 + 2^-8 +
    2^-15 (above the tie: up) and -(1 + 2^-8); a second head uses its own map."""
    q = _bf16(np.array([[[1.0, 2.0 ** -8], [2.0, 0.0]]]))                       # [1][2][2]
    P = np.zeros((2, 2, 4))
    P[0] = np.array([[1.0, 1.0, 1.0, -1.0], [1.0, 3.0, 1.0 + 2.0 ** -7, -1.0]])
    P[1] = np.array([[0.5, 0.0, 3.0, 1.0], [7.0, 1.0, 1.0, 1.0]])
    got = O.fast_reduce_queries(q, _bf16(P))
    assert got.dtype == np.uint16 and got.shape == (1, 2, 4)
    assert [int(b) for b in got[0, 0]] == [0x3F80, 0x3F82, 0x3F81, 0xBF80]
    assert [float(x) for x in _widen(got[0, 1])] == [1.0, 0.0, 6.0, 2.0]


# ----------------------------------------------------------------------------
# second residual stage (QVG's progressive residual quantisation; the reading
# in the oracle's header)
# ----------------------------------------------------------------------------

def test_encode2_worked_examples():
    for case in _golden("eq1_two_stage_worked_examples.json")["cases"]:
        x = np.array(case["x"], np.float32)[None, None, :]
        cent = np.zeros((1, 1, 4), np.uint16)
        idx, codes, meta, codes2, meta2 = O.encode2(x, cent, case["bits"], 4)
        assert [float(v) for v in meta[0, 0, 0]] == [case["s1"], case["z1"]]
        assert O.unpack(codes[0, 0], 4, case["bits"]).tolist() == case["q1"]
        s2, z2 = (float(v) for v in meta2[0, 0, 0])
        assert s2 == np.float32(case["s2"]) and z2 == case["z2"] and math.copysign(1.0, z2) == \
            math.copysign(1.0, case["z2"])
        assert O.unpack(codes2[0, 0], 4, case["bits"]).tolist() == case["q2"]
        out = O.decode2(idx, codes, meta, codes2, meta2, cent, case["bits"], 4)
        assert out[0, 0].tolist() == case["x_hat"]


def test_encode2_stage_one_is_encode_and_error_bound():
    """The stage-1 arrays are exactly ``encode``'s; every value is within half
    a stage-2 step (plus the rounding of the two additions) of its
    reconstruction, and the stage-2 step is at most the stage-1 step over
    2^b - 1, so two stages never do worse than one."""
    rng = np.random.default_rng(41)
    for bits, G in ((2, 16), (4, 32), (2, 64)):
        x = (rng.standard_normal((120, 3, 64)) * np.exp(rng.uniform(-3, 3, (120, 3, 1)))).astype(np.float32)
        cent = O.fit(x, 16, 1)
        e1 = O.encode(x, cent, bits, G)
        idx, codes, meta, codes2, meta2 = O.encode2(x, cent, bits, G)
        for a, b in zip((idx, codes, meta), e1):
            assert np.array_equal(a, b)
        xh1 = O.decode(*e1, cent, bits, G).astype(np.float64)
        xh2 = O.decode2(idx, codes, meta, codes2, meta2, cent, bits, G).astype(np.float64)
        s1 = np.repeat(meta[:, :, :, 0], G, axis=2).transpose(1, 0, 2).astype(np.float64)
        s2 = np.repeat(meta2[:, :, :, 0], G, axis=2).transpose(1, 0, 2).astype(np.float64)
        z2 = np.repeat(meta2[:, :, :, 1], G, axis=2).transpose(1, 0, 2)
        err2 = np.abs(xh2 - x)
        ulp = 2.0 ** -22 * (np.abs(x) + np.abs(xh1 - x) + 1e-30)
        live = z2 == np.rint(z2)  # every group, degenerate ones included, has an integer zero
        assert np.all(err2[live] <= s2[live] / 2 + ulp[live] + 2.0 ** -23 * s1[live])
        assert np.all(s2 <= s1 / ((1 << bits) - 1) * (1 + 2.0 ** -20) + 1e-37)
        assert np.abs(xh2 - x).mean() < np.abs(xh1 - x).mean()


def test_encode2_residual_on_the_stage_one_grid_leaves_nothing():
    """Residuals that stage 1 represents exactly leave e = 0: stage 2 is the
    zero-range group (s2 = 0, z2 = 0, codes 0) and the reconstruction is the
    stage-1 one."""
    x = np.array([[[0.0, 0.5, 1.0, 1.5, 1.5, 0.0, 1.0, 0.5]]], np.float32)
    cent = np.zeros((1, 1, 8), np.uint16)
    idx, codes, meta, codes2, meta2 = O.encode2(x, cent, 2, 8)
    assert np.all(meta2 == 0.0) and np.all(codes2 == 0)
    assert np.array_equal(O.decode2(idx, codes, meta, codes2, meta2, cent, 2, 8), x)
