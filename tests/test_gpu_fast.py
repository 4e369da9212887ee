"""GPU parity of NanoKV-Fast's mixed-dimensional history attention (NanoKV
page, Fig. 4(a,d), Tables 6 and 8) against the oracle.

The joint workload's K and V histories (12 heads x 128, rank 192, INT4 group
32) are joint-coded by the oracle; the analytical low-dimensional maps of
each branch (oracle's fast_maps_analytical, resident in bf16) give the folded
decoders and low-space centres.  Checked:

* the history decoded straight into the low space by kvq_decode (a joint view
  with head_dim = d_low) against the oracle's joint decoder on the same
  folded maps, within the decoder's derived bound, and its bf16 output the
  round-to-nearest-even of its binary32 output;
* kvq_fast_attention_lse fed the ORACLE's low-space keys and values against
  the oracle's fast_attention within the attention tolerances: whole history,
  a ragged sub-range, split into partials, d_low = 64 and 128, bf16 output;
* the whole path (GPU decode into the low space, then the GPU attention)
  against the oracle's, in tolerance;
* d = 64 heads with random maps, and an empty key range.
"""

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_attention_close, bits_u16, to_dev

pytestmark = pytest.mark.gpu


def _K():
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _widen(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


@pytest.fixture(scope="module")
def joint_case():
    w = synth.workload("joint")
    H, d, r, G, C = w.num_heads, w.head_dim, w.joint_rank, w.joint_group, w.num_centroids
    T, Tq = 2001, 700
    w_enc = synth.make_orthonormal_encoder(w)
    w_dec = np.ascontiguousarray(w_enc.T)
    q = synth.make_queries(w, max_tokens=Tq)
    branches = []
    for which, bits in (("K", w.bits_k), ("V", w.bits_v)):
        x = synth.make_history(w, which, max_tokens=T)
        cent = O.fit(x[:C], C, 0)
        idx, codes, meta, coef = O.joint_encode(x, cent, w_enc, bits, G)
        branches.append(dict(x=x, cent=cent, idx=idx, codes=codes, meta=meta, coef=coef, bits=bits))
    return dict(w=w, H=H, d=d, r=r, G=G, C=C, T=T, q=q, w_dec=w_dec, branches=branches)


def _low_maps(case, dl):
    """Per branch: bf16 (P, W_low, c_low) and the oracle's low-space history
    (binary32 and bf16)."""
    out = []
    for b in case["branches"]:
        P, W_low, c_low = O.fast_maps_analytical(case["w_dec"], b["cent"], dl)
        Pb, Wb, cb = O.bf16_bits(P), O.bf16_bits(W_low), O.bf16_bits(c_low)
        low32 = O.joint_decode(b["idx"], b["codes"], b["meta"], cb, Wb, b["bits"], case["G"])
        out.append(dict(P=Pb, W=Wb, c=cb, low32=low32, low=O.bf16_bits(low32)))
    return out


@pytest.mark.parametrize("dl", [64, 128])
def test_low_space_decode_within_bound(joint_case, dl):
    K = _K()
    c = joint_case
    H, r, G, T = c["H"], c["r"], c["G"], c["T"]
    for b, m in zip(c["branches"], _low_maps(c, dl)):
        codec = K.Codec(H, dl, c["C"], b["bits"], G, r)
        comp = K.Compressed(codec, T, to_dev(m["c"]), to_dev(b["idx"].view(np.int16)), to_dev(b["codes"]),
                            to_dev(b["meta"]), w_dec=to_dev(m["W"]))
        out = torch.empty((T, H, dl), dtype=torch.float32, device="cuda")
        K.kvq_decode(comp, out)
        outb = torch.empty((T, H, dl), dtype=torch.bfloat16, device="cuda")
        K.kvq_decode(comp, outb)
        torch.cuda.synchronize()
        assert K.kvq_last_device_status() == K.KVQ_OK
        got = out.cpu().numpy().astype(np.float64)
        s = np.repeat(b["meta"][:, :, 0], G, axis=1).astype(np.float64)
        S = (np.abs(b["coef"]) + s) @ np.abs(_widen(m["W"]))
        bound = ((2.0 ** -15 + (r + 2) * 2.0 ** -24) * S).reshape(T, H, dl) + 2.0 ** -23 * np.abs(m["low32"])
        err = np.abs(got - m["low32"])
        assert np.all(err <= bound), f"low-space decode off by {np.max(err / bound):.2f} x bound"
        assert np.array_equal(bits_u16(outb), bits_u16(out.to(torch.bfloat16)))


@pytest.mark.parametrize("dl", [64, 128])
def test_fast_attention_against_oracle(joint_case, dl):
    K = _K()
    c = joint_case
    H, d, T, q = c["H"], c["d"], c["T"], c["q"]
    Tq = q.shape[0]
    mk, mv = _low_maps(c, dl)
    R = np.ascontiguousarray(np.transpose(mv["P"], (0, 2, 1)))
    qd, kd, vd = to_dev(q), to_dev(mk["low"]), to_dev(mv["low"])
    Pd, Rd = to_dev(mk["P"]), to_dev(R)
    o = torch.empty((Tq, H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    small = torch.empty(6 * Tq * H * dl + 1024, dtype=torch.uint8, device="cuda")   # no room to split
    full = K.fast_attention_workspace(H, d, dl, Tq, "cuda")
    for t0, t1, ws in ((0, T, small), (T // 6, T - T // 4, small), (0, T, full)):
        K.kvq_fast_attention_lse(qd, kd, vd, Pd, Rd, o, lse, ws, t_begin=t0, t_end=t1)
        o_ref, lse_ref = O.fast_attention(q, mk["low"][t0:t1], mv["low"][t0:t1], mk["P"], R)
        assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"fast d_low={dl} [{t0},{t1})")
    # bf16 output: the binary32 result rounded to nearest even, within the
    # attention tolerance plus half a bf16 ulp of the value
    K.kvq_fast_attention_lse(qd, kd, vd, Pd, Rd, o, lse, full)
    ob = torch.empty((Tq, H, d), dtype=torch.bfloat16, device="cuda")
    K.kvq_fast_attention_lse(qd, kd, vd, Pd, Rd, ob, lse, full)
    assert np.array_equal(bits_u16(ob), bits_u16(o.to(torch.bfloat16)))
    o_ref, lse_ref = O.fast_attention(q, mk["low"], mv["low"], mk["P"], R)
    err = np.abs(ob.float().cpu().numpy().astype(np.float64) - o_ref)
    assert np.all(err <= 3e-2 + 2.0 ** -8 * np.abs(o_ref)), f"bf16 output off by {err.max():.3e}"
    assert K.kvq_last_device_status() == K.KVQ_OK


def test_fast_path_end_to_end(joint_case):
    """GPU decode into the 64-dim space, then the GPU low-space attention,
    against the oracle's decode and fast_attention."""
    K = _K()
    c = joint_case
    H, d, r, G, T, q = c["H"], c["d"], c["r"], c["G"], c["T"], c["q"]
    dl, Tq = 64, q.shape[0]
    maps = _low_maps(c, dl)
    lows = []
    for b, m in zip(c["branches"], maps):
        comp = K.Compressed(K.Codec(H, dl, c["C"], b["bits"], G, r), T, to_dev(m["c"]),
                            to_dev(b["idx"].view(np.int16)), to_dev(b["codes"]), to_dev(b["meta"]),
                            w_dec=to_dev(m["W"]))
        out = torch.empty((T, H, dl), dtype=torch.bfloat16, device="cuda")
        K.kvq_decode(comp, out)
        lows.append(out)
    R = np.ascontiguousarray(np.transpose(maps[1]["P"], (0, 2, 1)))
    o = torch.empty((Tq, H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    K.kvq_fast_attention_lse(to_dev(q), lows[0], lows[1], to_dev(maps[0]["P"]), to_dev(R), o, lse,
                             K.fast_attention_workspace(H, d, dl, Tq, "cuda"))
    o_ref, lse_ref = O.fast_attention(q, maps[0]["low"], maps[1]["low"], maps[0]["P"], R)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fast end to end")
    assert K.kvq_last_device_status() == K.KVQ_OK


def test_fast_attention_d64_random_maps_and_empty_range():
    K = _K()
    rng = np.random.default_rng(21)
    Tq, T, H, d = 333, 1111, 3, 64
    bf = lambda a: O.bf16_bits(a)
    q = bf(rng.standard_normal((Tq, H, d)))
    k = bf(rng.standard_normal((T, H, d)) * 0.7)
    v = bf(rng.standard_normal((T, H, d)))
    P = bf(rng.standard_normal((H, d, d)) / 8.0)
    R = bf(rng.standard_normal((H, d, d)) / 8.0)
    o = torch.empty((Tq, H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, Tq), dtype=torch.float32, device="cuda")
    ws = K.fast_attention_workspace(H, d, d, Tq, "cuda")
    K.kvq_fast_attention_lse(to_dev(q), to_dev(k), to_dev(v), to_dev(P), to_dev(R), o, lse, ws)
    o_ref, lse_ref = O.fast_attention(q, k, v, P, R)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, "fast d=64")
    K.kvq_fast_attention_lse(to_dev(q), to_dev(k), to_dev(v), to_dev(P), to_dev(R), o, lse, ws, t_begin=5, t_end=5)
    assert np.all(np.isneginf(lse.cpu().numpy())) and not o.cpu().numpy().any()
    assert K.kvq_last_device_status() == K.KVQ_OK
