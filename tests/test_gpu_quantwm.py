"""GPU parity of QuantWM's two additions (QuantWM: Temporally Consistent 2-Bit
KV Cache Quantization for Video World Models) against the oracle.

* QSAC (Sec. 4.1): kvq_encode_qsac's idx, codes and {s, z} bit-exact against
  the oracle's qsac_encode, with channel weights from the diagonal of the
  queries' second moments and at cold start (unit weights), candidate counts
  1, 4 and 8 (more than the centres), bf16 and float32 histories, d = 64 and
  128, both code widths and every group size; M = 1 with unit weights is the
  plain nearest-centre encode, so its idx must equal the oracle's assign.
* PSAC (Sec. 4.2, rank 8): kvq_psac_coefficients within the derived binary32
  bound of the oracle's psac_coefficients (fed the same binary32 basis and the
  oracle's own reconstruction, which the GPU decode matches bit for bit), and
  kvq_attention_psac_lse, fed the oracle's coefficients, within the attention
  tolerances of the oracle's attention_psac: whole history, a ragged
  sub-range, split into workspace partials, and compact {s, z}.
"""

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth
from oracle import oracle as O
from tests.gpu_util import assert_attention_close, bits_u16, f32_bits, to_dev, u8

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def _K():
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _inputs(name, T, H, Tq=600):
    w = synth.workload(name)
    xk = np.ascontiguousarray(synth.make_history(w, "K", max_tokens=T)[:, :H])
    xv = np.ascontiguousarray(synth.make_history(w, "V", max_tokens=T)[:, :H])
    q = np.ascontiguousarray(synth.make_queries(w, max_tokens=Tq)[:, :H])
    return w, xk, xv, q


@pytest.mark.parametrize("name,T,H,bits,G,C,M,cold,f32", [
    ("wan13b", 2999, 4, 2, 16, 256, 4, False, False),
    ("wan13b", 1029, 3, 4, 32, 64, 1, True, False),     # M = 1, unit weights: the plain assign
    ("14b", 777, 2, 2, 64, 5, 8, False, False),        # more candidates than centres
    ("tiny", 1000, 2, 4, 16, 128, 4, False, True),     # d = 64, float32 history
    ("tiny", 130, 2, 2, 32, 16, 8, True, False),
])
def test_qsac_encode_bit_exact(name, T, H, bits, G, C, M, cold, f32):
    K = _K()
    w, xk, _, q = _inputs(name, T, H)
    T, d = xk.shape[0], w.head_dim  # the tiny workload holds fewer tokens than asked
    if xk.dtype == np.float32 and not f32:      # the tiny workload is float32: take its bf16 rounding
        xk = synth.bf16_bits_from_f64(xk.astype(np.float64))
    x = synth.bf16_bits_to_f32(xk) if (f32 and xk.dtype == np.uint16) else xk
    cent = O.fit(xk[:C], C, 0)
    wts = O.qsac_weights(None if cold else O.query_moments(q), H, d)
    codec = K.Codec(H, d, C, bits, G)
    idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
    K.kvq_encode_qsac(codec, to_dev(x), to_dev(cent), to_dev(wts), idx, codes, meta, M=M)
    assert K.kvq_last_device_status() == K.KVQ_OK
    idx_r, codes_r, meta_r = O.qsac_encode(x, cent, wts, bits, G, M)
    got = bits_u16(idx).reshape(H, T)
    assert np.array_equal(got, idx_r), f"idx mismatch at {np.argwhere(got != idx_r)[:5]}"
    assert np.array_equal(u8(codes).reshape(H, T, d * bits // 8), codes_r)
    assert np.array_equal(f32_bits(meta).reshape(H, T, d // G, 2), f32_bits(meta_r))
    if M == 1 and cold:
        assert np.array_equal(got, O.assign(x, cent))


def _psac_setup(K, name, T, H, bits_k, bits_v, G, C, meta_format):
    w, xk, xv, q = _inputs(name, T, H)
    d = w.head_dim
    U = O.psac_basis(O.query_moments(q), 8).astype(np.float32)
    comps, decs = [], []
    for x, bits in ((xk, bits_k), (xv, bits_v)):
        cent = O.fit(x[:C], C, 0)
        codec = K.Codec(H, d, C, bits, G, 0, meta_format)
        idx, codes, meta = K.alloc_encoded(codec, T, "cuda")
        K.kvq_encode(codec, to_dev(x), to_dev(cent), idx, codes, meta)
        comps.append(K.Compressed(codec, T, to_dev(cent), idx, codes, meta))
        if meta_format == K.KVQ_META_F16:
            decs.append(O.decode16(*O.encode16(x, cent, bits, G), cent, bits, G))
        else:
            decs.append(O.decode(*O.encode(x, cent, bits, G), cent, bits, G))
    return xk, q, U, comps, decs


@pytest.mark.parametrize("name,T,H,bits_k,bits_v,G,C,compact", [
    ("wan13b", 3001, 4, 2, 2, 16, 256, False),
    ("14b", 1700, 3, 4, 2, 32, 512, False),
    ("wan13b", 1100, 2, 2, 4, 32, 64, True),
])
def test_psac_coefficients_and_attention(name, T, H, bits_k, bits_v, G, C, compact):
    K = _K()
    fmt = K.KVQ_META_F16 if compact else K.KVQ_META_F32
    xk, q, U, (kc, vc), (khat, vhat) = _psac_setup(K, name, T, H, bits_k, bits_v, G, C, fmt)
    d = xk.shape[2]
    # (1) coefficients: e = x - x^ and eight binary32 FMA chains over d channels
    coef = torch.empty((H, T, 8), dtype=torch.float32, device="cuda")
    K.kvq_psac_coefficients(kc, to_dev(xk), to_dev(U), coef)
    assert K.kvq_last_device_status() == K.KVQ_OK
    Uw = U.astype(np.float64)
    ref = O.psac_coefficients(xk, khat, Uw)                         # [T][H][8], binary32
    e = synth.bf16_bits_to_f32(xk).astype(np.float64) - khat.astype(np.float64)
    S = np.einsum("thd,hdr->thr", np.abs(e), np.abs(Uw))
    bound = (d + 2) * U32 * S + 2 * U32 * np.abs(ref)
    err = np.abs(coef.cpu().numpy().transpose(1, 0, 2).astype(np.float64) - ref)
    assert np.all(err <= bound), f"coefficients off by {np.max(err / np.maximum(bound, 1e-300)):.2f} x bound"
    # (2) attention over k^ + U C, fed the oracle's coefficients
    coef_ref = to_dev(np.ascontiguousarray(ref.transpose(1, 0, 2)))
    Ud, qd = to_dev(U), to_dev(q)
    o = torch.empty((q.shape[0], H, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    ws = K.alloc_workspace(K.KVQ_OP_ATTENTION, kc.codec, T, "cuda", num_queries=q.shape[0])
    for t0, t1, wsp in ((0, T, None), (T // 7, T - T // 5, None), (0, T, ws)):
        K.kvq_attention_psac_lse(qd, kc, vc, Ud, coef_ref, o, lse, t_begin=t0, t_end=t1, workspace=wsp)
        o_ref, lse_ref = O.attention_psac(q, khat[t0:t1], vhat[t0:t1], Uw, ref[t0:t1])
        assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"psac {name} [{t0},{t1})")
    # the correction is visible: without it the logits are those of k^ alone
    K.kvq_attention_lse(qd, kc, vc, o, lse)
    o_ref, lse_ref = O.attention(q, khat, vhat)
    assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"plain {name}")
    _, lse_psac = O.attention_psac(q, khat, vhat, Uw, ref)
    assert np.max(np.abs(lse_psac - lse_ref)) > 10 * 1e-3 or np.allclose(ref, 0)
    assert K.kvq_last_device_status() == K.KVQ_OK
