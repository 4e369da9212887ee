"""GPU parity of the joint head-channel code (NanoKV page, Fig. 4(b)): the
tensor-core encoder (assignment, bf16 residual, R W_enc, Eq. 1 per group of
coefficients) and decoder (c^ W_dec plus the centres) against the oracle.

Bars:
* centroid indices bit-exact everywhere;
* where every coefficient is one exact product (a signed power-of-two column
  selection as W_enc), coefficients, codes and {scale, zero} bits are
  bit-exact too;
* with a dense W_enc the coefficients are binary32 sums whose order the
  tensor cores choose, so they are held to the summation bound
  (K + 2) 2^-24 sum_i |r_i w_in| against the oracle's binary64 sums; a code
  may then differ by one step only where the two coefficients straddle a
  rounding boundary, and every GPU code still reconstructs the oracle's
  coefficient within s/2 plus that bound;
* the decoder, fed the oracle's own codes, matches the oracle within
  2^-15 sum_n |c^_n w_ni| (c^ carried as bf16 high part plus bf16
  remainder, about 16 significant bits) plus binary32 rounding of the sum.
"""

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


def _widen(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def _selection_encoder(n: int, r: int, seed: int) -> np.ndarray:
    """W_enc [n][r]: column j holds a single +-2^e (e in -2..2) at a distinct
    row, so every coefficient is one exact product."""
    rng = np.random.default_rng(seed)
    rows = rng.choice(n, size=r, replace=False)
    w = np.zeros((n, r))
    w[rows, np.arange(r)] = rng.choice([-1.0, 1.0], size=r) * np.exp2(rng.integers(-2, 3, size=r))
    return synth.bf16_bits_from_f64(w)


def _history(H, d, T, seed):
    w = synth.sweep_point(max(T, 64), 16, 4, 4, 32, 64)
    w = synth.Workload(**{**w.__dict__, "num_heads": H, "head_dim": d, "config_id": 900 + seed})
    return synth.make_history(w, "K")[:T]


def _gpu_joint_encode(codec, x_np, cent_np, w_np):
    K = _K()
    T = x_np.shape[0]
    x, cent, w = to_dev(x_np), to_dev(cent_np), to_dev(w_np)
    idx, codes, meta = K.alloc_encoded(codec, T, x.device)
    K.kvq_encode(codec, x, cent, idx, codes, meta, w_enc=w)
    idx2 = torch.empty_like(idx)
    coef = torch.empty((T, codec.joint_rank), dtype=torch.float32, device=x.device)
    K.kvq_joint_coefficients(codec, x, cent, w, idx2, coef)
    torch.cuda.synchronize()
    H, r, b, G = codec.num_heads, codec.joint_rank, codec.bits, codec.group_size
    out = (bits_u16(idx).reshape(H, T), u8(codes).reshape(T, r * b // 8),
           meta.cpu().numpy().reshape(T, r // G, 2), coef.cpu().numpy(), bits_u16(idx2).reshape(H, T))
    assert K.kvq_last_device_status() == K.KVQ_OK
    return out


def _unpack_rows(codes: np.ndarray, r: int, bits: int) -> np.ndarray:
    """Integer codes [T][r] from packed rows (low bits first)."""
    per = 8 // bits
    mask = (1 << bits) - 1
    shifts = (np.arange(per) * bits).astype(np.uint8)
    return ((codes[:, :, None] >> shifts[None, None, :]) & mask).reshape(codes.shape[0], r)


@pytest.mark.parametrize("H,d,T,r,bits,G", [
    (12, 128, 1000, 192, 4, 32),   # the joint workload's codec, ragged tail
    (3, 64, 129, 64, 2, 16),       # odd number of 64-channel blocks, one token past a tile
    (4, 128, 300, 256, 4, 64),
    (2, 64, 1, 128, 2, 32),        # a single token
])
def test_joint_encode_exact_coefficients(H, d, T, r, bits, G):
    K = _K()
    x = _history(H, d, T, seed=H + r)
    C = min(64, T)
    cent = O.fit(x[:C], C, 0)  # seeds = first C tokens: their residual rows are exactly zero
    w = _selection_encoder(H * d, r, seed=7 * r + bits)
    codec = K.Codec(H, d, C, bits, G, r)
    idx, codes, meta, coef, idx2 = _gpu_joint_encode(codec, x, cent, w)
    idx_r, codes_r, meta_r, coef_r = O.joint_encode(x, cent, w, bits, G)
    assert np.array_equal(idx, idx_r) and np.array_equal(idx2, idx_r)
    assert np.array_equal(coef, coef_r), f"coef mismatch at {np.argwhere(coef != coef_r)[:5]}"
    assert np.array_equal(codes, codes_r), f"codes mismatch at {np.argwhere(codes != codes_r)[:5]}"
    assert np.array_equal(f32_bits(meta), f32_bits(meta_r)), "meta mismatch"


def test_joint_encode_zero_tokens_is_noop():
    K = _K()
    codec = K.Codec(12, 128, 256, 4, 32, 192)
    x = torch.empty((0, 12, 128), dtype=torch.bfloat16, device="cuda")
    cent = torch.zeros((12, 256, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((1536, 192), dtype=torch.bfloat16, device="cuda")
    idx, codes, meta = K.alloc_encoded(codec, 0, "cuda")
    K.kvq_encode(codec, x, cent, idx, codes, meta, w_enc=w)
    torch.cuda.synchronize()


@pytest.fixture(scope="module")
def joint():
    w = synth.workload("joint")
    x = synth.make_history(w, "K")
    cent = O.fit(x[: w.num_centroids], w.num_centroids, 0)
    w_enc = synth.make_orthonormal_encoder(w)
    return w, x, cent, w_enc


def _residual_bound(x, cent, idx, w_enc):
    """(K + 2) 2^-24 sum_i |r_i w_in| per coefficient, r the bf16 residual."""
    T, H, d = x.shape
    xf = _widen(x)
    mu = _widen(cent)
    res = np.empty((T, H * d))
    for h in range(H):
        e = (xf[:, h, :].astype(np.float32) - mu[h][idx[h]].astype(np.float32)).astype(np.float64)
        res[:, h * d:(h + 1) * d] = _widen(synth.bf16_bits_from_f64(e))
    return (H * d + 2) * 2.0 ** -24 * (np.abs(res) @ np.abs(_widen(w_enc))) + 1e-30


def test_joint_encode_full_size_sampled(joint):
    """The joint workload at full size (32,760 tokens, 12 x 128 channels,
    W_enc 1536 x 192 orthonormal, INT4 group 32), checked on sampled tokens."""
    K = _K()
    w, x, cent, w_enc = joint
    T, H, d = x.shape
    r, bits, G = w.joint_rank, w.bits_k, w.joint_group
    codec = K.Codec(H, d, w.num_centroids, bits, G, r)
    idx, codes, meta, coef, idx2 = _gpu_joint_encode(codec, x, cent, w_enc)
    rng = np.random.default_rng(5)
    toks = np.array(sorted(set(range(128)) | set(range(T - 100, T)) | set(rng.choice(T, 2048, replace=False))))
    xs = np.ascontiguousarray(x[toks])
    idx_r, codes_r, meta_r, coef_r = O.joint_encode(xs, cent, w_enc, bits, G)
    assert np.array_equal(idx[:, toks], idx_r) and np.array_equal(idx2[:, toks], idx_r)
    bound = _residual_bound(xs, cent, idx_r, w_enc)
    err = np.abs(coef[toks].astype(np.float64) - coef_r)
    assert np.all(err <= bound), f"coefficient error {np.max(err / bound):.2f} x bound"
    # codes: one step apart at most, and only where the decision is that close
    q_g = _unpack_rows(codes[toks], r, bits).astype(np.int64)
    q_r = _unpack_rows(codes_r, r, bits).astype(np.int64)
    assert np.max(np.abs(q_g - q_r)) <= 1
    assert np.mean(q_g != q_r) < 1e-3, f"{np.mean(q_g != q_r):.2e} of codes differ"
    m = meta[toks]
    s = np.repeat(m[:, :, 0], G, axis=1).astype(np.float64)
    z = np.repeat(m[:, :, 1], G, axis=1).astype(np.float64)
    rec = (q_g - z) * s
    gbound = np.repeat(bound.reshape(len(toks), r // G, G).max(axis=2), G, axis=1)
    assert np.all(np.abs(rec - coef_r) <= s / 2 * (1 + 1e-5) + 2 * gbound + 1e-30)
    # scales agree to the coefficient error (the range moves by at most 2 bounds)
    s_r = meta_r[:, :, 0].astype(np.float64)
    assert np.all(np.abs(m[:, :, 0] - s_r) <= (2 * gbound[:, ::G] + 1e-30) / ((1 << bits) - 1) + 2e-7 * s_r)


def _decode_bound(coef_r, meta_r, w_dec, G, T, H, d):
    s = np.repeat(meta_r[:, :, 0], G, axis=1).astype(np.float64)
    S = (np.abs(coef_r) + s) @ np.abs(_widen(w_dec))
    return (2.0 ** -15 + (w_dec.shape[0] + 2) * 2.0 ** -24) * S.reshape(T, H, d)


@pytest.mark.parametrize("H,d,T,r,bits,G,dense", [
    (12, 128, 700, 192, 4, 32, True),
    (3, 64, 129, 64, 2, 16, True),
    (4, 128, 300, 256, 4, 64, False),
])
def test_joint_decode_against_oracle(H, d, T, r, bits, G, dense):
    K = _K()
    x = _history(H, d, T, seed=31 + H)
    C = 64
    cent = O.fit(x[:C], C, 0)
    if dense:
        wq = synth.Workload(**{**synth.workload("joint").__dict__, "num_heads": H, "head_dim": d, "joint_rank": r})
        w_enc = synth.make_orthonormal_encoder(wq)
    else:
        w_enc = _selection_encoder(H * d, r, seed=r)
    w_dec = np.ascontiguousarray(w_enc.T)
    idx_r, codes_r, meta_r, coef_r = O.joint_encode(x, cent, w_enc, bits, G)
    ref = O.joint_decode(idx_r, codes_r, meta_r, cent, w_dec, bits, G)
    codec = K.Codec(H, d, C, bits, G, r)
    comp = K.Compressed(codec, T, to_dev(cent), to_dev(idx_r.view(np.int16)), to_dev(codes_r), to_dev(meta_r),
                        w_dec=to_dev(w_dec))
    out32 = torch.empty((T, H, d), dtype=torch.float32, device="cuda")
    out16 = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
    K.kvq_decode(comp, out32)
    K.kvq_decode(comp, out16)
    torch.cuda.synchronize()
    assert K.kvq_last_device_status() == K.KVQ_OK
    g = out32.cpu().numpy().astype(np.float64)
    bound = _decode_bound(coef_r, meta_r, w_dec, G, T, H, d) + 2.0 ** -23 * np.abs(ref)
    err = np.abs(g - ref)
    assert np.all(err <= bound), f"decode error {np.max(err / bound):.2f} x bound"
    # the bf16 output is the round-to-nearest-even of the binary32 one
    assert np.array_equal(bits_u16(out16), synth.bf16_bits_from_f64(out32.cpu().numpy().astype(np.float64)))
