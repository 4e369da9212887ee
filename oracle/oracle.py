"""Python face of the CPU oracle.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline / reference leg may import this module.  It
shares no code with the CUDA library: the codec steps run in the plain C file
next to it (strict IEEE, no FMA) and attention / log-sum-exp merging run here
in NumPy float64.

Functions and the passages they follow:

* ``assign``, ``fit``, ``encode``, ``decode``: centroid-residual codec -- see
  the header of kvq_oracle.c (QuantWM Sec. 4.1; TempoKV Sec. 3.1 Eq. 1 and
  Sec. 3.3 Eq. 2; CORAL-KV Sec. 2; NanoKV page Tables 4-5).
* ``encode2``, ``decode2``: a second residual stage (QVG's progressive
  residual quantisation, named by TempoKV Sec. 2; the reading in the header
  of kvq_oracle.c).
* ``joint_encode``, ``joint_decode``, ``quant_rows``: joint head-channel
  encoder/decoder with INT4 coefficients (NanoKV page, abstract, Fig. 4(b)).
* ``attention``: softmax attention of the current chunk's queries over the
  reconstructed history, returning the output and the natural-log
  log-sum-exp of the logits (NanoKV page, Fig. 4(a,d)).
* ``lse_merge``: combination of partial attention results over history parts
  by their log-sum-exp (NanoKV page, Fig. 4(d)).
* ``layer_attention``: the current chunk's full attention -- one softmax over
  the reconstructed history and the uncompressed keys of the chunk itself
  (and of any raw protected tokens; NanoKV page, Table 4), written as plain
  attention over the union of both key sets (NanoKV page, Fig. 4(a,d)).
* ``stored_bytes_per_token_head`` / ``bits_per_value``: storage accounting.
* ``query_moments``, ``qsac_weights``, ``weighted_distance``, ``qsac_score``,
  ``qsac_assign``, ``qsac_encode``: QuantWM's query-sensitive centre selection
  (Sec. 4.1): per-head second moments of the historical queries, their
  diagonal as channel weights, top-M candidates by the weighted distance, the
  final centre by the expected squared logit error of its quantised residual.
* ``bf16_bits``, ``fast_maps_analytical``, ``fast_reduce_queries``,
  ``fast_attention``, ``fast_history_mac_ratio``: NanoKV-Fast's
  mixed-dimensional attention (NanoKV page, abstract, Fig. 4(a,d), Tables 6,
  8 and 11): queries reduced into a head's low-dimensional space, attention
  there over keys and values decoded straight into that space from the
  stored coefficients, outputs restored to the head dimension before the
  LSE merge.
* ``psac_basis``, ``psac_coefficients``, ``attention_psac``: QuantWM's
  principal-subspace logit correction (the PSAC section after Sec. 4.1;
  r = 8, Table 9): the remaining key error
  projected on the top-r eigenvectors of the query second moments, added back
  to the logits.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkvq_oracle.so")
_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(
            os.path.join(_HERE, "kvq_oracle.c")):
        from . import build as _b  # type: ignore
        _b.build()
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.kvqo_assign.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp, vp]
    lib.kvqo_fit.argtypes = [vp, i32, i64, i32, i32, i32, i32, vp, vp]
    lib.kvqo_encode.argtypes = [vp, i32, i64, i32, i32, vp, i32, i32, i32, vp, vp, vp]
    lib.kvqo_decode.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp]
    lib.kvqo_encode2.argtypes = [vp, i32, i64, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.kvqo_decode2.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp]
    lib.kvqo_quant_rows.argtypes = [vp, i64, i32, i32, i32, vp, vp]
    lib.kvqo_joint_encode.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp, i32, i32, i32, vp, vp, vp, vp]
    lib.kvqo_joint_decode.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, i32, vp]
    lib.kvqo_distance.argtypes = [vp, vp, i32]
    lib.kvqo_distance.restype = ctypes.c_float
    lib.kvqo_weighted_distance.argtypes = [vp, vp, vp, i32]
    lib.kvqo_weighted_distance.restype = ctypes.c_float
    lib.kvqo_qsac_score.argtypes = [vp, vp, i32, i32]
    lib.kvqo_qsac_score.restype = ctypes.c_float
    lib.kvqo_qsac_assign.argtypes = [vp, i32, i64, i32, i32, vp, i32, vp, i32, i32, vp, vp]
    lib.kvqo_encode_given.argtypes = [vp, i32, i64, i32, i32, vp, i32, i32, i32, vp, vp, vp]
    lib.kvqo_quant_group.argtypes = [vp, i32, i32, vp, vp, vp]
    lib.kvqo_dequant.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
    lib.kvqo_dequant.restype = ctypes.c_float
    lib.kvqo_pack.argtypes = [vp, i32, i32, vp]
    lib.kvqo_unpack.argtypes = [vp, i32, i32, vp]
    lib.kvqo_bf16_round.argtypes = [ctypes.c_float]
    lib.kvqo_bf16_round.restype = ctypes.c_uint16
    lib.kvqo_f16_round.argtypes = [ctypes.c_float]
    lib.kvqo_f16_round.restype = ctypes.c_uint16
    lib.kvqo_f16_widen.argtypes = [ctypes.c_uint16]
    lib.kvqo_f16_widen.restype = ctypes.c_float
    lib.kvqo_quant_group16.argtypes = [vp, i32, i32, vp, vp, vp]
    lib.kvqo_encode16.argtypes = [vp, i32, i64, i32, i32, vp, i32, i32, i32, vp, vp, vp]
    lib.kvqo_decode16.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp]
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _x_arg(x: np.ndarray) -> Tuple[np.ndarray, int]:
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), 0
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 1
    raise TypeError("history must be float32 or uint16 bf16 bits")


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


# ----------------------------------------------------------------------------
# scalar helpers (exposed for pinning)
# ----------------------------------------------------------------------------

def distance(x: np.ndarray, mu: np.ndarray) -> float:
    """The specified binary32 squared distance of two float32 vectors."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    mu = np.ascontiguousarray(mu, dtype=np.float32)
    return float(_load().kvqo_distance(_ptr(x), _ptr(mu), x.shape[0]))


def quant_group(r: np.ndarray, bits: int) -> Tuple[float, float, np.ndarray]:
    """Eq. 1 on one group of residuals: (scale, zero, codes)."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    q = np.zeros(r.shape[0], np.uint8)
    _load().kvqo_quant_group(_ptr(r), r.shape[0], bits, _ptr(s), _ptr(z), _ptr(q))
    return float(s[0]), float(z[0]), q


def dequant(q: int, s: float, z: float) -> float:
    return float(_load().kvqo_dequant(q, s, z))


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    out = np.zeros(q.shape[0] * bits // 8, np.uint8)
    _load().kvqo_pack(_ptr(q), q.shape[0], bits, _ptr(out))
    return out


def unpack(b: np.ndarray, n: int, bits: int) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.zeros(n, np.uint8)
    _load().kvqo_unpack(_ptr(b), n, bits, _ptr(out))
    return out


def bf16_round(f: float) -> int:
    return int(_load().kvqo_bf16_round(f))


def f16_round(f: float) -> int:
    """binary32 -> binary16 bits: nearest, ties to even, subnormals, saturating
    at 65504 (the compact {s, z} storage)."""
    return int(_load().kvqo_f16_round(f))


def f16_widen(h: int) -> float:
    return float(_load().kvqo_f16_widen(h))


def quant_group16(r: np.ndarray, bits: int) -> Tuple[int, int, np.ndarray]:
    """Eq. 1 on one group with 16-bit {s, z}: (s16 bits, z16 bits, codes)."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    q = np.zeros(r.shape[0], np.uint8)
    _load().kvqo_quant_group16(_ptr(r), r.shape[0], bits, _ptr(s), _ptr(z), _ptr(q))
    return int(s[0]), int(z[0]), q


# ----------------------------------------------------------------------------
# codec
# ----------------------------------------------------------------------------

def assign(x: np.ndarray, cent: np.ndarray, return_dist: bool = False):
    """idx [H][T] of the nearest centre per token-head.  x [T][H][d], cent [H][C][d] bf16 bits."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    idx = np.zeros((H, T), np.uint16)
    dist = np.zeros((H, T), np.float32)
    _check(_load().kvqo_assign(_ptr(x), xb, T, H, d, _ptr(cent), C, _ptr(idx), _ptr(dist)), "assign")
    return (idx, dist) if return_dist else idx


def fit(x: np.ndarray, num_centroids: int, iters: int, return_inertia: bool = False):
    """Per-head k-means centres [H][C][d] (bf16 bits)."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    cent = np.zeros((H, num_centroids, d), np.uint16)
    inertia = np.zeros((H, iters + 1), np.float64)
    _check(_load().kvqo_fit(_ptr(x), xb, T, H, d, num_centroids, iters, _ptr(cent), _ptr(inertia)), "fit")
    return (cent, inertia) if return_inertia else cent


def encode(x: np.ndarray, cent: np.ndarray, bits: int, group: int):
    """(idx [H][T] u16, codes [H][T][d*bits/8] u8, meta [H][T][d/G][2] f32)."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    idx = np.zeros((H, T), np.uint16)
    codes = np.zeros((H, T, d * bits // 8), np.uint8)
    meta = np.zeros((H, T, d // group, 2), np.float32)
    _check(_load().kvqo_encode(_ptr(x), xb, T, H, d, _ptr(cent), C, bits, group,
                               _ptr(idx), _ptr(codes), _ptr(meta)), "encode")
    return idx, codes, meta


def encode16(x: np.ndarray, cent: np.ndarray, bits: int, group: int):
    """encode with 16-bit {s, z}: (idx, codes, meta16 [H][T][d/G][2] binary16 bits as u16)."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    idx = np.zeros((H, T), np.uint16)
    codes = np.zeros((H, T, d * bits // 8), np.uint8)
    meta = np.zeros((H, T, d // group, 2), np.uint16)
    _check(_load().kvqo_encode16(_ptr(x), xb, T, H, d, _ptr(cent), C, bits, group,
                                 _ptr(idx), _ptr(codes), _ptr(meta)), "encode16")
    return idx, codes, meta


def decode16(idx: np.ndarray, codes: np.ndarray, meta16: np.ndarray, cent: np.ndarray,
             bits: int, group: int) -> np.ndarray:
    """Reconstruction [T][H][d] float32 from the 16-bit {s, z} form."""
    H, T = idx.shape
    C, d = cent.shape[1], cent.shape[2]
    out = np.zeros((T, H, d), np.float32)
    args = [np.ascontiguousarray(a) for a in (idx, codes, meta16, cent)]
    _check(_load().kvqo_decode16(*(_ptr(a) for a in args), T, H, d, C, bits, group, _ptr(out)), "decode16")
    return out


def encode2(x: np.ndarray, cent: np.ndarray, bits: int, group: int):
    """encode with a second residual stage: (idx, codes, meta, codes2, meta2);
    the first three exactly as ``encode``, the stage-2 arrays in the same
    layouts (the reading in kvq_oracle.c's header)."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    idx = np.zeros((H, T), np.uint16)
    codes = np.zeros((H, T, d * bits // 8), np.uint8)
    meta = np.zeros((H, T, d // group, 2), np.float32)
    codes2 = np.zeros_like(codes)
    meta2 = np.zeros_like(meta)
    _check(_load().kvqo_encode2(_ptr(x), xb, T, H, d, _ptr(cent), C, bits, group, _ptr(idx), _ptr(codes),
                                _ptr(meta), _ptr(codes2), _ptr(meta2)), "encode2")
    return idx, codes, meta, codes2, meta2


def decode2(idx, codes, meta, codes2, meta2, cent, bits: int, group: int) -> np.ndarray:
    """Reconstruction [T][H][d] float32 from both residual stages."""
    H, T = idx.shape
    C, d = cent.shape[1], cent.shape[2]
    out = np.zeros((T, H, d), np.float32)
    args = [np.ascontiguousarray(a) for a in (idx, codes, meta, codes2, meta2, cent)]
    _check(_load().kvqo_decode2(*(_ptr(a) for a in args), T, H, d, C, bits, group, _ptr(out)), "decode2")
    return out


def decode(idx: np.ndarray, codes: np.ndarray, meta: np.ndarray, cent: np.ndarray,
           bits: int, group: int) -> np.ndarray:
    """Reconstruction [T][H][d] float32."""
    H, T = idx.shape
    C, d = cent.shape[1], cent.shape[2]
    out = np.zeros((T, H, d), np.float32)
    args = [np.ascontiguousarray(a) for a in (idx, codes, meta, cent)]
    _check(_load().kvqo_decode(*(_ptr(a) for a in args), T, H, d, C, bits, group, _ptr(out)), "decode")
    return out


def quant_rows(coef: np.ndarray, bits: int, group: int):
    """Eq. 1 per contiguous group along rows of a [T][r] float32 matrix."""
    coef = np.ascontiguousarray(coef, dtype=np.float32)
    T, r = coef.shape
    codes = np.zeros((T, r * bits // 8), np.uint8)
    meta = np.zeros((T, r // group, 2), np.float32)
    _check(_load().kvqo_quant_rows(_ptr(coef), T, r, bits, group, _ptr(codes), _ptr(meta)), "quant_rows")
    return codes, meta


def joint_encode(x: np.ndarray, cent: np.ndarray, w_enc: np.ndarray, bits: int, group: int):
    """(idx [H][T], codes [T][r*bits/8], meta [T][r/G][2], coef [T][r] f32)."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    r = w_enc.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    w_enc = np.ascontiguousarray(w_enc, dtype=np.uint16)
    idx = np.zeros((H, T), np.uint16)
    codes = np.zeros((T, r * bits // 8), np.uint8)
    meta = np.zeros((T, r // group, 2), np.float32)
    coef = np.zeros((T, r), np.float32)
    _check(_load().kvqo_joint_encode(_ptr(x), xb, T, H, d, _ptr(cent), C, _ptr(w_enc), r, bits, group,
                                     _ptr(idx), _ptr(codes), _ptr(meta), _ptr(coef)), "joint_encode")
    return idx, codes, meta, coef


def joint_decode(idx, codes, meta, cent, w_dec, bits: int, group: int) -> np.ndarray:
    H, T = idx.shape
    C, d = cent.shape[1], cent.shape[2]
    r = w_dec.shape[0]
    out = np.zeros((T, H, d), np.float32)
    args = [np.ascontiguousarray(a) for a in (idx, codes, meta, cent, w_dec)]
    _check(_load().kvqo_joint_decode(*(_ptr(a) for a in args), T, H, d, C, r, bits, group, _ptr(out)),
           "joint_decode")
    return out


# ----------------------------------------------------------------------------
# attention and merging (NumPy float64)
# ----------------------------------------------------------------------------

def _widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:  # bf16 bit patterns
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: Optional[float] = None,
              rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of queries over a (reconstructed) history.

    q [Tq][H][d] (bf16 bits or float), k, v [T][H][d] float32 reconstructions
    (or bf16 bits: uncompressed keys and values).
    Logits s_ij = scale * q_i . k_j with scale = 1/sqrt(d) unless given; no
    mask (the history strictly precedes the current chunk).
    Returns O [n][H][d] float64 and lse [H][n] float64 (natural log), where n
    = Tq or len(rows) when only some query rows are evaluated.  An empty
    history gives O = 0 and lse = -inf.
    """
    qf = _widen(q)
    if rows is not None:
        qf = qf[rows]
    kf = _widen(k)
    vf = _widen(v)
    n, H, d = qf.shape
    T = kf.shape[0]
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    O = np.zeros((n, H, d), np.float64)
    lse = np.full((H, n), -np.inf, np.float64)
    if T == 0:
        return O, lse
    for h in range(H):
        s = (qf[:, h, :] @ kf[:, h, :].T) * sc          # [n][T]
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[:, h, :] = (p @ vf[:, h, :]) / l
        lse[h, :] = (m + np.log(l))[:, 0]
    return O, lse


def layer_attention(q: np.ndarray, k_hist: np.ndarray, v_hist: np.ndarray, k_cur: np.ndarray, v_cur: np.ndarray,
                    scale: Optional[float] = None, rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Full attention of the current chunk's queries: one softmax over the
    history keys k_hist [T][H][d] (float32 reconstructions) together with the
    uncompressed keys k_cur [Tc][H][d] (bf16 bits or float), values likewise.
    The plain definition: attention over the union of the two key sets (the
    order of keys does not change a softmax-weighted sum).  Returns O [n][H][d]
    and lse [H][n] as ``attention`` does.
    """
    k = np.concatenate([_widen(k_hist), _widen(k_cur)], axis=0)
    v = np.concatenate([_widen(v_hist), _widen(v_cur)], axis=0)
    return attention(q, k, v, scale, rows)


def lse_merge(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Merge partial attention results over disjoint history parts.

    lse = m + ln sum_b exp(lse_b - m), m = max_b lse_b;
    O = sum_b exp(lse_b - lse) O_b.  Parts with lse = -inf carry weight 0; if
    every part is empty the result is O = 0, lse = -inf.
    o_parts[b] [Tq][H][d], lse_parts[b] [H][Tq].
    """
    L = np.stack([np.asarray(l, np.float64) for l in lse_parts])     # [n][H][Tq]
    Os = np.stack([np.asarray(o, np.float64) for o in o_parts])      # [n][Tq][H][d]
    m = L.max(axis=0)                                                # [H][Tq]
    finite = np.isfinite(m)
    msafe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(L), np.exp(L - msafe[None]), 0.0)       # [n][H][Tq]
    tot = w.sum(axis=0)
    lse = np.where(finite, msafe + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite[None], w / np.where(finite, tot, 1.0)[None], 0.0)
    O = np.einsum("nht,nthd->thd", wn, Os)
    return O, lse


# ----------------------------------------------------------------------------
# QuantWM: query-sensitive centre selection (QSAC) and principal-subspace
# logit correction (PSAC)
# ----------------------------------------------------------------------------

def query_moments(q: np.ndarray) -> np.ndarray:
    """M_h = mean over the observed query tokens of q q^T, per head (binary64).

    q [n][H][d] (bf16 bits or float) -> [H][d][d].  These are the historical
    query statistics both QSAC and PSAC read (QuantWM, Sec. 4.1)."""
    qf = _widen(q)
    n = qf.shape[0]
    return np.einsum("nhc,nhe->hce", qf, qf) / max(n, 1)


def qsac_weights(moments: Optional[np.ndarray], H: int, d: int) -> np.ndarray:
    """Channel weights w_{h,c} = [M_h]_cc rounded to binary32; all ones before
    any query has been observed (cold start)."""
    if moments is None:
        return np.ones((H, d), np.float32)
    return np.ascontiguousarray(np.einsum("hcc->hc", moments).astype(np.float32))


def weighted_distance(x: np.ndarray, mu: np.ndarray, w: np.ndarray) -> float:
    """QSAC's query-weighted distance sum_c w_c (x_c - mu_c)^2 in binary32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    mu = np.ascontiguousarray(mu, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    return float(_load().kvqo_weighted_distance(_ptr(x), _ptr(mu), _ptr(w), x.shape[0]))


def qsac_score(r: np.ndarray, w: np.ndarray, group: int) -> float:
    """QSAC score of one residual: sum over groups of (sum of w_c) * R_g^2."""
    r = np.ascontiguousarray(r, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    return float(_load().kvqo_qsac_score(_ptr(r), _ptr(w), r.shape[0], group))


def qsac_assign(x: np.ndarray, cent: np.ndarray, w: np.ndarray, group: int, M: int = 4,
                return_candidates: bool = False):
    """idx [H][T] chosen by QSAC; optionally the ranked candidates [H][T][M]
    (-1 where there are fewer than M centres).  x [T][H][d], cent [H][C][d]
    bf16 bits, w [H][d] binary32."""
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    idx = np.zeros((H, T), np.uint16)
    cand = np.zeros((H, T, M), np.int32)
    _check(_load().kvqo_qsac_assign(_ptr(x), xb, T, H, d, _ptr(cent), C, _ptr(w), group, M, _ptr(idx),
                                    _ptr(cand)), "qsac_assign")
    return (idx, cand) if return_candidates else idx


def qsac_encode(x: np.ndarray, cent: np.ndarray, w: np.ndarray, bits: int, group: int, M: int = 4):
    """encode with the QSAC centre choice: (idx, codes, meta) in the layouts
    of ``encode``."""
    idx = qsac_assign(x, cent, w, group, M)
    x, xb = _x_arg(x)
    T, H, d = x.shape
    C = cent.shape[1]
    cent = np.ascontiguousarray(cent, dtype=np.uint16)
    codes = np.zeros((H, T, d * bits // 8), np.uint8)
    meta = np.zeros((H, T, d // group, 2), np.float32)
    _check(_load().kvqo_encode_given(_ptr(x), xb, T, H, d, _ptr(cent), C, bits, group, _ptr(idx), _ptr(codes),
                                     _ptr(meta)), "encode_given")
    return idx, codes, meta


def psac_basis(moments: np.ndarray, r: int) -> np.ndarray:
    """U_r [H][d][r]: eigenvectors of M_h for its r largest eigenvalues, in
    decreasing order (numpy.linalg.eigh), each with its largest-magnitude
    component made positive."""
    H, d, _ = moments.shape
    U = np.zeros((H, d, r), np.float64)
    for h in range(H):
        lam, vec = np.linalg.eigh(moments[h])
        order = np.argsort(-lam, kind="stable")[:r]
        V = vec[:, order]
        sign = np.sign(V[np.argmax(np.abs(V), axis=0), np.arange(r)])
        U[h] = V * np.where(sign == 0, 1.0, sign)[None, :]
    return U


def psac_coefficients(x: np.ndarray, k_hat: np.ndarray, U: np.ndarray) -> np.ndarray:
    """C [T][H][r] = (k - k^) U_r per head: the remaining key error along the
    principal query directions, stored in binary32.  x the original keys
    (bf16 bits or float), k_hat the reconstruction [T][H][d]."""
    e = _widen(x) - _widen(k_hat)
    return np.einsum("thd,hdr->thr", e, U).astype(np.float32)


def attention_psac(q: np.ndarray, k_hat: np.ndarray, v: np.ndarray, U: np.ndarray, coef: np.ndarray,
                   scale: Optional[float] = None, rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention with PSAC's corrected logits s_ij = scale (q_i . k^_j +
    (q_i U_r) . C_j); otherwise as ``attention``.  Equivalent to attention over
    the corrected keys k^_j + U_r C_j, which is how it is evaluated."""
    kc = _widen(k_hat) + np.einsum("hdr,thr->thd", U, coef.astype(np.float64))
    return attention(q, kc, v, scale, rows)


# ----------------------------------------------------------------------------
# NanoKV-Fast: mixed-dimensional attention on the joint code
# ----------------------------------------------------------------------------

def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of real values (float64, or float32 widened) to
    bf16, as bit patterns [uint16].  Values past the largest finite bf16
    round to infinity; the subnormal range keeps the fixed 2^-133 spacing."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                       # a = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                  # bf16 normals start at 2^-126
    q = np.rint(np.ldexp(a, 8 - e))          # 8 significant bits, ties to even
    r = np.ldexp(q, e - 8)
    with np.errstate(over="ignore"):
        f = r.astype(np.float32)             # exact unless past the range (-> inf)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def fast_maps_analytical(w_dec: np.ndarray, cent: np.ndarray, d_low: int):
    """Analytical low-dimensional maps of one branch (the "analytical
    initialization" row of Table 8), per head h of the joint decoder W_dec
    [r][H d] (bf16 bits or float) and the centres [H][C][d]:

      P_h     [d][d_low]  the d_low leading right singular vectors of the head's
                          decoder slice W_dec[:, h d:(h+1) d] (numpy.linalg.svd,
                          descending singular values), each with its
                          largest-magnitude component made positive;
      W_low   [r][H d_low] the folded decoder, W_dec,h P_h per head;
      c_low   [H][C][d_low] the centres in the low space, mu_h P_h.

    Keys use their branch's P_h to reduce queries; values use theirs, P_h^T,
    to restore outputs.  Returned in float64; the resident copies are bf16."""
    W = _widen(np.asarray(w_dec))
    cf = _widen(np.asarray(cent))
    H, C, d = cf.shape
    r = W.shape[0]
    P = np.zeros((H, d, d_low))
    W_low = np.zeros((r, H * d_low))
    c_low = np.zeros((H, C, d_low))
    for h in range(H):
        Wh = W[:, h * d:(h + 1) * d]
        _, _, vt = np.linalg.svd(Wh, full_matrices=True)
        V = vt[:d_low].T                                        # [d][d_low]
        sign = np.sign(V[np.argmax(np.abs(V), axis=0), np.arange(d_low)])
        V = V * np.where(sign == 0, 1.0, sign)[None, :]
        P[h] = V
        W_low[:, h * d_low:(h + 1) * d_low] = Wh @ V
        c_low[h] = cf[h] @ V
    return P, W_low, c_low


def fast_reduce_queries(q: np.ndarray, P: np.ndarray) -> np.ndarray:
    """Queries reduced into each head's low space, q_h P_h, rounded to bf16
    (the model's activation type): q [Tq][H][d], P [H][d][d_low] (bf16 bits
    or float) -> [Tq][H][d_low] bf16 bits."""
    return bf16_bits(np.einsum("thc,hcl->thl", _widen(q), _widen(P)))


def fast_attention(q: np.ndarray, k_low: np.ndarray, v_low: np.ndarray, P: np.ndarray, R: np.ndarray,
                   scale: Optional[float] = None, rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """NanoKV-Fast's low-dimensional history attention of one head set
    (NanoKV page, Fig. 4(d)): the queries are reduced, q_low = bf16(q_h P_h);
    attention runs in the low space over k_low, v_low [T][H][d_low] with the
    softmax scale of the full head dimension (the low-space logits stand in
    for q . k), and the output is restored, O_h = O_low,h R_h with R [H][d_low][d].
    Returns O [n][H][d] and lse [H][n] as ``attention`` does."""
    d = _widen(P).shape[1]
    q_low = fast_reduce_queries(q, P)
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o_low, lse = attention(q_low, k_low, v_low, sc, rows)
    return np.einsum("thl,hld->thd", o_low, _widen(R)), lse


def fast_history_mac_ratio(dim_counts: dict, d: int = 128) -> float:
    """History-attention MACs of the deployed head dims relative to full
    dimension, when every head-layer attends its whole history at its own
    dim d_h: both Q K^T and P V scale with d_h, so the ratio is
    sum_h count_h d_h / (sum_h count_h d) (NanoKV page, Table 6's counts)."""
    num = sum(int(n) * int(dh) for dh, n in dim_counts.items())
    den = sum(int(n) for n in dim_counts.values()) * d
    return num / den


# ----------------------------------------------------------------------------
# storage accounting
# ----------------------------------------------------------------------------

def stored_bytes_per_token_head(d: int, bits: int, group: int, meta_bytes_per_group: int = 8,
                                index_bytes: int = 2) -> float:
    """Bytes stored per d-vector: packed codes + per-group {scale, zero} + index."""
    return d * bits / 8 + (d // group) * meta_bytes_per_group + index_bytes


def bits_per_value(bits: int, group: int, meta_bits_per_group: int) -> float:
    """Stored bits per cached value for b-bit codes with per-group metadata."""
    return bits + meta_bits_per_group / group


def compression_ratio(bits: int, group: int, meta_bits_per_group: int, base_bits: int = 16) -> float:
    return base_bits / bits_per_value(bits, group, meta_bits_per_group)


def joint_nominal_ratio(channels: int, rank: int, coef_bits: int = 4, base_bits: int = 16) -> float:
    """Nominal coefficient compression: channels*16 / (rank*coef_bits)."""
    return channels * base_bits / (rank * coef_bits)
