"""ctypes binding of libkvq (include/kvq.h).

Argument marshalling only: every step of the codec and of the attention runs
in the CUDA library.  Tensors are torch CUDA tensors (device memory and the
current stream come from torch); the functions take the same names as the C
entry points.  If libkvq.so is missing or fails to load, importing this module
raises -- there is no fallback.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional, Sequence, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_UNSUPPORTED = 2
KVQ_ERR_ALIGNMENT = 3
KVQ_ERR_WORKSPACE = 4
KVQ_ERR_CUDA = 5
KVQ_ERR_DEVICE_TIMEOUT = 6

KVQ_F32 = 0
KVQ_BF16 = 1

KVQ_META_F32 = 0
KVQ_META_F16 = 1

KVQ_OP_FIT = 0
KVQ_OP_ENCODE = 1
KVQ_OP_DECODE = 2
KVQ_OP_ATTENTION = 3
KVQ_OP_LAYER_ATTENTION = 4

EXPORTED = (
    "kvq_status_string", "kvq_encoded_sizes", "kvq_workspace_size", "kvq_fit_centroids",
    "kvq_fit_centroids_static", "kvq_encode", "kvq_encode_qsac", "kvq_encode_stages",
    "kvq_joint_coefficients", "kvq_decode", "kvq_psac_coefficients", "kvq_attention_lse", "kvq_attention_psac_lse",
    "kvq_attention_dense_lse", "kvq_fast_attention_lse", "kvq_fast_attention_workspace_size", "kvq_layer_attention",
    "kvq_set_wait_limit",
    "kvq_lse_merge", "kvq_last_device_status",
)


class KvqError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what} failed: {status_string(code)} ({code})")


class CodecDesc(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("num_centroids", ctypes.c_int32),
                ("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("joint_rank", ctypes.c_int32),
                ("meta_format", ctypes.c_int32), ("residual_stages", ctypes.c_int32)]


class CompressedView(ctypes.Structure):
    _fields_ = [("desc", CodecDesc), ("num_tokens", ctypes.c_int64), ("centroids", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p),
                ("w_dec", ctypes.c_void_p), ("codes2", ctypes.c_void_p), ("meta2", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built ({LIB_PATH}); run python -m kv_cache_compression_head_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pdesc, pview = ctypes.POINTER(CodecDesc), ctypes.POINTER(CompressedView)
    lib.kvq_status_string.argtypes = [ctypes.c_int]
    lib.kvq_status_string.restype = ctypes.c_char_p
    sig = {
        "kvq_encoded_sizes": [pdesc, i64, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz)],
        "kvq_workspace_size": [ctypes.c_int, pdesc, i64, i64, ctypes.POINTER(sz)],
        "kvq_fit_centroids": [pdesc, vp, ctypes.c_int, i64, i32, vp, vp, sz, vp],
        "kvq_fit_centroids_static": [pdesc, vp, ctypes.c_int, i64, i32, vp, vp],
        "kvq_encode": [pdesc, vp, ctypes.c_int, i64, vp, vp, vp, vp, vp, vp, sz, vp],
        "kvq_encode_qsac": [pdesc, vp, ctypes.c_int, i64, vp, vp, i32, vp, vp, vp, vp],
        "kvq_encode_stages": [pdesc, vp, ctypes.c_int, i64, vp, vp, vp, vp, vp, vp, vp],
        "kvq_joint_coefficients": [pdesc, vp, ctypes.c_int, i64, vp, vp, vp, vp, vp, sz, vp],
        "kvq_decode": [pview, vp, ctypes.c_int, vp, sz, vp],
        "kvq_attention_lse": [vp, i64, pview, pview, i64, i64, ctypes.c_float, vp, ctypes.c_int, vp, vp, sz, vp],
        "kvq_psac_coefficients": [pview, vp, ctypes.c_int, vp, i32, vp, vp],
        "kvq_attention_psac_lse": [vp, i64, pview, pview, vp, vp, i32, i64, i64, ctypes.c_float, vp, ctypes.c_int, vp,
                                   vp, sz, vp],
        "kvq_fast_attention_lse": [vp, i64, vp, vp, i64, i32, i32, i32, vp, vp, i64, i64, ctypes.c_float, vp,
                                   ctypes.c_int, vp, vp, sz, vp],
        "kvq_fast_attention_workspace_size": [i32, i32, i32, i64, ctypes.POINTER(sz)],
        "kvq_set_wait_limit": [ctypes.c_uint32],
        "kvq_attention_dense_lse": [vp, i64, vp, vp, i64, i32, i32, i64, i64, ctypes.c_float, vp, ctypes.c_int, vp,
                                    vp, sz, vp],
        "kvq_layer_attention": [vp, i64, pview, pview, i64, i64, vp, vp, i64, ctypes.c_float, vp, ctypes.c_int, vp,
                                vp, sz, vp],
        "kvq_lse_merge": [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i64, i32, i32, vp, ctypes.c_int, vp, vp],
        "kvq_last_device_status": [vp],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    return lib


_lib = _load()


def status_string(code: int) -> str:
    return _lib.kvq_status_string(code).decode()


def _check(code: int, what: str):
    if code != KVQ_OK:
        raise KvqError(code, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream=None) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KVQ_BF16
    if t.dtype == torch.float32:
        return KVQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


_IDX_DTYPES = (torch.int16, getattr(torch, "uint16", torch.int16))


def _want(what: str, t: Optional[torch.Tensor], dtypes, shape=None, numel=None, min_numel=None) -> None:
    """Refuse a tensor the library would misread or overrun.

    The C ABI takes raw pointers, so a wrong dtype, shape, stride or device
    would become an out-of-bounds access on the GPU rather than an error.
    Checked here: present, dtype, shape / element count, contiguity.  The
    device is checked by _on_cuda once every tensor of a call has passed
    these."""
    if t is None:
        raise ValueError(f"{what}: tensor required")
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    if t.dtype not in dtypes:
        raise TypeError(f"{what}: expected {' or '.join(str(d) for d in dtypes)}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{what}: expected {numel} elements, got {t.numel()}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{what}: expected at least {min_numel} elements, got {t.numel()}")
    if not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous tensor")


def _on_cuda(what: str, *ts) -> None:
    """Every tensor given (None skipped; Compressed records expanded) lives on a CUDA device."""
    for t in ts:
        if isinstance(t, Compressed):
            _on_cuda(what, t.centroids, t.idx, t.codes, t.meta, t.w_dec, t.codes2, t.meta2)
        elif t is not None and not t.is_cuda:
            raise ValueError(f"{what}: expected CUDA tensors, got one on {t.device}")


_X_DTYPES = (torch.bfloat16, torch.float32)


def _want_history(what: str, codec: "Codec", x: torch.Tensor) -> int:
    """x [T][H][d] in bf16 or float32; returns T."""
    if x is None or x.dim() != 3:
        raise ValueError(f"{what}: expected a [T][H][d] tensor")
    _want(what, x, _X_DTYPES, shape=(x.shape[0], codec.num_heads, codec.head_dim))
    return x.shape[0]


def _want_encoded(what: str, codec: "Codec", num_tokens: int, idx, codes, meta) -> None:
    ib, cb, mb = encoded_sizes(codec, num_tokens)
    _want(f"{what} idx", idx, _IDX_DTYPES, numel=ib // 2)
    _want(f"{what} codes", codes, torch.uint8, numel=cb)
    if codec.meta_format == KVQ_META_F16:
        _want(f"{what} meta", meta, torch.float16, numel=mb // 2)
    else:
        _want(f"{what} meta", meta, torch.float32, numel=mb // 4)


def _want_workspace(what: str, ws: Optional[torch.Tensor]) -> None:
    if ws is not None:
        _want(f"{what} workspace", ws, torch.uint8)


def _want_compressed(what: str, comp: "Compressed") -> None:
    c = comp.codec
    _want(f"{what} centroids", comp.centroids, torch.bfloat16, shape=(c.num_heads, c.num_centroids, c.head_dim))
    _want_encoded(what, c, comp.num_tokens, comp.idx, comp.codes, comp.meta)
    if comp.w_dec is not None:
        _want(f"{what} w_dec", comp.w_dec, torch.bfloat16, shape=(c.joint_rank, c.num_heads * c.head_dim))
    if c.residual_stages == 2 or comp.codes2 is not None or comp.meta2 is not None:
        _want(f"{what} codes2", comp.codes2, torch.uint8, numel=comp.codes.numel())
        _want(f"{what} meta2", comp.meta2, torch.float32, numel=comp.meta.numel())


def _want_attention_io(what: str, q: torch.Tensor, H: int, d: int, o_out, lse_out) -> int:
    """q [Tq][H][d] bf16, o_out [Tq][H][d] bf16/float32, lse_out [H][Tq] float32; returns Tq."""
    if q is None or q.dim() != 3:
        raise ValueError(f"{what}: expected queries [Tq][H][d]")
    Tq = q.shape[0]
    _want(f"{what} q", q, torch.bfloat16, shape=(Tq, H, d))
    _want(f"{what} o_out", o_out, _X_DTYPES, shape=(Tq, H, d))
    _want(f"{what} lse_out", lse_out, torch.float32, shape=(H, Tq))
    return Tq


# ----------------------------------------------------------------------------
# descriptors
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Codec:
    """One K or V branch: heads, head dim, centroids, bits, group size, joint
    rank, and the storage of {scale, zero} (KVQ_META_F32 or KVQ_META_F16)."""

    num_heads: int
    head_dim: int
    num_centroids: int
    bits: int
    group_size: int
    joint_rank: int = 0
    meta_format: int = KVQ_META_F32
    residual_stages: int = 1

    def c(self) -> CodecDesc:
        return CodecDesc(self.num_heads, self.head_dim, self.num_centroids, self.bits, self.group_size,
                         self.joint_rank, self.meta_format, self.residual_stages)


@dataclasses.dataclass
class Compressed:
    """Device tensors of one encoded K or V history."""

    codec: Codec
    num_tokens: int
    centroids: torch.Tensor  # [H][C][d] bf16
    idx: torch.Tensor        # [H][T] int16 (uint16 bits)
    codes: torch.Tensor      # uint8
    meta: torch.Tensor       # float32, or float16 with compact {s, z}
    w_dec: Optional[torch.Tensor] = None
    codes2: Optional[torch.Tensor] = None  # second residual stage: as codes
    meta2: Optional[torch.Tensor] = None   # and as meta (float32)

    def view(self) -> CompressedView:
        return CompressedView(self.codec.c(), self.num_tokens, _ptr(self.centroids), _ptr(self.idx),
                              _ptr(self.codes), _ptr(self.meta), _ptr(self.w_dec), _ptr(self.codes2),
                              _ptr(self.meta2))


def encoded_sizes(codec: Codec, num_tokens: int) -> Tuple[int, int, int]:
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    d = codec.c()
    _check(_lib.kvq_encoded_sizes(ctypes.byref(d), num_tokens, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "kvq_encoded_sizes")
    return a.value, b.value, c.value


def workspace_size(op: int, codec: Codec, num_tokens: int, num_queries: int = 0) -> int:
    out = ctypes.c_size_t()
    d = codec.c()
    _check(_lib.kvq_workspace_size(op, ctypes.byref(d), num_tokens, num_queries, ctypes.byref(out)),
           "kvq_workspace_size")
    return out.value


def alloc_encoded(codec: Codec, num_tokens: int, device) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Allocate idx, codes and meta tensors of the sizes kvq_encoded_sizes reports."""
    ib, cb, mb = encoded_sizes(codec, num_tokens)
    idx = torch.empty(ib // 2, dtype=torch.int16, device=device)
    codes = torch.empty(cb, dtype=torch.uint8, device=device)
    if codec.meta_format == KVQ_META_F16:
        meta = torch.empty(mb // 2, dtype=torch.float16, device=device)
    else:
        meta = torch.empty(mb // 4, dtype=torch.float32, device=device)
    return idx, codes, meta


def alloc_workspace(op: int, codec: Codec, num_tokens: int, device, num_queries: int = 0) -> Optional[torch.Tensor]:
    n = workspace_size(op, codec, num_tokens, num_queries)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


# ----------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------

def kvq_fit_centroids(codec: Codec, x: torch.Tensor, iters: int, centroids_out: torch.Tensor,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    T = _want_history("kvq_fit_centroids x", codec, x)
    _want("kvq_fit_centroids centroids_out", centroids_out, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    if workspace is None:
        workspace = alloc_workspace(KVQ_OP_FIT, codec, T, x.device)
    _want_workspace("kvq_fit_centroids", workspace)
    _on_cuda("kvq_fit_centroids", x, centroids_out, workspace)
    d = codec.c()
    _check(_lib.kvq_fit_centroids(ctypes.byref(d), _ptr(x), _dtype_code(x), T, iters, _ptr(centroids_out),
                                  _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                  _stream(stream)), "kvq_fit_centroids")
    return centroids_out


def kvq_fit_centroids_static(codec: Codec, x: torch.Tensor, iters: int, centroids_out: torch.Tensor,
                             stream=None) -> torch.Tensor:
    """kvq_fit_centroids with the library's fixed device scratch (no workspace)."""
    _want_history("kvq_fit_centroids_static x", codec, x)
    _want("kvq_fit_centroids_static centroids_out", centroids_out, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    _on_cuda("kvq_fit_centroids_static", x, centroids_out)
    d = codec.c()
    _check(_lib.kvq_fit_centroids_static(ctypes.byref(d), _ptr(x), _dtype_code(x), x.shape[0], iters,
                                         _ptr(centroids_out), _stream(stream)), "kvq_fit_centroids_static")
    return centroids_out


def kvq_encode(codec: Codec, x: torch.Tensor, centroids: torch.Tensor, idx: torch.Tensor, codes: torch.Tensor,
               meta: torch.Tensor, w_enc: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None) -> None:
    T = _want_history("kvq_encode x", codec, x)
    _want("kvq_encode centroids", centroids, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    _want_encoded("kvq_encode", codec, T, idx, codes, meta)
    if w_enc is not None:
        _want("kvq_encode w_enc", w_enc, torch.bfloat16, shape=(codec.num_heads * codec.head_dim, codec.joint_rank))
    _want_workspace("kvq_encode", workspace)
    _on_cuda("kvq_encode", x, centroids, idx, codes, meta, w_enc, workspace)
    d = codec.c()
    _check(_lib.kvq_encode(ctypes.byref(d), _ptr(x), _dtype_code(x), x.shape[0], _ptr(centroids), _ptr(w_enc),
                           _ptr(idx), _ptr(codes), _ptr(meta), _ptr(workspace),
                           workspace.numel() if workspace is not None else 0, _stream(stream)), "kvq_encode")


def kvq_encode_qsac(codec: Codec, x: torch.Tensor, centroids: torch.Tensor, w: torch.Tensor, idx: torch.Tensor,
                    codes: torch.Tensor, meta: torch.Tensor, M: int = 4, stream=None) -> None:
    """Encode with QuantWM's query-sensitive centre selection; w [H][d]
    float32 channel weights (the queries' second moments' diagonal)."""
    T = _want_history("kvq_encode_qsac x", codec, x)
    _want("kvq_encode_qsac centroids", centroids, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    _want("kvq_encode_qsac w", w, torch.float32, shape=(codec.num_heads, codec.head_dim))
    _want_encoded("kvq_encode_qsac", codec, T, idx, codes, meta)
    _on_cuda("kvq_encode_qsac", x, centroids, w, idx, codes, meta)
    d = codec.c()
    _check(_lib.kvq_encode_qsac(ctypes.byref(d), _ptr(x), _dtype_code(x), T, _ptr(centroids), _ptr(w), M, _ptr(idx),
                                _ptr(codes), _ptr(meta), _stream(stream)), "kvq_encode_qsac")


def kvq_encode_stages(codec: Codec, x: torch.Tensor, centroids: torch.Tensor, idx: torch.Tensor,
                      codes: torch.Tensor, meta: torch.Tensor, codes2: torch.Tensor, meta2: torch.Tensor,
                      stream=None) -> None:
    """Encode with two residual stages (codec.residual_stages == 2): the
    stage-2 arrays have the shapes and types of codes and meta."""
    T = _want_history("kvq_encode_stages x", codec, x)
    _want("kvq_encode_stages centroids", centroids, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    _want_encoded("kvq_encode_stages", codec, T, idx, codes, meta)
    _want("kvq_encode_stages codes2", codes2, torch.uint8, numel=codes.numel())
    _want("kvq_encode_stages meta2", meta2, torch.float32, numel=meta.numel())
    _on_cuda("kvq_encode_stages", x, centroids, idx, codes, meta, codes2, meta2)
    d = codec.c()
    _check(_lib.kvq_encode_stages(ctypes.byref(d), _ptr(x), _dtype_code(x), T, _ptr(centroids), _ptr(idx),
                                  _ptr(codes), _ptr(meta), _ptr(codes2), _ptr(meta2), _stream(stream)),
           "kvq_encode_stages")


def kvq_joint_coefficients(codec: Codec, x: torch.Tensor, centroids: torch.Tensor, w_enc: torch.Tensor,
                           idx: torch.Tensor, coef_out: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> None:
    T = _want_history("kvq_joint_coefficients x", codec, x)
    _want("kvq_joint_coefficients centroids", centroids, torch.bfloat16,
          shape=(codec.num_heads, codec.num_centroids, codec.head_dim))
    _want("kvq_joint_coefficients w_enc", w_enc, torch.bfloat16,
          shape=(codec.num_heads * codec.head_dim, codec.joint_rank))
    _want("kvq_joint_coefficients idx", idx, _IDX_DTYPES, numel=codec.num_heads * T)
    _want("kvq_joint_coefficients coef_out", coef_out, torch.float32, shape=(T, codec.joint_rank))
    _want_workspace("kvq_joint_coefficients", workspace)
    _on_cuda("kvq_joint_coefficients", x, centroids, w_enc, idx, coef_out, workspace)
    d = codec.c()
    _check(_lib.kvq_joint_coefficients(ctypes.byref(d), _ptr(x), _dtype_code(x), x.shape[0], _ptr(centroids),
                                       _ptr(w_enc), _ptr(idx), _ptr(coef_out), _ptr(workspace),
                                       workspace.numel() if workspace is not None else 0, _stream(stream)),
           "kvq_joint_coefficients")


def kvq_decode(comp: Compressed, x_out: torch.Tensor, workspace: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    _want_compressed("kvq_decode", comp)
    c = comp.codec
    _want("kvq_decode x_out", x_out, _X_DTYPES, shape=(comp.num_tokens, c.num_heads, c.head_dim))
    _want_workspace("kvq_decode", workspace)
    _on_cuda("kvq_decode", comp, x_out, workspace)
    v = comp.view()
    _check(_lib.kvq_decode(ctypes.byref(v), _ptr(x_out), _dtype_code(x_out), _ptr(workspace),
                           workspace.numel() if workspace is not None else 0, _stream(stream)), "kvq_decode")
    return x_out


def kvq_attention_lse(q: torch.Tensor, k: Compressed, v: Compressed, o_out: torch.Tensor, lse_out: torch.Tensor,
                      t_begin: int = 0, t_end: Optional[int] = None, softmax_scale: float = 0.0,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    _want_compressed("kvq_attention_lse k", k)
    _want_compressed("kvq_attention_lse v", v)
    _want_attention_io("kvq_attention_lse", q, k.codec.num_heads, k.codec.head_dim, o_out, lse_out)
    _want_workspace("kvq_attention_lse", workspace)
    _on_cuda("kvq_attention_lse", q, k, v, o_out, lse_out, workspace)
    if t_end is None:
        t_end = k.num_tokens
    kv, vv = k.view(), v.view()
    _check(_lib.kvq_attention_lse(_ptr(q), q.shape[0], ctypes.byref(kv), ctypes.byref(vv), t_begin, t_end,
                                  softmax_scale, _ptr(o_out), _dtype_code(o_out), _ptr(lse_out), _ptr(workspace),
                                  workspace.numel() if workspace is not None else 0, _stream(stream)),
           "kvq_attention_lse")


PSAC_RANK = 8
KVQ_WAIT_LIMIT_DEFAULT = 4194304


def kvq_set_wait_limit(polls: int) -> None:
    """Test hook: polls before a bounded wait of the encode filter or the
    d = 128 attention kernels gives up (KVQ_WAIT_LIMIT_DEFAULT restores)."""
    _check(_lib.kvq_set_wait_limit(int(polls)), "kvq_set_wait_limit")


def kvq_psac_coefficients(k: Compressed, x: torch.Tensor, U: torch.Tensor, coef_out: torch.Tensor,
                          stream=None) -> None:
    """QuantWM's PSAC coefficients C [H][T][8] = (k - k^) U_h of a K history;
    x [T][H][d] the original keys, U [H][d][8] float32."""
    _want_compressed("kvq_psac_coefficients k", k)
    c = k.codec
    _want("kvq_psac_coefficients x", x, _X_DTYPES, shape=(k.num_tokens, c.num_heads, c.head_dim))
    _want("kvq_psac_coefficients U", U, torch.float32, shape=(c.num_heads, c.head_dim, PSAC_RANK))
    _want("kvq_psac_coefficients coef_out", coef_out, torch.float32, shape=(c.num_heads, k.num_tokens, PSAC_RANK))
    _on_cuda("kvq_psac_coefficients", k, x, U, coef_out)
    kv = k.view()
    _check(_lib.kvq_psac_coefficients(ctypes.byref(kv), _ptr(x), _dtype_code(x), _ptr(U), PSAC_RANK, _ptr(coef_out),
                                      _stream(stream)), "kvq_psac_coefficients")


def kvq_attention_psac_lse(q: torch.Tensor, k: Compressed, v: Compressed, U: torch.Tensor, coef: torch.Tensor,
                           o_out: torch.Tensor, lse_out: torch.Tensor, t_begin: int = 0, t_end: Optional[int] = None,
                           softmax_scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> None:
    """kvq_attention_lse over the PSAC-corrected keys k^ + U_h C (d = 128)."""
    _want_compressed("kvq_attention_psac_lse k", k)
    _want_compressed("kvq_attention_psac_lse v", v)
    c = k.codec
    _want_attention_io("kvq_attention_psac_lse", q, c.num_heads, c.head_dim, o_out, lse_out)
    _want("kvq_attention_psac_lse U", U, torch.float32, shape=(c.num_heads, c.head_dim, PSAC_RANK))
    _want("kvq_attention_psac_lse coef", coef, torch.float32, shape=(c.num_heads, k.num_tokens, PSAC_RANK))
    _want_workspace("kvq_attention_psac_lse", workspace)
    _on_cuda("kvq_attention_psac_lse", q, k, v, U, coef, o_out, lse_out, workspace)
    if t_end is None:
        t_end = k.num_tokens
    kv, vv = k.view(), v.view()
    _check(_lib.kvq_attention_psac_lse(_ptr(q), q.shape[0], ctypes.byref(kv), ctypes.byref(vv), _ptr(U), _ptr(coef),
                                       PSAC_RANK, t_begin, t_end, softmax_scale, _ptr(o_out), _dtype_code(o_out),
                                       _ptr(lse_out), _ptr(workspace),
                                       workspace.numel() if workspace is not None else 0, _stream(stream)),
           "kvq_attention_psac_lse")


def kvq_attention_dense_lse(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_out: torch.Tensor,
                            lse_out: torch.Tensor, t_begin: int = 0, t_end: Optional[int] = None,
                            softmax_scale: float = 0.0, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Attention over uncompressed bf16 keys/values k, v [Tk][H][d]."""
    if k is None or k.dim() != 3:
        raise ValueError("kvq_attention_dense_lse: expected keys [Tk][H][d]")
    Tk, H, d = k.shape
    _want("kvq_attention_dense_lse k", k, torch.bfloat16)
    _want("kvq_attention_dense_lse v", v, torch.bfloat16, shape=(Tk, H, d))
    _want_attention_io("kvq_attention_dense_lse", q, H, d, o_out, lse_out)
    _want_workspace("kvq_attention_dense_lse", workspace)
    _on_cuda("kvq_attention_dense_lse", q, k, v, o_out, lse_out, workspace)
    if t_end is None:
        t_end = Tk
    _check(_lib.kvq_attention_dense_lse(_ptr(q), q.shape[0], _ptr(k), _ptr(v), Tk, H, d, t_begin, t_end,
                                        softmax_scale, _ptr(o_out), _dtype_code(o_out), _ptr(lse_out),
                                        _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                        _stream(stream)),
           "kvq_attention_dense_lse")


def fast_attention_workspace(num_heads: int, head_dim: int, d_low: int, num_queries: int, device) -> torch.Tensor:
    n = ctypes.c_size_t()
    _check(_lib.kvq_fast_attention_workspace_size(num_heads, head_dim, d_low, num_queries, ctypes.byref(n)),
           "kvq_fast_attention_workspace_size")
    return torch.empty(max(1, n.value), dtype=torch.uint8, device=device)


def kvq_fast_attention_lse(q: torch.Tensor, k_low: torch.Tensor, v_low: torch.Tensor, P: torch.Tensor,
                           R: torch.Tensor, o_out: torch.Tensor, lse_out: torch.Tensor, workspace: torch.Tensor,
                           t_begin: int = 0, t_end: Optional[int] = None, softmax_scale: float = 0.0,
                           stream=None) -> None:
    """NanoKV-Fast: attention in each head's low space over k_low, v_low
    [Tk][H][d_low] (bf16), queries reduced by P [H][d][d_low], outputs
    restored by R [H][d_low][d] (both bf16)."""
    if k_low is None or k_low.dim() != 3:
        raise ValueError("kvq_fast_attention_lse: expected low-space keys [Tk][H][d_low]")
    Tk, H, dl = k_low.shape
    if q is None or q.dim() != 3:
        raise ValueError("kvq_fast_attention_lse: expected queries [Tq][H][d]")
    d = q.shape[2]
    _want("kvq_fast_attention_lse k_low", k_low, torch.bfloat16)
    _want("kvq_fast_attention_lse v_low", v_low, torch.bfloat16, shape=(Tk, H, dl))
    _want("kvq_fast_attention_lse P", P, torch.bfloat16, shape=(H, d, dl))
    _want("kvq_fast_attention_lse R", R, torch.bfloat16, shape=(H, dl, d))
    _want_attention_io("kvq_fast_attention_lse", q, H, d, o_out, lse_out)
    _want_workspace("kvq_fast_attention_lse", workspace)
    _on_cuda("kvq_fast_attention_lse", q, k_low, v_low, P, R, o_out, lse_out, workspace)
    if t_end is None:
        t_end = Tk
    _check(_lib.kvq_fast_attention_lse(_ptr(q), q.shape[0], _ptr(k_low), _ptr(v_low), Tk, H, d, dl, _ptr(P), _ptr(R),
                                       t_begin, t_end, softmax_scale, _ptr(o_out), _dtype_code(o_out), _ptr(lse_out),
                                       _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                       _stream(stream)), "kvq_fast_attention_lse")


def kvq_layer_attention(q: torch.Tensor, k_hist: Compressed, v_hist: Compressed, k_cur: Optional[torch.Tensor],
                        v_cur: Optional[torch.Tensor], o_out: torch.Tensor, lse_out: torch.Tensor,
                        workspace: Optional[torch.Tensor] = None, t_begin: int = 0, t_end: Optional[int] = None,
                        softmax_scale: float = 0.0, stream=None) -> None:
    """One softmax over the compressed history and the uncompressed keys
    k_cur, v_cur [Tc][H][d] (the current chunk and any raw protected tokens).
    The call needs a workspace; one is allocated when none is given."""
    _want_compressed("kvq_layer_attention k_hist", k_hist)
    _want_compressed("kvq_layer_attention v_hist", v_hist)
    H, dh = k_hist.codec.num_heads, k_hist.codec.head_dim
    _want_attention_io("kvq_layer_attention", q, H, dh, o_out, lse_out)
    if k_cur is not None or v_cur is not None:
        if k_cur is None or v_cur is None or k_cur.dim() != 3:
            raise ValueError("kvq_layer_attention: k_cur and v_cur are given together as [Tc][H][d]")
        _want("kvq_layer_attention k_cur", k_cur, torch.bfloat16, shape=(k_cur.shape[0], H, dh))
        _want("kvq_layer_attention v_cur", v_cur, torch.bfloat16, shape=tuple(k_cur.shape))
    if t_end is None:
        t_end = k_hist.num_tokens
    if workspace is None:
        workspace = alloc_workspace(KVQ_OP_LAYER_ATTENTION, k_hist.codec, k_hist.num_tokens, q.device,
                                    num_queries=q.shape[0])
    _want_workspace("kvq_layer_attention", workspace)
    _on_cuda("kvq_layer_attention", q, k_hist, v_hist, k_cur, v_cur, o_out, lse_out, workspace)
    n_cur = 0 if k_cur is None else k_cur.shape[0]
    kv, vv = k_hist.view(), v_hist.view()
    _check(_lib.kvq_layer_attention(_ptr(q), q.shape[0], ctypes.byref(kv), ctypes.byref(vv), t_begin, t_end,
                                    _ptr(k_cur), _ptr(v_cur), n_cur, softmax_scale, _ptr(o_out), _dtype_code(o_out),
                                    _ptr(lse_out), _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                    _stream(stream)),
           "kvq_layer_attention")


def kvq_lse_merge(o_parts: Sequence[torch.Tensor], lse_parts: Sequence[torch.Tensor], o_out: torch.Tensor,
                  lse_out: torch.Tensor, stream=None) -> None:
    n = len(o_parts)
    if n < 1 or len(lse_parts) != n:
        raise ValueError("kvq_lse_merge: need matching, non-empty lists of partial outputs and LSEs")
    if o_parts[0].dim() != 3:
        raise ValueError("kvq_lse_merge: partial outputs are [Tq][H][d]")
    Tq, H, d = o_parts[0].shape
    for i, (o, l) in enumerate(zip(o_parts, lse_parts)):
        _want(f"kvq_lse_merge o_parts[{i}]", o, torch.float32, shape=(Tq, H, d))
        _want(f"kvq_lse_merge lse_parts[{i}]", l, torch.float32, shape=(H, Tq))
    _want("kvq_lse_merge o_out", o_out, _X_DTYPES, shape=(Tq, H, d))
    _want("kvq_lse_merge lse_out", lse_out, torch.float32, shape=(H, Tq))
    _on_cuda("kvq_lse_merge", *o_parts, *lse_parts, o_out, lse_out)
    arr_o = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    arr_l = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    _check(_lib.kvq_lse_merge(n, arr_o, arr_l, Tq, H, d, _ptr(o_out), _dtype_code(o_out), _ptr(lse_out),
                              _stream(stream)), "kvq_lse_merge")


def kvq_last_device_status(stream=None) -> int:
    return _lib.kvq_last_device_status(_stream(stream))


# ----------------------------------------------------------------------------
# convenience: fit + encode one history into a Compressed record
# ----------------------------------------------------------------------------

def compress(codec: Codec, x: torch.Tensor, iters: int, centroids: Optional[torch.Tensor] = None,
             fit_workspace: Optional[torch.Tensor] = None, stream=None) -> Compressed:
    """Fit (unless centroids are given) and encode one K or V history."""
    T = x.shape[0]
    dev = x.device
    if centroids is None:
        centroids = torch.empty((codec.num_heads, codec.num_centroids, codec.head_dim), dtype=torch.bfloat16,
                                device=dev)
        kvq_fit_centroids(codec, x, iters, centroids, fit_workspace, stream)
    idx, codes, meta = alloc_encoded(codec, T, dev)
    kvq_encode(codec, x, centroids, idx, codes, meta, stream=stream)
    return Compressed(codec, T, centroids, idx, codes, meta)
