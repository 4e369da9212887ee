"""Host-side checks of the C ABI: the library loads, exports every entry point
include/kvq.h declares, reports sizes, and rejects bad arguments before any
device work (these calls never reach the GPU, so they run without one)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    from kv_cache_compression_head_b200 import build

    build.build()
    from kv_cache_compression_head_b200 import kvq

    return kvq


def _declared():
    with open(os.path.join(ROOT, "include", "kvq.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]*?\b(kvq_\w+)\s*\(", src)))


def test_header_symbols_exported(K):
    names = _declared()
    assert len(names) >= 10
    lib = ctypes.CDLL(K.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(K.EXPORTED)


def test_status_strings(K):
    for code in range(7):
        assert K.status_string(code).startswith("KVQ_")
    assert K.status_string(99) == "KVQ_ERR_UNKNOWN"


def test_encoded_sizes_and_workspace(K):
    c = K.Codec(12, 128, 256, 2, 16)
    ib, cb, mb = K.encoded_sizes(c, 32760)
    assert ib == 12 * 32760 * 2
    assert cb == 12 * 32760 * 32
    assert mb == 12 * 32760 * 8 * 8
    # 98 bytes per token-head: 2 index + 32 codes + 64 metadata
    assert (ib + cb + mb) == 12 * 32760 * 98
    c4 = K.Codec(40, 128, 512, 4, 32)
    assert K.encoded_sizes(c4, 10)[1] == 40 * 10 * 64
    assert K.workspace_size(K.KVQ_OP_FIT, c, 32760) >= 12 * 32760 * (2 + 4)
    assert K.workspace_size(K.KVQ_OP_ATTENTION, c, 32760, 4680) >= 4 * 4680 * 12 * 128 * 4
    assert K.workspace_size(K.KVQ_OP_ENCODE, c, 32760) == 0


def _err(K, fn, *args):
    return getattr(K._lib, fn)(*args)


def test_bad_descriptors_rejected(K):
    sz = ctypes.c_size_t()
    for bad, want in [((12, 96, 256, 2, 16, 0), K.KVQ_ERR_UNSUPPORTED), ((12, 128, 256, 3, 16, 0), K.KVQ_ERR_UNSUPPORTED),
                      ((12, 128, 256, 2, 24, 0), K.KVQ_ERR_INVALID_ARG), ((12, 128, 0, 2, 16, 0), K.KVQ_ERR_INVALID_ARG),
                      ((0, 128, 256, 2, 16, 0), K.KVQ_ERR_INVALID_ARG), ((12, 128, 70000, 2, 16, 0), K.KVQ_ERR_INVALID_ARG),
                      ((12, 128, 256, 2, 8, 0), K.KVQ_ERR_UNSUPPORTED), ((12, 128, 256, 4, 20, 192), K.KVQ_ERR_INVALID_ARG)]:
        d = K.CodecDesc(*bad)
        assert _err(K, "kvq_encoded_sizes", ctypes.byref(d), 10, ctypes.byref(sz), None, None) == want, bad
    d = K.CodecDesc(12, 128, 256, 2, 16, 0)
    assert _err(K, "kvq_encoded_sizes", ctypes.byref(d), -1, None, None, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_encoded_sizes", None, 10, None, None, None) == K.KVQ_ERR_INVALID_ARG


def test_bad_pointers_and_sizes_rejected_on_host(K):
    d = K.CodecDesc(12, 128, 256, 2, 16, 0)
    A = 1 << 20  # a fake, 16-byte-aligned address: never dereferenced
    # encode: null input, misaligned codes
    assert _err(K, "kvq_encode", ctypes.byref(d), None, K.KVQ_BF16, 100, A, None, A, A, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_encode", ctypes.byref(d), A, K.KVQ_BF16, 100, A, None, A, A + 8, A, None, 0, None) \
        == K.KVQ_ERR_ALIGNMENT
    assert _err(K, "kvq_encode", ctypes.byref(d), A, 7, 100, A, None, A, A, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    # fit: T < C, too little workspace
    assert _err(K, "kvq_fit_centroids", ctypes.byref(d), A, K.KVQ_BF16, 100, 2, A, A, 1 << 30, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_fit_centroids", ctypes.byref(d), A, K.KVQ_BF16, 1000, 2, A, A, 16, None) \
        == K.KVQ_ERR_WORKSPACE
    assert _err(K, "kvq_fit_centroids", ctypes.byref(d), A, K.KVQ_BF16, 1000, -1, A, A, 1 << 30, None) \
        == K.KVQ_ERR_INVALID_ARG
    # attention: range outside the history, mismatched views
    v = K.CompressedView(d, 1000, A, A, A, A, None)
    v2 = K.CompressedView(K.CodecDesc(8, 128, 256, 2, 16, 0), 1000, A, A, A, A, None)
    assert _err(K, "kvq_attention_lse", A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1001, ctypes.c_float(0),
                A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_attention_lse", A, 10, ctypes.byref(v), ctypes.byref(v), 5, 4, ctypes.c_float(0),
                A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_attention_lse", A, 10, ctypes.byref(v), ctypes.byref(v2), 0, 10, ctypes.c_float(0),
                A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_attention_lse", A + 4, 10, ctypes.byref(v), ctypes.byref(v), 0, 10, ctypes.c_float(0),
                A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_ALIGNMENT
    # zero query rows is a no-op even with null outputs
    assert _err(K, "kvq_attention_lse", None, 0, ctypes.byref(v), ctypes.byref(v), 0, 10, ctypes.c_float(0),
                None, K.KVQ_F32, None, None, 0, None) == K.KVQ_OK
    # merge: part counts out of range, null part
    arr = (ctypes.c_void_p * 65)(*([A] * 65))
    assert _err(K, "kvq_lse_merge", 0, arr, arr, 10, 2, 128, A, K.KVQ_F32, A, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_lse_merge", 65, arr, arr, 10, 2, 128, A, K.KVQ_F32, A, None) == K.KVQ_ERR_INVALID_ARG
    arr_null = (ctypes.c_void_p * 2)(A, None)
    assert _err(K, "kvq_lse_merge", 2, arr_null, arr, 10, 2, 128, A, K.KVQ_F32, A, None) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_lse_merge", 2, arr, arr, 10, 2, 96, A, K.KVQ_F32, A, None) == K.KVQ_ERR_UNSUPPORTED
    # joint codec: decoder matrix missing or misaligned, unsupported rank,
    # encoder matrix without a rank (and the reverse), f32 input
    dj = K.CodecDesc(12, 128, 256, 4, 32, 192)
    vj = K.CompressedView(dj, 10, A, A, A, A, None)
    assert _err(K, "kvq_decode", ctypes.byref(vj), A, K.KVQ_F32, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    vj = K.CompressedView(dj, 10, A, A, A, A, A + 8)
    assert _err(K, "kvq_decode", ctypes.byref(vj), A, K.KVQ_F32, None, 0, None) == K.KVQ_ERR_ALIGNMENT
    d96 = K.CodecDesc(12, 128, 256, 4, 32, 96)
    assert _err(K, "kvq_encoded_sizes", ctypes.byref(d96), 10, ctypes.byref(ctypes.c_size_t()), None, None) \
        == K.KVQ_ERR_UNSUPPORTED
    assert _err(K, "kvq_encode", ctypes.byref(d), A, K.KVQ_BF16, 100, A, A, A, A, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_encode", ctypes.byref(dj), A, K.KVQ_BF16, 100, A, None, A, A, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_encode", ctypes.byref(dj), A, K.KVQ_F32, 100, A, A, A, A, A, None, 0, None) \
        == K.KVQ_ERR_UNSUPPORTED
    assert _err(K, "kvq_joint_coefficients", ctypes.byref(dj), A, K.KVQ_BF16, 100, A, A, A, None, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_joint_coefficients", ctypes.byref(dj), A, K.KVQ_BF16, 100, A, A, A, A + 4, None, 0, None) \
        == K.KVQ_ERR_ALIGNMENT
    assert K.workspace_size(K.KVQ_OP_ENCODE, K.Codec(12, 128, 256, 4, 32, 192), 32760) == 0


def test_dense_and_layer_attention_rejected_on_host(K):
    A = 1 << 20
    f0 = ctypes.c_float(0)
    dense = lambda *a: _err(K, "kvq_attention_dense_lse", *a)
    # range outside the keys, unsupported head dim, too many heads, bad dtype
    assert dense(A, 10, A, A, 100, 12, 128, 0, 101, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert dense(A, 10, A, A, 100, 12, 96, 0, 100, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_UNSUPPORTED
    assert dense(A, 10, A, A, 100, 70000, 128, 0, 100, f0, A, K.KVQ_F32, A, None, 0, None) \
        == K.KVQ_ERR_UNSUPPORTED
    assert dense(A, 10, A, A, 100, 0, 128, 0, 100, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert dense(A, 10, A, A, 100, 12, 128, 0, 100, f0, A, 7, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    # null keys with a non-empty range; misaligned values
    assert dense(A, 10, None, A, 100, 12, 128, 0, 100, f0, A, K.KVQ_F32, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    assert dense(A, 10, A, A + 2, 100, 12, 128, 0, 100, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_ALIGNMENT
    assert dense(None, 0, None, None, 0, 12, 128, 0, 0, f0, None, K.KVQ_F32, None, None, 0, None) == K.KVQ_OK

    d = K.CodecDesc(12, 128, 256, 2, 16, 0)
    v = K.CompressedView(d, 1000, A, A, A, A, None)
    dj = K.CompressedView(K.CodecDesc(12, 128, 256, 4, 32, 192), 1000, A, A, A, A, A)
    layer = lambda *a: _err(K, "kvq_layer_attention", *a)
    need = K.workspace_size(K.KVQ_OP_LAYER_ATTENTION, K.Codec(12, 128, 256, 2, 16), 1000, 10)
    # eight binary32 partials of O [10][12][128] and of lse [12][10]
    assert need == 8 * 10 * 12 * 128 * 4 + 8 * 12 * 10 * 4
    ok_args = (A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1000, A, A, 50, f0, A, K.KVQ_F32, A)
    # workspace missing or short
    assert layer(*ok_args, None, 0, None) == K.KVQ_ERR_WORKSPACE
    assert layer(*ok_args, A, need - 1, None) == K.KVQ_ERR_WORKSPACE
    assert layer(*ok_args[:-1], A + 4, A, need, None) == K.KVQ_ERR_ALIGNMENT
    # joint history, history range outside it, chunk keys missing, negative chunk length
    assert layer(A, 10, ctypes.byref(dj), ctypes.byref(dj), 0, 1000, A, A, 50, f0, A, K.KVQ_F32, A, A, need,
                 None) == K.KVQ_ERR_UNSUPPORTED
    assert layer(A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1001, A, A, 50, f0, A, K.KVQ_F32, A, A, need,
                 None) == K.KVQ_ERR_INVALID_ARG
    assert layer(A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1000, None, A, 50, f0, A, K.KVQ_F32, A, A, need,
                 None) == K.KVQ_ERR_INVALID_ARG
    assert layer(A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1000, A, A, -1, f0, A, K.KVQ_F32, A, A, need,
                 None) == K.KVQ_ERR_INVALID_ARG
    assert layer(A, 10, ctypes.byref(v), ctypes.byref(v), 0, 1000, A, A + 8, 50, f0, A, K.KVQ_F32, A, A, need,
                 None) == K.KVQ_ERR_ALIGNMENT
    assert layer(None, 0, ctypes.byref(v), ctypes.byref(v), 0, 1000, None, None, 0, f0, None, K.KVQ_F32, None,
                 None, 0, None) == K.KVQ_OK


def test_binding_refuses_non_bf16_queries_keys_values(K):
    """Queries and dense keys/values cross the ABI as raw bf16 bits; the
    binding refuses other dtypes before calling the library."""
    import torch

    f = torch.zeros((4, 2, 64), dtype=torch.float32)
    b = torch.zeros((4, 2, 64), dtype=torch.bfloat16)
    o = torch.zeros((4, 2, 64))
    lse = torch.zeros((2, 4))
    with pytest.raises(TypeError):
        K.kvq_attention_dense_lse(f, b, b, o, lse)
    with pytest.raises(TypeError):
        K.kvq_attention_dense_lse(b, b, f, o, lse)
    comp = _cpu_compressed(K, K.Codec(2, 64, 4, 2, 16), 4)
    with pytest.raises(TypeError):
        K.kvq_attention_lse(f, comp, comp, o, lse)
    with pytest.raises(TypeError):
        K.kvq_layer_attention(b, comp, comp, f, b, o, lse, workspace=torch.zeros(16, dtype=torch.uint8))


def _cpu_compressed(K, codec, T):
    """A compressed record of the right dtypes and sizes, on the CPU."""
    import torch

    ib, cb, mb = K.encoded_sizes(codec, T)
    cent = torch.zeros((codec.num_heads, codec.num_centroids, codec.head_dim), dtype=torch.bfloat16)
    return K.Compressed(codec, T, cent, torch.zeros(ib // 2, dtype=torch.int16), torch.zeros(cb, dtype=torch.uint8),
                        torch.zeros(mb // 4, dtype=torch.float32))


def test_binding_checks_every_tensor_before_the_library(K):
    """Every wrapper checks dtype, shape, contiguity and device of each tensor
    before a pointer reaches the library: a float32 LSE buffer, a view of the
    wrong head count or a CPU tensor would otherwise be read or written out of
    bounds on the GPU.  With correct dtypes and shapes, CPU tensors are refused
    for not being on a CUDA device."""
    import torch

    H, d, C, T, Tq = 2, 64, 4, 8, 4
    codec = K.Codec(H, d, C, 2, 16)
    comp = _cpu_compressed(K, codec, T)
    bf = torch.bfloat16
    q = torch.zeros((Tq, H, d), dtype=bf)
    o = torch.zeros((Tq, H, d))
    lse = torch.zeros((H, Tq))
    x = torch.zeros((T, H, d), dtype=bf)
    cent = torch.zeros((H, C, d), dtype=bf)
    idx, codes, meta = comp.idx, comp.codes, comp.meta

    def raises(exc, fn, *a, match=None, **kw):
        with pytest.raises(exc, match=match):
            fn(*a, **kw)

    # attention: wrong LSE dtype, wrong head count in the output, CPU tensors
    raises(TypeError, K.kvq_attention_lse, q, comp, comp, o, lse.to(bf))
    raises(ValueError, K.kvq_attention_lse, q, comp, comp, torch.zeros((Tq, H + 1, d)), lse, match="shape")
    raises(ValueError, K.kvq_attention_lse, q.transpose(0, 1).contiguous().transpose(0, 1), comp, comp, o, lse,
           match="contiguous")
    raises(ValueError, K.kvq_attention_lse, q, comp, comp, o, lse, match="CUDA")
    raises(ValueError, K.kvq_attention_lse, q, _cpu_compressed(K, K.Codec(H, d, C, 4, 16), T - 1), comp, o,
           torch.zeros((H, Tq)), match="CUDA")
    bad = K.Compressed(codec, T, cent, idx, codes[:-1], meta)
    raises(ValueError, K.kvq_attention_lse, q, bad, comp, o, lse, match="elements")
    raises(ValueError, K.kvq_attention_dense_lse, q, x, x[:, :, :32], o, lse, match="shape")
    raises(ValueError, K.kvq_attention_dense_lse, q, x, x, o, lse, match="CUDA")
    raises(ValueError, K.kvq_layer_attention, q, comp, comp, x, x[:1], o, lse, match="shape")
    raises(ValueError, K.kvq_layer_attention, q, comp, comp, x, None, o, lse, match="together")
    # codec calls
    raises(ValueError, K.kvq_fit_centroids, codec, x[:, :1], 2, cent, match="shape")
    raises(TypeError, K.kvq_fit_centroids, codec, x, 2, cent.float())
    raises(ValueError, K.kvq_fit_centroids_static, codec, x, 2, cent, match="CUDA")
    raises(TypeError, K.kvq_encode, codec, x.to(torch.float16), cent, idx, codes, meta)
    raises(TypeError, K.kvq_encode, codec, x, cent, idx.int(), codes, meta)
    raises(ValueError, K.kvq_encode, codec, x, cent, idx, codes, meta[:-2], match="elements")
    raises(ValueError, K.kvq_encode, codec, x, cent, idx, codes, meta, match="CUDA")
    jc = K.Codec(H, d, C, 4, 32, 64)
    raises(ValueError, K.kvq_joint_coefficients, jc, x, cent, torch.zeros((H * d, 32), dtype=bf), idx,
           torch.zeros((T, 64)), match="shape")
    raises(ValueError, K.kvq_decode, comp, torch.zeros((T - 1, H, d)), match="shape")
    raises(ValueError, K.kvq_decode, comp, torch.zeros((T, H, d)), match="CUDA")
    # merge: binary32 parts only, matching shapes
    raises(TypeError, K.kvq_lse_merge, [o.to(bf), o], [lse, lse], o, lse)
    raises(ValueError, K.kvq_lse_merge, [o, o], [lse, lse[:, :2]], o, lse, match="shape")
    raises(ValueError, K.kvq_lse_merge, [o, o], [lse], o, lse, match="matching")
    raises(ValueError, K.kvq_lse_merge, [o, o], [lse, lse], o, lse, match="CUDA")


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """A copy of the package without libkvq.so: importing the binding raises
    (the product path has no fallback)."""
    import shutil
    import subprocess
    import sys

    pkg = tmp_path / "kv_cache_compression_head_b200"
    pkg.mkdir()
    for name in ("__init__.py", "kvq.py"):
        shutil.copy(os.path.join(ROOT, "kv_cache_compression_head_b200", name), pkg / name)
    r = subprocess.run([sys.executable, "-c", "import kv_cache_compression_head_b200.kvq"], cwd=tmp_path,
                       capture_output=True, text=True, env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libkvq.so not built" in r.stderr


def test_compact_meta_sizes_and_refusals(K):
    """Compact 16-bit {s, z}: 4 metadata bytes per group (TempoKV, Table 1:
    b + 1 bits per value at G = 32, i.e. 5.33x for INT2 and 3.20x for INT4
    against bf16); an unknown format is an invalid argument; the joint codec
    and the d = 64 attention refuse the compact format before any launch."""
    import ctypes

    for bits, ratio in ((2, 16 / 3), (4, 16 / 5)):
        d16 = K.CodecDesc(12, 128, 256, bits, 32, 0, K.KVQ_META_F16)
        ib, cb, mb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        assert K._lib.kvq_encoded_sizes(ctypes.byref(d16), 1000, ctypes.byref(ib), ctypes.byref(cb),
                                        ctypes.byref(mb)) == K.KVQ_OK
        assert mb.value == 12 * 1000 * (128 // 32) * 4
        values = 12 * 1000 * 128
        assert abs(16 * values / ((cb.value + mb.value) * 8) - ratio) < 1e-12
    bad = K.CodecDesc(12, 128, 256, 2, 32, 0, 2)
    sz = ctypes.c_size_t()
    assert K._lib.kvq_encoded_sizes(ctypes.byref(bad), 10, None, None, None) == K.KVQ_ERR_INVALID_ARG
    joint16 = K.CodecDesc(12, 128, 256, 4, 32, 192, K.KVQ_META_F16)
    assert K._lib.kvq_encoded_sizes(ctypes.byref(joint16), 10, None, None, None) == K.KVQ_ERR_UNSUPPORTED
    A = 1 << 20  # a 16-byte aligned fake address: validation fails before any use
    v64 = K.CompressedView(K.CodecDesc(2, 64, 16, 2, 32, 0, K.KVQ_META_F16), 100, A, A, A, A, None)
    o = ctypes.c_void_p(A)
    assert K._lib.kvq_attention_lse(A, 10, ctypes.byref(v64), ctypes.byref(v64), 0, 100, ctypes.c_float(0.0), o,
                                    K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_UNSUPPORTED
    del sz


def test_quantwm_entry_points_rejected_on_host(K):
    """QSAC encode and the PSAC calls refuse bad arguments before any launch:
    candidate counts outside 1..8, compact {s, z} or a joint codec for QSAC,
    a PSAC rank other than 8, d = 64 PSAC attention, misaligned bases."""
    A = 1 << 20
    f0 = ctypes.c_float(0)
    d = K.CodecDesc(12, 128, 256, 2, 16, 0)
    qsac = lambda desc, *a: _err(K, "kvq_encode_qsac", ctypes.byref(desc), *a)
    ok = (A, K.KVQ_BF16, 100, A, A)
    assert qsac(d, *ok, 0, A, A, A, None) == K.KVQ_ERR_INVALID_ARG
    assert qsac(d, *ok, 9, A, A, A, None) == K.KVQ_ERR_INVALID_ARG
    assert qsac(d, A, K.KVQ_BF16, 100, A, None, 4, A, A, A, None) == K.KVQ_ERR_INVALID_ARG
    assert qsac(d, A, K.KVQ_BF16, 100, A, A + 4, 4, A, A, A, None) == K.KVQ_ERR_ALIGNMENT
    assert qsac(K.CodecDesc(12, 128, 256, 2, 16, 0, K.KVQ_META_F16), *ok, 4, A, A, A, None) \
        == K.KVQ_ERR_UNSUPPORTED
    assert qsac(K.CodecDesc(12, 128, 256, 4, 32, 192), *ok, 4, A, A, A, None) == K.KVQ_ERR_UNSUPPORTED
    assert qsac(d, A, K.KVQ_BF16, 0, A, A, 4, A, A, A, None) == K.KVQ_OK

    v = K.CompressedView(d, 1000, A, A, A, A, None)
    coef = lambda view, *a: _err(K, "kvq_psac_coefficients", ctypes.byref(view), *a)
    assert coef(v, A, K.KVQ_BF16, A, 4, A, None) == K.KVQ_ERR_UNSUPPORTED
    assert coef(v, A, K.KVQ_BF16, A + 8, 8, A, None) == K.KVQ_ERR_ALIGNMENT
    assert coef(v, A, K.KVQ_BF16, A, 8, None, None) == K.KVQ_ERR_INVALID_ARG
    assert coef(v, A, 7, A, 8, A, None) == K.KVQ_ERR_INVALID_ARG
    vj = K.CompressedView(K.CodecDesc(12, 128, 256, 4, 32, 192), 1000, A, A, A, A, A)
    assert coef(vj, A, K.KVQ_BF16, A, 8, A, None) == K.KVQ_ERR_UNSUPPORTED
    assert coef(K.CompressedView(d, 0, A, A, A, A, None), None, K.KVQ_BF16, None, 8, None, None) == K.KVQ_OK

    att = lambda kv, vv, *a: _err(K, "kvq_attention_psac_lse", A, 10, ctypes.byref(kv), ctypes.byref(vv), *a)
    assert att(v, v, A, A, 4, 0, 1000, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_UNSUPPORTED
    assert att(v, v, A, None, 8, 0, 1000, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    assert att(v, v, A, A + 4, 8, 0, 1000, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_ALIGNMENT
    assert att(v, v, A, A, 8, 0, 1001, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    v64 = K.CompressedView(K.CodecDesc(12, 64, 256, 2, 16, 0), 1000, A, A, A, A, None)
    assert att(v64, v64, A, A, 8, 0, 1000, f0, A, K.KVQ_F32, A, None, 0, None) == K.KVQ_ERR_UNSUPPORTED


def test_fast_attention_rejected_on_host(K):
    """kvq_fast_attention_lse refuses before any launch: low dims outside
    {64, 128} or above d, a missing or short workspace, misaligned maps, a
    key range outside the keys; zero queries is a no-op."""
    A = 1 << 20
    f0 = ctypes.c_float(0)
    need = 6 * 10 * 12 * 64
    fast = lambda *a: _err(K, "kvq_fast_attention_lse", *a)
    ok = lambda d, dl, ws=A, nws=1 << 20, P=A, t1=100: fast(A, 10, A, A, 100, 12, d, dl, P, A, 0, t1, f0, A,
                                                         K.KVQ_F32, A, ws, nws, None)
    assert ok(128, 32) == K.KVQ_ERR_UNSUPPORTED
    assert ok(128, 96) == K.KVQ_ERR_UNSUPPORTED
    assert ok(64, 128) == K.KVQ_ERR_UNSUPPORTED
    assert ok(128, 64, ws=None, nws=0) == K.KVQ_ERR_WORKSPACE
    assert ok(128, 64, nws=need - 1) == K.KVQ_ERR_WORKSPACE
    assert ok(128, 64, P=A + 2) == K.KVQ_ERR_ALIGNMENT
    assert ok(128, 64, t1=101) == K.KVQ_ERR_INVALID_ARG
    assert fast(None, 0, None, None, 0, 12, 128, 64, None, None, 0, 0, f0, None, K.KVQ_F32, None, None, 0,
                None) == K.KVQ_OK
    n = ctypes.c_size_t()
    assert K._lib.kvq_fast_attention_workspace_size(12, 128, 64, 10, ctypes.byref(n)) == K.KVQ_OK
    assert n.value >= need
    assert K._lib.kvq_fast_attention_workspace_size(12, 128, 32, 10, ctypes.byref(n)) == K.KVQ_ERR_UNSUPPORTED


def test_two_stage_codec_refusals_on_host(K):
    """A second residual stage: only through kvq_encode_stages, per-head codec
    with binary32 {s, z}; the attention calls and QSAC / PSAC refuse two-stage
    views; decode needs the stage-2 arrays."""
    A = 1 << 20
    f0 = ctypes.c_float(0)
    d2 = K.CodecDesc(12, 128, 256, 2, 16, 0, K.KVQ_META_F32, 2)
    sizes = lambda desc: K._lib.kvq_encoded_sizes(ctypes.byref(desc), 10, None, None, None)
    assert sizes(d2) == K.KVQ_OK
    assert sizes(K.CodecDesc(12, 128, 256, 2, 16, 0, K.KVQ_META_F16, 2)) == K.KVQ_ERR_UNSUPPORTED
    assert sizes(K.CodecDesc(12, 128, 256, 4, 32, 192, K.KVQ_META_F32, 2)) == K.KVQ_ERR_UNSUPPORTED
    assert sizes(K.CodecDesc(12, 128, 256, 2, 16, 0, K.KVQ_META_F32, 3)) == K.KVQ_ERR_UNSUPPORTED
    assert sizes(K.CodecDesc(12, 128, 256, 2, 16, 0, K.KVQ_META_F32, -1)) == K.KVQ_ERR_INVALID_ARG
    assert _err(K, "kvq_encode", ctypes.byref(d2), A, K.KVQ_BF16, 100, A, None, A, A, A, None, 0, None) \
        == K.KVQ_ERR_INVALID_ARG
    stages = lambda desc, *a: _err(K, "kvq_encode_stages", ctypes.byref(desc), A, K.KVQ_BF16, 100, A, *a, None)
    assert stages(K.CodecDesc(12, 128, 256, 2, 16, 0), A, A, A, A, A) == K.KVQ_ERR_INVALID_ARG
    assert stages(d2, A, A, A, None, A) == K.KVQ_ERR_INVALID_ARG
    assert stages(d2, A, A, A, A + 8, A) == K.KVQ_ERR_ALIGNMENT
    v2 = K.CompressedView(d2, 1000, A, A, A, A, None, None, None)
    assert _err(K, "kvq_decode", ctypes.byref(v2), A, K.KVQ_F32, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    v2 = K.CompressedView(d2, 1000, A, A, A, A, None, A, A)
    v1 = K.CompressedView(K.CodecDesc(12, 128, 256, 2, 16, 0), 1000, A, A, A, A, None)
    assert _err(K, "kvq_attention_lse", A, 10, ctypes.byref(v2), ctypes.byref(v1), 0, 1000, f0, A, K.KVQ_F32, A,
                None, 0, None) == K.KVQ_ERR_UNSUPPORTED
    assert _err(K, "kvq_psac_coefficients", ctypes.byref(v2), A, K.KVQ_BF16, A, 8, A, None) == K.KVQ_ERR_UNSUPPORTED
    assert _err(K, "kvq_encode_qsac", ctypes.byref(d2), A, K.KVQ_BF16, 100, A, A, 4, A, A, A, None) \
        == K.KVQ_ERR_UNSUPPORTED
