"""kvq_fit_centroids_static -- the fit for callers that cannot allocate device
memory on demand (a serving runtime whose HBM is pre-reserved and pooled, or
a C caller with no allocator at hand) -- must give exactly what
kvq_fit_centroids gives with a caller workspace.

Two calls of the static-scratch entry point run back to back (different
shapes and input dtypes) before the workspace fits are computed, so state
left in the shared scratch by the first call would show up in the second.
Collected last on purpose: it stays meaningful both alone in a fresh process
and after every other test has run."""

import ctypes

import numpy as np
import pytest
import torch

from kv_cache_compression_head_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(a):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def test_static_scratch_fit_matches_workspace_fit():
    from kv_cache_compression_head_b200 import kvq as K

    wan = synth.workload("wan13b")
    tiny = synth.workload("tiny")
    cases = [
        (K.Codec(wan.num_heads, wan.head_dim, wan.num_centroids, wan.bits_k, wan.group_size),
         _dev(synth.make_history(wan, "K", max_tokens=8192)), wan.kmeans_iters),
        (K.Codec(tiny.num_heads, tiny.head_dim, tiny.num_centroids, tiny.bits_k, tiny.group_size),
         _dev(synth.make_history(tiny, "V")), tiny.kmeans_iters),
    ]
    outs = []
    for codec, x, iters in cases:  # two static-scratch calls in a row, through the C ABI
        out = torch.full((codec.num_heads, codec.num_centroids, codec.head_dim), float("nan"),
                         dtype=torch.bfloat16, device="cuda")
        d = codec.c()
        rc = K._lib.kvq_fit_centroids_static(ctypes.byref(d), x.data_ptr(), K._dtype_code(x), x.shape[0], iters,
                                             out.data_ptr(), torch.cuda.current_stream().cuda_stream or None)
        assert rc == K.KVQ_OK, K.status_string(rc)
        outs.append(out)
    torch.cuda.synchronize()
    for (codec, x, iters), out in zip(cases, outs):
        ref = torch.empty_like(out)
        K.kvq_fit_centroids(codec, x, iters, ref)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert K.kvq_last_device_status() == K.KVQ_OK

    # a request beyond the fixed scratch is refused before any launch
    big = K.Codec(40, 128, 512, 4, 32)
    d = big.c()
    rc = K._lib.kvq_fit_centroids_static(ctypes.byref(d), outs[0].data_ptr(), K.KVQ_BF16, 93600, 2,
                                         outs[0].data_ptr(), None)
    assert rc == K.KVQ_ERR_WORKSPACE
