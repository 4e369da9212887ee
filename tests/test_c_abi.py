"""The C ABI consumed from plain C, without Python or torch in the process: a
C11 program that includes include/kvq.h (gcc -std=c11 -Wall -Wextra -Werror
-pedantic) and links libkvq.so calls the host-only entry points -- status
strings, the encoded array sizes against their closed forms for both {s, z}
formats, the fit workspace against the binding's figure -- and argument
refusals that return before any device work.  CPU only."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "kv_cache_compression_head_b200")
LIB = os.path.join(PKG, "libkvq.so")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "kvq.h"

int main(void)
{
    kvq_codec_desc d;
    size_t ib = 0, cb = 0, mb = 0, ws = 0;
    memset(&d, 0, sizeof d);
    d.num_heads = 12;
    d.head_dim = 128;
    d.num_centroids = 256;
    d.bits = 2;
    d.group_size = 16;
    if (kvq_encoded_sizes(&d, 32760, &ib, &cb, &mb) != KVQ_OK)
        return 2;
    printf("f32 %zu %zu %zu\n", ib, cb, mb);
    d.meta_format = KVQ_META_F16;
    if (kvq_encoded_sizes(&d, 32760, &ib, &cb, &mb) != KVQ_OK)
        return 3;
    printf("f16 %zu %zu %zu\n", ib, cb, mb);
    d.meta_format = KVQ_META_F32;
    d.bits = 4;
    d.group_size = 32;
    if (kvq_encoded_sizes(&d, 1001, &ib, &cb, &mb) != KVQ_OK)
        return 4;
    printf("b4 %zu %zu %zu\n", ib, cb, mb);
    d.bits = 2;
    d.group_size = 16;
    if (kvq_workspace_size(KVQ_OP_FIT, &d, 32760, 0, &ws) != KVQ_OK)
        return 5;
    printf("fit %zu\n", ws);
    printf("null_desc %d\n", (int)kvq_encoded_sizes(NULL, 1, &ib, &cb, &mb));
    d.bits = 3;
    printf("bits3 %d\n", (int)kvq_encoded_sizes(&d, 1, &ib, &cb, &mb));
    d.bits = 2;
    d.group_size = 12;
    printf("group12 %d\n", (int)kvq_encoded_sizes(&d, 1, &ib, &cb, &mb));
    d.group_size = 16;
    printf("encode_null %d\n", (int)kvq_encode(&d, NULL, KVQ_BF16, 5, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL));
    printf("timeout %s\n", kvq_status_string(KVQ_ERR_DEVICE_TIMEOUT));
    printf("ok %s\n", kvq_status_string(KVQ_OK));
    return 0;
}
"""


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    assert os.path.exists(LIB), "libkvq.so is not built (python -m kv_cache_compression_head_b200.build)"
    d = tmp_path_factory.mktemp("c_abi")
    src, exe = d / "use_kvq.c", d / "use_kvq"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", PKG, "-lkvq", f"-Wl,-rpath,{PKG}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    return dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())


def test_encoded_sizes_closed_forms(program):
    H, T, d = 12, 32760, 128
    # idx 2 B, codes d b / 8 B, {s, z} (d / G) x 8 B (binary32) or x 4 B (binary16) per token-head
    assert program["f32"] == f"{2 * H * T} {H * T * d * 2 // 8} {H * T * (d // 16) * 8}"
    assert program["f16"] == f"{2 * H * T} {H * T * d * 2 // 8} {H * T * (d // 16) * 4}"
    assert program["b4"] == f"{2 * H * 1001} {H * 1001 * d * 4 // 8} {H * 1001 * (d // 32) * 8}"


def test_fit_workspace_matches_the_binding(program):
    from kv_cache_compression_head_b200 import kvq

    assert int(program["fit"]) == kvq.workspace_size(kvq.KVQ_OP_FIT, kvq.Codec(12, 128, 256, 2, 16), 32760)


def test_refusals_before_device_work(program):
    assert int(program["null_desc"]) == 1       # KVQ_ERR_INVALID_ARG
    assert int(program["bits3"]) == 2           # KVQ_ERR_UNSUPPORTED
    assert int(program["group12"]) == 1         # G not dividing d
    assert int(program["encode_null"]) == 1     # null history and outputs
    assert program["timeout"] and program["ok"]
