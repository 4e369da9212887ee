"""bench.py's host-side choices on CPU: the sweep's points cover every code
width pair, group size, centre count, history length and query-chunk length
of the 12-head sweep; the default workload of the headline line is the
largest single-GPU one."""

import itertools
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_sweep_points_cover_the_sweep():
    pts = bench.sweep_points()
    assert len(set(pts)) == len(pts)
    assert {(bk, bv) for _, _, bk, bv, _, _ in pts} == set(itertools.product((2, 4), (2, 4)))
    assert {G for *_, G, _ in pts} == {16, 32, 64}
    assert {C for *_, C in pts} == {64, 256, 1024}
    assert {T for T, *_ in pts} == {4096, 8192, 16384, 32768, 65536, 131072}
    assert {Tq for _, Tq, *_ in pts} == {1560, 4680}


def test_default_run_is_the_headline_workload(monkeypatch):
    from kv_cache_compression_head_b200 import synth

    monkeypatch.setattr(sys, "argv", ["bench.py"])
    args = bench.parse_args()
    assert args.gpus == 1 and args.warmup >= 3 and args.steps >= 1 and args.impl == "kvq"
    assert args.workload == "14b"
    size = {n: w.num_heads * w.history_tokens for n, w in synth.WORKLOADS.items()}
    assert max(size, key=size.get) == args.workload
