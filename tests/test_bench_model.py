"""CPU checks of the bench's work model, which every reported TFLOP/s and
roofline fraction divides by: the L- and R-step contraction sizes against
their closed forms, and the visible fraction of the frame-chunk mask against
the oracle's mask counted entry by entry."""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import monarch as om  # noqa: E402
from structured_sparse_attention_grid_b200.workloads import WORKLOADS  # noqa: E402


def test_contraction_sizes_of_the_chunk_workload():
    w = WORKLOADS["chunk_4680_bf16"]          # 12 heads, 3 x 30 x 52, d 128, 6 x 4 tiles, 2 iterations
    m = bench.work_model(w)
    b1, b2, d = 3 * 5 * 13, 24, 128
    assert m["FL"] == 2.0 * b2 * b1 * b1 * d
    assert m["FR"] == 2.0 * b1 * b2 * b2 * d
    assert m["flops"] == 12 * (2 * 2 * m["FL"] + (2 * 2 + 1) * m["FR"])
    assert m["dense_flops"] == 4.0 * 12 * 4680 * 4680 * d
    bm = bench.backward_work_model(w)
    assert bm["flops"] == 12 * (4 * m["FL"] + 6 * m["FR"])


def test_kv_cache_sizes_use_the_key_tiles():
    w = WORKLOADS["kvcache_4680x32760_bf16"]
    m = bench.work_model(w)
    assert m["FL"] == 2.0 * 24 * 195 * 1365 * 128
    assert m["FR"] == 2.0 * 1365 * 24 * 24 * 128


def test_visible_fraction_counts_the_oracle_mask():
    for name in ("train_32760_bf16_causal", "full_32760_bf16"):
        w = WORKLOADS[name]
        g = om.Grid(w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
        vis = g.visible() if w.chunk_frames else np.ones((1, 1), dtype=bool)
        assert abs(bench.visible_fraction(w) - float(vis.mean())) < 1e-12


def test_roofline_bytes_of_the_chunk_workload():
    """Compulsory call bytes = Q, K, V, O in the input dtype (57.5 MB for 12
    heads of 4680 tokens at d = 128, bf16); the R-step launch moves q~ (or q),
    k in and k~ out, and in the final launch also v in and z out, plus h."""
    w = WORKLOADS["chunk_4680_bf16"]
    m = bench.work_model(w)
    n = 12 * 4680 * 128 * 2                      # bytes of one [heads, N, d] bf16 tensor
    assert m["io_bytes"] == 4 * n
    hb = 12 * 24 * 195 * 4
    assert m["phases"]["r_step"]["bytes"] == (3 * n + 5 * n) / 2 + hb
    peaks = {"bf16_tflops": 1646.3, "hbm_gbs": 6550.4, "source": "measured"}
    r = bench.call_roofline(w, m, peaks, 1.0)
    assert abs(r["roofline_ms"] - 4 * n / 6550.4e9 * 1e3) < 1e-12 and r["bound"] == "hbm"
    assert abs(r["roofline_ms"] * 1e3 - 8.78) < 0.01   # microseconds
