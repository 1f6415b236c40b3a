"""Shared pieces of the GPU parity tests: the oracle's output per workload
(computed once per test session and reused), the per-head comparison and the
tolerances.

Tolerances: fp32 max|err| <= 1e-4; bf16/f16 max|err| <= 2e-2 * RMS of the
oracle output, checked head by head against that head's own RMS (a head with
a small output would otherwise hide its error under another head's RMS)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import monarch as om

TOL_F32 = 1e-4
TOL_LOWP = 2e-2
# significant bits of a stored output element: one round-to-nearest store of
# a bf16 (f16) value moves it by at most 2^-8 (2^-11) of its magnitude
STORE_BITS = {"bf16": 8, "f16": 11}

_ORACLE = {}


def grid_of(w):
    return om.Grid(w.T, w.H, w.W, w.th, w.tw, Tk=w.Tkey if w.Tk else None, chunk_frames=w.chunk_frames)


def oracle_out(w, q, k, v, heads=None):
    """The fp64 oracle's output for workload w on the given inputs (which must
    be the workload's own seeded inputs when w is a named workload: the
    result is cached under the workload's name and head list)."""
    key = (w, tuple(heads) if heads else None)
    if key not in _ORACLE:
        qn, kn, vn = (t.double().numpy() for t in (q, k, v))
        _ORACLE[key] = om.monarch_attention(qn, kn, vn, grid_of(w), w.iters, heads=heads)
    return _ORACLE[key]


def compare_per_head(w, got, ref, heads=None, store_bits=None):
    """Checks every listed head against its own bar; returns the worst
    (error / bar) ratio.  store_bits: the output was stored in a 16-bit type
    with this many significant bits, which adds 2^-store_bits |ref| per
    element to the bar."""
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    hs = heads or [(b, h) for b in range(w.B) for h in range(w.heads)]
    worst = 0.0
    for b, h in hs:
        r = ref[b, h]
        e = np.abs(got[b, h] - r)
        if w.dtype == "f32":
            bar = np.full_like(r, TOL_F32)
        else:
            bar = np.full_like(r, TOL_LOWP * float(np.sqrt((r ** 2).mean())))
        if store_bits:
            bar = bar + 2.0 ** -store_bits * np.abs(r)
        ratio = float((e / bar).max())
        worst = max(worst, ratio)
        assert ratio <= 1.0, (f"{w.name} head ({b},{h}): max|err|/bar {ratio:.3f} "
                              f"(max|err| {float(e.max()):.3e})")
    return worst
