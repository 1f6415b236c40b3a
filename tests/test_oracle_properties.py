"""Property-based pins of the fp64 oracle over randomly drawn tiny grids.

The fixed-shape pins in test_oracle_pins.py check each fact on a handful of
hand-picked grids.  Here hypothesis draws the grid (tile shape, tiles per
frame, query frames, extra cached key frames, frame-chunk mask, refinement
steps, head dimension) and the same facts must hold on every draw:
  * the factored output equals M V for the Monarch matrix
    M[(a1,a2),(c1,c2)] = L_a2[a1,c1] R_c1[a2,c2] materialised entry by entry
    from the token coordinates (gist.science explainer §2.A, block alignment;
    §2.B, tiled parameterisation), and M is non-negative, row-stochastic and
    zero outside the frame-chunk mask;
  * with scores separable across the two Monarch axes the output is the
    (masked) dense softmax attention, the case the aligned blocks represent
    exactly.
The backward of the one-step forward (self-attention, optional mask) must
match central finite differences of the forward in random directions, and
keep the two exact invariants of a row-stochastic operator: sum_keys dv =
sum_queries dy, and sum_keys dk = 0.
Draws are derandomised, so the CPU suite sees the same cases on every run.
Planted mistakes (positions reversed inside every tile, a missing beta
normalisation) fail one of the two properties on a fixed masked KV grid.
"""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import monarch as om
from structured_sparse_attention_grid_b200.workloads import Workload, make_inputs


@st.composite
def grids(draw):
    th, tw = draw(st.integers(1, 3)), draw(st.integers(1, 3))
    nty, ntx = draw(st.integers(1, 2)), draw(st.integers(1, 3))
    T = draw(st.integers(1, 3))
    extra = draw(st.integers(0, 2))
    C = draw(st.sampled_from([0, 0, 1, 2]))
    return om.Grid(T, th * nty, tw * ntx, th, tw, Tk=T + extra if extra else None, chunk_frames=C)


def _materialise_M(s: om.HeadState, g: om.Grid) -> np.ndarray:
    """M over grid tokens from the token coordinates, by plain loops."""
    nty, ntx = g.H // g.th, g.W // g.tw
    hw = g.H * g.W

    def block(n):
        t, y, x = n // hw, (n // g.W) % g.H, n % g.W
        return (t * nty + y // g.th) * ntx + x // g.tw, (y % g.th) * g.tw + x % g.tw

    M = np.zeros((g.Nq, g.Nk))
    for n in range(g.Nq):
        a1, a2 = block(n)
        for m in range(g.Nk):
            c1, c2 = block(m)
            M[n, m] = s.L[a2, a1, c1] * s.R[c1, a2, c2]
    return M


def _mask(g: om.Grid) -> np.ndarray:
    if not g.chunk_frames:
        return np.ones((g.Nq, g.Nk), dtype=bool)
    return om.frame_chunk_mask(g.T, g.Tkey, g.H, g.W, g.chunk_frames)


def _check_factored(g, iters, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, g.Nq, d))
    k = rng.standard_normal((1, 1, g.Nk, d))
    v = rng.standard_normal((1, 1, g.Nk, d))
    out, states = om.monarch_attention(q, k, v, g, iters, return_states=True)
    M = _materialise_M(states[(0, 0)], g)
    assert (M >= 0).all()
    assert (M[~_mask(g)] == 0).all()
    np.testing.assert_allclose(M.sum(axis=1), 1.0, atol=1e-12)
    np.testing.assert_allclose(out[0, 0], M @ v[0, 0], atol=1e-12)


def _check_separable(g, iters, seed):
    w = Workload("sep", 1, 1, g.T, g.H, g.W, 8, g.th, g.tw, iters, "f32", seed, "separable",
                 Tk=g.Tkey if g.Tkey != g.T else 0)
    q, k, v = (t.double().numpy() for t in make_inputs(w))
    out = om.monarch_attention(q, k, v, g, iters)
    ref = om.dense_attention(q, k, v, mask=_mask(g))
    np.testing.assert_allclose(out, ref, atol=1e-11, rtol=0)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(g=grids(), iters=st.integers(1, 3), d=st.sampled_from([2, 3, 5]), seed=st.integers(0, 2**16))
def test_factored_output_is_M_times_V_on_random_grids(g, iters, d, seed):
    _check_factored(g, iters, d, seed)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(g=grids(), iters=st.integers(1, 3), seed=st.integers(0, 2**16))
def test_separable_scores_give_masked_dense_attention_on_random_grids(g, iters, seed):
    _check_separable(g, iters, seed)


# Planted mistakes (in the oracle, on the CPU): each must fail a property.
_MASKED_KV = om.Grid(3, 4, 6, 2, 3, Tk=4, chunk_frames=2)


def test_positions_reversed_inside_tiles_fail_the_explicit_M(monkeypatch):
    orig = om.block_index
    monkeypatch.setattr(om, "block_index", lambda *a: orig(*a)[:, ::-1].copy())
    with pytest.raises(AssertionError):
        _check_factored(_MASKED_KV, 2, 3, seed=5)


def test_missing_beta_normalisation_fails_the_separable_case(monkeypatch):
    def no_beta(L, qb):
        return np.swapaxes(np.matmul(np.swapaxes(L, 1, 2), np.swapaxes(qb, 0, 1)), 0, 1)
    monkeypatch.setattr(om, "_column_qtilde", no_beta)
    with pytest.raises(AssertionError):
        _check_separable(_MASKED_KV, 2, seed=5)


def test_unmutated_oracle_passes_the_planted_cases():
    _check_factored(_MASKED_KV, 2, 3, seed=5)
    _check_separable(_MASKED_KV, 2, seed=5)


@st.composite
def self_grids(draw):
    g = draw(grids())
    return om.Grid(g.T, g.H, g.W, g.th, g.tw, chunk_frames=g.chunk_frames)


@settings(max_examples=30, deadline=None, derandomize=True)
@given(g=self_grids(), d=st.sampled_from([2, 3, 5]), seed=st.integers(0, 2**16))
def test_backward_matches_finite_differences_on_random_grids(g, d, seed):
    rng = np.random.default_rng(seed)
    q, k, v, dy = (rng.standard_normal((1, 1, g.Nq, d)) for _ in range(4))
    grads = dict(zip("qkv", om.monarch_attention_backward(q, k, v, dy, g)))
    eps = 1e-6
    for which in "qkv":
        delta = rng.standard_normal(q.shape)

        def f(x):
            args = {"q": q, "k": k, "v": v, which: x}
            return float((om.monarch_attention(args["q"], args["k"], args["v"], g, 1) * dy).sum())
        x = {"q": q, "k": k, "v": v}[which]
        fd = (f(x + eps * delta) - f(x - eps * delta)) / (2 * eps)
        an = float((grads[which] * delta).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (which, fd, an)
    # a row-stochastic operator: dv = M^T dy keeps the column sums of dy; the
    # scores enter through softmaxes, whose gradients sum to zero over keys
    np.testing.assert_allclose(grads["v"].sum(axis=2), dy.sum(axis=2), atol=1e-10, rtol=0)
    assert np.abs(grads["k"].sum(axis=2)).max() <= 1e-10 * max(1.0, np.abs(grads["k"]).sum(axis=2).max())
