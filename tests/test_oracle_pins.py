"""Pins of the fp64 oracle against facts that do not come from the oracle.

The pages print no worked example and no equations, so the oracle is pinned
by what the mathematics of the Monarch reading fixes:
  * the grid -> (tile, position) map against a hand-written table;
  * the factored product against an explicitly materialised M (brute force);
  * M non-negative and row-stochastic;
  * scores separable across the two Monarch axes  =>  dense softmax attention
    (the case the aligned block structure is built to represent exactly,
    gist.science explainer §2.A);
  * one position per tile, or one tile per sequence  =>  dense attention;
  * each block update is the exact maximiser of the variational objective
    (perturbation test), the objective never decreases and stays below its
    unconstrained maximum sum(logsumexp(S));
  * constant values pass through; mirroring the frame commutes with the op;
  * the KV-cache initialisation equals its eps -> 0 definition.
A plausible mistake (dropped entropy bias, missing beta normalisation, L in
place of L^T, a wrong tile/position index, wrong scale) fails one of these.
"""

import itertools
import math
import os

import numpy as np
import pytest

from oracle import monarch as om
from structured_sparse_attention_grid_b200.workloads import WORKLOADS, Workload, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _separable(B, Hh, g: om.Grid, d, seed):
    w = Workload("sep", B, Hh, g.T, g.H, g.W, d, g.th, g.tw, 1, "f32", seed, "separable",
                 Tk=g.Tkey if g.Tkey != g.T else 0)
    q, k, v = make_inputs(w)
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


def test_block_index_matches_hand_table():
    lines = [l.split() for l in open(os.path.join(GOLDEN, "block_index.txt"))
             if l.strip() and not l.startswith("#")]
    tables, cur = [], None
    for l in lines:
        if l[0] == "grid":
            cur = (tuple(int(x) for x in l[1:]), [])
            tables.append(cur)
        else:
            cur[1].append([int(x) for x in l[1:]])
    assert len(tables) == 2
    for (T, H, W, th, tw), rows in tables:
        idx = om.block_index(T, H, W, th, tw)
        assert idx.tolist() == rows


@pytest.mark.parametrize("T,H,W,th,tw", [(3, 30, 52, 6, 4), (2, 16, 16, 8, 8), (4, 8, 8, 4, 4), (1, 6, 10, 3, 5)])
def test_block_index_is_a_bijection(T, H, W, th, tw):
    idx = om.block_index(T, H, W, th, tw)
    assert idx.shape == (T * (H // th) * (W // tw), th * tw)
    assert np.array_equal(np.sort(idx.ravel()), np.arange(T * H * W))
    # tokens of one tile lie in one frame and one th x tw window
    for c1 in range(0, idx.shape[0], max(1, idx.shape[0] // 7)):
        n = idx[c1]
        t, y, x = n // (H * W), (n // W) % H, n % W
        assert len(set(t)) == 1
        assert y.max() - y.min() == th - 1 and x.max() - x.min() == tw - 1


def _brute_force_M(st: om.HeadState, g: om.Grid):
    """Materialise M over grid tokens with plain loops: row n=(t,y,x) of the
    query grid, column m of the key grid."""
    Nq, Nk = g.Nq, g.Nk
    M = np.zeros((Nq, Nk))
    nty, ntx = g.H // g.th, g.W // g.tw
    coords = lambda n: (n // (g.H * g.W), (n // g.W) % g.H, n % g.W)
    for n in range(Nq):
        t, y, x = coords(n)
        a1 = (t * nty + y // g.th) * ntx + x // g.tw
        a2 = (y % g.th) * g.tw + x % g.tw
        for m in range(Nk):
            tk, yk, xk = coords(m)
            c1 = (tk * nty + yk // g.th) * ntx + xk // g.tw
            c2 = (yk % g.th) * g.tw + xk % g.tw
            M[n, m] = st.L[a2, a1, c1] * st.R[c1, a2, c2]
    return M


@pytest.mark.parametrize("g,iters", [(om.Grid(2, 4, 4, 2, 2), 1), (om.Grid(2, 4, 4, 2, 2), 3),
                                      (om.Grid(1, 4, 6, 2, 3, Tk=3), 2)])
def test_factored_output_equals_explicit_M(g, iters):
    d = 6
    q = _rand((1, 1, g.Nq, d), 1)
    k = _rand((1, 1, g.Nk, d), 2)
    v = _rand((1, 1, g.Nk, d), 3)
    out, states = om.monarch_attention(q, k, v, g, iters, return_states=True)
    M = _brute_force_M(states[(0, 0)], g)
    assert (M >= 0).all()
    np.testing.assert_allclose(M.sum(axis=1), 1.0, atol=1e-13)
    np.testing.assert_allclose(out[0, 0], M @ v[0, 0], atol=1e-13)


@pytest.mark.parametrize("g,iters", [
    (om.Grid(4, 8, 8, 4, 4), 1),
    (om.Grid(4, 8, 8, 4, 4), 2),
    (om.Grid(3, 6, 8, 3, 2), 3),
    (om.Grid(2, 4, 6, 2, 3, Tk=5), 1),
    (om.Grid(2, 4, 6, 2, 3, Tk=5), 2),
])
def test_separable_scores_give_dense_attention(g, iters):
    q, k, v = _separable(1, 2, g, 16, seed=11)
    out = om.monarch_attention(q, k, v, g, iters)
    ref = om.dense_attention(q, k, v)
    np.testing.assert_allclose(out, ref, atol=1e-12, rtol=0)


def test_toy_separable_workload_is_dense():
    w = WORKLOADS["toy_256_f32_separable"]
    q, k, v = (t.double().numpy() for t in make_inputs(w))
    g = om.Grid(w.T, w.H, w.W, w.th, w.tw)
    out = om.monarch_attention(q, k, v, g, w.iters)
    np.testing.assert_allclose(out, om.dense_attention(q, k, v), atol=1e-12, rtol=0)


def test_generic_inputs_are_not_dense():
    """Guard for the two tests above: on generic inputs the Monarch output
    differs from dense attention, so equality there is a real property."""
    g = om.Grid(2, 4, 4, 2, 2)
    q, k, v = (_rand((1, 1, g.Nq, 8), s) for s in (5, 6, 7))
    out = om.monarch_attention(q, k, v, g, 2)
    assert np.abs(out - om.dense_attention(q, k, v)).max() > 1e-3


@pytest.mark.parametrize("iters", [1, 2])
def test_one_position_per_tile_is_dense(iters):
    g = om.Grid(2, 3, 4, 1, 1)  # b2 = 1: R = [1], L spans every token
    q, k, v = (_rand((1, 2, g.Nq, 8), s) for s in (21, 22, 23))
    out = om.monarch_attention(q, k, v, g, iters)
    np.testing.assert_allclose(out, om.dense_attention(q, k, v), atol=1e-13, rtol=0)


@pytest.mark.parametrize("iters", [1, 3])
def test_one_tile_per_sequence_is_dense(iters):
    g = om.Grid(1, 4, 6, 4, 6)  # b1 = 1: L = [1], R spans every token
    q, k, v = (_rand((2, 1, g.Nq, 8), s) for s in (31, 32, 33))
    out = om.monarch_attention(q, k, v, g, iters)
    np.testing.assert_allclose(out, om.dense_attention(q, k, v), atol=1e-13, rtol=0)


def test_dense_reference_matches_loops():
    q, k, v = (_rand((1, 1, 5, 3), s) for s in (41, 42, 43))
    s = 1 / math.sqrt(3)
    ref = np.zeros((5, 3))
    for i in range(5):
        w = [math.exp(s * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(3))) for j in range(5)]
        tot = sum(w)
        for c in range(3):
            ref[i, c] = sum(w[j] * v[0, 0, j, c] for j in range(5)) / tot
    np.testing.assert_allclose(om.dense_attention(q, k, v)[0, 0], ref, atol=1e-14)


@pytest.mark.parametrize("g", [om.Grid(3, 4, 4, 2, 2), om.Grid(1, 4, 4, 2, 2, Tk=3)])
def test_constant_values_pass_through(g):
    q, k = _rand((1, 2, g.Nq, 8), 51), _rand((1, 2, g.Nk, 8), 52)
    c = _rand((8,), 53)
    v = np.broadcast_to(c, (1, 2, g.Nk, 8)).copy()
    out = om.monarch_attention(q, k, v, g, 2)
    np.testing.assert_allclose(out, np.broadcast_to(c, out.shape), atol=1e-13)


@pytest.mark.parametrize("g", [om.Grid(2, 4, 6, 2, 3), om.Grid(1, 4, 6, 2, 3, Tk=3)])
def test_mirroring_the_frame_commutes(g):
    d = 8
    q, k, v = _rand((1, 1, g.Nq, d), 61), _rand((1, 1, g.Nk, d), 62), _rand((1, 1, g.Nk, d), 63)

    def flip(a, frames):
        return a.reshape(1, 1, frames, g.H, g.W, d)[:, :, :, :, ::-1].reshape(a.shape)

    out = om.monarch_attention(q, k, v, g, 3)
    out_f = om.monarch_attention(flip(q, g.T), flip(k, g.Tkey), flip(v, g.Tkey), g, 3)
    np.testing.assert_allclose(out_f, flip(out, g.T), atol=1e-13)


def _objective_setup():
    g = om.Grid(2, 4, 4, 2, 2)
    d = 6
    scale = 1 / math.sqrt(d)
    q, k = _rand((1, 1, g.Nq, d), 71) * 1.5, _rand((1, 1, g.Nk, d), 72) * 1.5
    iq = om.block_index(g.T, g.H, g.W, g.th, g.tw)
    return g, scale, q[0, 0][iq], k[0, 0][iq]


def _perturb(P, rng, eps):
    """Random feasible direction on the row simplex (rows of the last axis)."""
    D = rng.standard_normal(P.shape)
    D -= (P * D).sum(axis=-1, keepdims=True)  # then sum(P*D) = 0 on every row
    return P + eps * P * D / (1 + np.abs(D).max())


def test_block_updates_are_exact_maximisers():
    g, scale, qb, kb = _objective_setup()
    rng = np.random.default_rng(0)
    st1 = om.monarch_head(qb, kb, kb, g, 1, scale)
    L1 = st1.L
    # R step given L1
    qt = om._column_qtilde(L1, qb)
    R2, h2 = om._r_step(qt, kb, scale)
    F_opt = om.head_objective(L1, R2, qb, kb, scale)
    assert F_opt >= om.head_objective(L1, st1.R, qb, kb, scale) - 1e-12
    for _ in range(40):
        Rp = _perturb(R2, rng, 1e-3)
        np.testing.assert_allclose(Rp.sum(-1), 1.0, atol=1e-13)
        assert om.head_objective(L1, Rp, qb, kb, scale) <= F_opt + 1e-12
    # L step given R2
    L2, _ = om._l_step(qb, np.matmul(R2, kb), h2, scale)
    F_opt = om.head_objective(L2, R2, qb, kb, scale)
    for _ in range(40):
        Lp = _perturb(L2, rng, 1e-3)
        assert om.head_objective(Lp, R2, qb, kb, scale) <= F_opt + 1e-12


def test_objective_is_monotone_and_bounded():
    g, scale, qb, kb = _objective_setup()
    st = om.monarch_head(qb, kb, kb, g, 8, scale, track_objective=True)
    F = np.array(st.objective)
    assert (np.diff(F) >= -1e-10).all()
    S = scale * np.einsum("apd,cjd->apcj", qb, kb).reshape(qb.shape[0] * qb.shape[1], -1)
    bound = om._logsumexp_last(S).sum()
    assert F[-1] <= bound + 1e-10
    assert F[-1] > F[0]


def test_kv_initialisation_is_the_eps_limit():
    g = om.Grid(2, 4, 6, 2, 3, Tk=5)
    d = 5
    qb = _rand((g.b1q, g.b2, d), 81)
    off = (g.Tkey - g.T) * g.tiles_per_frame
    eps = 1e-9
    aligned = np.zeros((g.b1q, g.b1k))
    aligned[np.arange(g.b1q), np.arange(g.b1q) + off] = 1.0
    L0 = (1 - eps) * aligned + eps / g.b1k
    beta = L0.sum(axis=0)
    qt_eps = np.einsum("ac,apd->cpd", L0, qb) / beta[:, None, None]
    np.testing.assert_allclose(om.initial_qtilde(qb, g), qt_eps, atol=1e-7)


def test_self_attention_initialisation_is_identity():
    g = om.Grid(2, 4, 6, 2, 3)
    qb = _rand((g.b1q, g.b2, 4), 91)
    np.testing.assert_array_equal(om.initial_qtilde(qb, g), qb)


def test_flop_counts_match_hand_values():
    g = om.Grid(3, 30, 52, 6, 4)
    assert (g.b1q, g.b2) == (195, 24)
    FL = 2 * 24 * 195 * 195 * 128
    FR = 2 * 195 * 24 * 24 * 128
    assert om.monarch_flops(g, 128, 2, 1, 12) == 12 * (4 * FL + 5 * FR)
    assert abs(om.monarch_flops(g, 128, 2, 1, 12) / 1e9 - 12.94) < 0.01
    assert om.dense_flops(g, 128, 1, 12) == 4 * 12 * 4680 * 4680 * 128


# ---- frame-chunk causal mask (D9) -------------------------------------------

def _masked_dense(q, k, v, g: om.Grid):
    mask = om.frame_chunk_mask(g.T, g.Tkey, g.H, g.W, g.chunk_frames)
    return om.dense_attention(q, k, v, mask=mask)


def test_frame_chunk_mask_matches_hand_table():
    # 3 frames, chunks of 2: frames {0, 1} | {2}; one token per frame
    m = om.frame_chunk_mask(3, 3, 1, 1, 2).astype(int)
    np.testing.assert_array_equal(m, [[1, 1, 0], [1, 1, 0], [1, 1, 1]])
    # tile-level visibility of a 2-tile-per-frame grid agrees with it
    g = om.Grid(3, 2, 4, 2, 2, chunk_frames=2)
    vis = g.visible().astype(int)
    expect = np.kron(np.array([[1, 1, 0], [1, 1, 0], [1, 1, 1]]), np.ones((2, 2), dtype=int))
    np.testing.assert_array_equal(vis, expect)


@pytest.mark.parametrize("C", [5, 6, 9])
def test_one_chunk_mask_is_the_bidirectional_result(C):
    g0 = om.Grid(5, 4, 6, 2, 3)
    g1 = om.Grid(5, 4, 6, 2, 3, chunk_frames=C)
    q, k, v = (_rand((1, 2, g0.Nq, 8), s) for s in (31, 32, 33))
    np.testing.assert_array_equal(om.monarch_attention(q, k, v, g1, 2), om.monarch_attention(q, k, v, g0, 2))


@pytest.mark.parametrize("g,iters", [
    (om.Grid(6, 4, 4, 2, 2, chunk_frames=2), 1),
    (om.Grid(6, 4, 4, 2, 2, chunk_frames=2), 2),
    (om.Grid(5, 4, 6, 2, 3, chunk_frames=1), 3),
    (om.Grid(7, 4, 4, 4, 2, chunk_frames=3), 2),   # ragged last chunk
])
def test_separable_scores_with_chunk_mask_give_masked_dense_attention(g, iters):
    q, k, v = _separable(1, 2, g, 16, seed=13)
    out = om.monarch_attention(q, k, v, g, iters)
    np.testing.assert_allclose(out, _masked_dense(q, k, v, g), atol=1e-12, rtol=0)


def test_masked_M_is_row_stochastic_and_zero_outside_the_mask():
    g = om.Grid(4, 4, 4, 2, 2, chunk_frames=2)
    q, k, v = (_rand((1, 1, g.Nq, 6), s) for s in (41, 42, 43))
    out, states = om.monarch_attention(q, k, v, g, 2, return_states=True)
    M = _brute_force_M(states[(0, 0)], g)
    mask = om.frame_chunk_mask(g.T, g.Tkey, g.H, g.W, g.chunk_frames)
    assert (M >= 0).all() and (M[~mask] == 0).all()
    np.testing.assert_allclose(M.sum(axis=1), 1.0, atol=1e-13)
    np.testing.assert_allclose(out[0, 0], M @ v[0, 0], atol=1e-13)
