"""Pins of the oracle's backward (iters = 1, self-attention): gradients
against central finite differences of the forward oracle (independent of the
backward's formulas), the one-position-per-tile case against the textbook
dense-attention gradient, and planted mistakes that these pins catch."""

import numpy as np
import pytest

from oracle import monarch as om


def _inputs(g, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((1, 2, g.Nq, d)) for _ in range(4)]


def _directional(g, q, k, v, dy, which, delta, eps=1e-6):
    def f(x):
        args = {"q": q, "k": k, "v": v}
        args[which] = x
        return float((om.monarch_attention(args["q"], args["k"], args["v"], g, 1) * dy).sum())
    x = {"q": q, "k": k, "v": v}[which]
    return (f(x + eps * delta) - f(x - eps * delta)) / (2 * eps)


GRIDS = [
    om.Grid(2, 4, 4, 2, 2),
    om.Grid(3, 4, 6, 2, 3),
    om.Grid(4, 4, 4, 2, 2, chunk_frames=2),
    om.Grid(5, 2, 4, 2, 2, chunk_frames=2),   # ragged last chunk
    om.Grid(2, 3, 4, 1, 1),                   # one position per tile
]


@pytest.mark.parametrize("g", GRIDS, ids=[f"{g.T}x{g.H}x{g.W}_{g.th}x{g.tw}_C{g.chunk_frames}" for g in GRIDS])
def test_backward_matches_finite_differences(g):
    q, k, v, dy = _inputs(g, 6, seed=3)
    grads = dict(zip("qkv", om.monarch_attention_backward(q, k, v, dy, g)))
    rng = np.random.default_rng(9)
    for which in "qkv":
        delta = rng.standard_normal(q.shape)
        fd = _directional(g, q, k, v, dy, which, delta)
        an = float((grads[which] * delta).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (which, fd, an)


def _dense_grad(q, k, v, dy, scale):
    """Textbook softmax-attention gradient, per (batch, head)."""
    s = scale * q @ np.swapaxes(k, -1, -2)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    dv = np.swapaxes(p, -1, -2) @ dy
    dp = dy @ np.swapaxes(v, -1, -2)
    ds = p * (dp - (p * dp).sum(-1, keepdims=True))
    return scale * ds @ k, scale * np.swapaxes(ds, -1, -2) @ q, dv


def test_one_position_per_tile_gives_the_dense_gradient():
    g = om.Grid(3, 4, 6, 1, 1)
    q, k, v, dy = _inputs(g, 8, seed=5)
    got = om.monarch_attention_backward(q, k, v, dy, g)
    ref = _dense_grad(q, k, v, dy, 1 / np.sqrt(8))
    for a, b in zip(got, ref):
        np.testing.assert_allclose(a, b, atol=1e-12, rtol=0)


def _fd_ok():
    g = om.Grid(3, 4, 6, 2, 3)
    q, k, v, dy = _inputs(g, 6, seed=3)
    grads = dict(zip("qkv", om.monarch_attention_backward(q, k, v, dy, g)))
    rng = np.random.default_rng(9)
    for which in "qkv":
        delta = rng.standard_normal(q.shape)
        fd = _directional(g, q, k, v, dy, which, delta)
        if abs(fd - float((grads[which] * delta).sum())) > 1e-6 * max(1.0, abs(fd)):
            return False
    return True


def test_unmutated_backward_passes():
    assert _fd_ok()


def _mutant(old, new):
    """The oracle backward with one textual mistake planted in its source."""
    import inspect
    src = inspect.getsource(om.monarch_head_backward)
    assert old in src
    ns = dict(vars(om))
    exec(src.replace(old, new), ns)
    return ns["monarch_head_backward"]


# Dropping the "+1" of -(log R + 1) is NOT a mistake: it shifts a row of dR by a
# constant, which the softmax backward R * (dR - rowsum(R * dR)) cancels.
@pytest.mark.parametrize("old,new", [
    ("- dh[..., None] * (np.log(R) + 1.0)", "+ dh[..., None] * (np.log(R) + 1.0)"),   # entropy sign
    ("dk = np.matmul(np.swapaxes(R, 1, 2), dkt) + scale",
     "dk = np.matmul(np.swapaxes(R, 1, 2), dkt) * 0 + scale"),                        # R^T dk~ lost
    ("dz_p = np.matmul(np.swapaxes(L, 1, 2), dy_p)", "dz_p = np.matmul(L, dy_p)"),       # L for L^T
    ("dq = dq + scale * np.matmul(dSr, kb)", "dq = dq"),                                # R-step dq lost
    ("dh = dS.sum(axis=1).T", "dh = dS.sum(axis=2).T"),                                  # wrong axis
])
def test_planted_backward_mistakes_are_caught(monkeypatch, old, new):
    monkeypatch.setattr(om, "monarch_head_backward", _mutant(old, new))
    assert not _fd_ok()


def test_entropy_plus_one_cancels_in_softmax_backward(monkeypatch):
    """A row-constant shift of dR leaves dSr unchanged, so the '+1' of the
    entropy derivative has no effect on any gradient."""
    monkeypatch.setattr(om, "monarch_head_backward",
                        _mutant("- dh[..., None] * (np.log(R) + 1.0)", "- dh[..., None] * np.log(R)"))
    assert _fd_ok()


@pytest.mark.parametrize("g", [om.Grid(4, 6, 8, 2, 4), om.Grid(6, 4, 4, 2, 2, chunk_frames=2)],
                         ids=["bidirectional", "chunk_causal"])
def test_gradient_invariants_of_a_row_stochastic_operator(g):
    """Rows of M sum to 1, so sum_tokens dv = sum_tokens dy; one shift of every
    key leaves R and every visible row of L unchanged, so sum_tokens dk = 0."""
    q, k, v, dy = _inputs(g, 16, seed=11)
    dq, dk, dv = om.monarch_attention_backward(q, k, v, dy, g)
    assert np.allclose(dv.sum(axis=2), dy.sum(axis=2), rtol=0, atol=1e-10)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-10 * np.abs(dk).sum(axis=2).max()
    assert np.isfinite(dq).all()
