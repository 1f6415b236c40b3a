"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each of them.  This is evidence that the pins constrain every term of
the oracle, not only that the oracle passes them."""

import math

import numpy as np
import pytest

from oracle import monarch as om
from tests.test_oracle_pins import (_objective_setup, _perturb, _rand, _separable)


def _separable_is_dense(iters=2):
    g = om.Grid(4, 8, 8, 4, 4)
    q, k, v = _separable(1, 1, g, 16, seed=11)
    out = om.monarch_attention(q, k, v, g, iters)
    return np.abs(out - om.dense_attention(q, k, v)).max() < 1e-10


def _r_is_maximiser():
    g, scale, qb, kb = _objective_setup()
    rng = np.random.default_rng(0)
    st1 = om.monarch_head(qb, kb, kb, g, 1, scale)
    qt = om._column_qtilde(st1.L, qb)
    R2, _ = om._r_step(qt, kb, scale)
    F = om.head_objective(st1.L, R2, qb, kb, scale)
    return all(om.head_objective(st1.L, _perturb(R2, rng, 1e-3), qb, kb, scale) <= F + 1e-12
               for _ in range(40))


def _one_position_is_dense():
    g = om.Grid(2, 3, 4, 1, 1)
    q, k, v = (_rand((1, 1, g.Nq, 8), s) for s in (21, 22, 23))
    return np.abs(om.monarch_attention(q, k, v, g, 2) - om.dense_attention(q, k, v)).max() < 1e-12


def _kv_separable_is_dense():
    g = om.Grid(2, 4, 6, 2, 3, Tk=5)
    q, k, v = _separable(1, 1, g, 16, seed=11)
    out = om.monarch_attention(q, k, v, g, 1)
    return np.abs(out - om.dense_attention(q, k, v)).max() < 1e-10


def test_unmutated_oracle_passes_every_check():
    assert _separable_is_dense() and _r_is_maximiser() and _one_position_is_dense()
    assert _kv_separable_is_dense()


def test_dropped_entropy_bias_is_caught(monkeypatch):
    orig = om._r_step
    monkeypatch.setattr(om, "_r_step", lambda qt, kb, s: (orig(qt, kb, s)[0], 0 * orig(qt, kb, s)[1]))
    assert not _separable_is_dense()


def test_flipped_entropy_sign_is_caught(monkeypatch):
    orig = om._r_step
    monkeypatch.setattr(om, "_r_step", lambda qt, kb, s: (orig(qt, kb, s)[0], -orig(qt, kb, s)[1]))
    assert not _separable_is_dense()


def test_missing_beta_normalisation_is_caught(monkeypatch):
    def no_beta(L, qb):
        num = np.matmul(np.swapaxes(L, 1, 2), np.swapaxes(qb, 0, 1))
        return np.swapaxes(num, 0, 1)
    monkeypatch.setattr(om, "_column_qtilde", no_beta)
    assert not (_separable_is_dense(2) and _r_is_maximiser())


def test_L_instead_of_L_transpose_is_caught(monkeypatch):
    def untransposed(L, qb):
        beta = L.sum(axis=2)
        num = np.matmul(L, np.swapaxes(qb, 0, 1))
        return np.swapaxes(num / beta[:, :, None], 0, 1)
    monkeypatch.setattr(om, "_column_qtilde", untransposed)
    assert not _r_is_maximiser()


def test_wrong_score_scale_is_caught(monkeypatch):
    orig = om._l_step
    monkeypatch.setattr(om, "_l_step", lambda qb, kt, h, s, vis=None: orig(qb, kt, h, s * 1.01, vis))
    assert not _one_position_is_dense()


def test_wrong_kv_alignment_is_caught(monkeypatch):
    orig = om.initial_qtilde

    def shifted(qb, grid):
        qt = orig(qb, grid)
        return np.roll(qt, 1, axis=0) if grid.Tkey != grid.T else qt
    monkeypatch.setattr(om, "initial_qtilde", shifted)
    # separability makes one step exact from any init, so the alignment is
    # pinned by the eps-limit test instead:
    from tests.test_oracle_pins import test_kv_initialisation_is_the_eps_limit
    with pytest.raises(AssertionError):
        test_kv_initialisation_is_the_eps_limit()


def test_wrong_position_index_is_caught(monkeypatch):
    orig = om.block_index

    def reversed_positions(frames, H, W, th, tw):
        return orig(frames, H, W, th, tw)[:, ::-1].copy()
    monkeypatch.setattr(om, "block_index", reversed_positions)
    from tests.test_oracle_pins import test_block_index_matches_hand_table
    with pytest.raises(AssertionError):
        test_block_index_matches_hand_table()


def _masked_separable_is_dense():
    from tests.test_oracle_pins import _masked_dense
    g = om.Grid(6, 4, 4, 2, 2, chunk_frames=2)
    q, k, v = _separable(1, 1, g, 16, seed=13)
    out = om.monarch_attention(q, k, v, g, 1)
    return np.abs(out - _masked_dense(q, k, v, g)).max() < 1e-10


def test_unmutated_mask_passes():
    assert _masked_separable_is_dense()


def test_mask_that_hides_the_own_chunk_is_caught(monkeypatch):
    # strict '<' instead of '<=' between chunk indices (own chunk invisible
    # except through the tile itself, which D3 needs)
    def strict(self):
        P = self.tiles_per_frame
        vis = np.ones((self.b1q, self.b1k), dtype=bool)
        for a1 in range(self.b1q):
            for c1 in range(self.b1k):
                vis[a1, c1] = (c1 // P) // self.chunk_frames < (a1 // P) // self.chunk_frames or c1 == a1
        return vis
    monkeypatch.setattr(om.Grid, "visible", strict)
    assert not _masked_separable_is_dense()


def test_mask_over_tiles_instead_of_frames_is_caught(monkeypatch):
    # chunk index taken from the tile index instead of its frame
    def by_tile(self):
        vis = np.ones((self.b1q, self.b1k), dtype=bool)
        for a1 in range(self.b1q):
            for c1 in range(self.b1k):
                vis[a1, c1] = c1 // self.chunk_frames <= a1 // self.chunk_frames
        return vis
    monkeypatch.setattr(om.Grid, "visible", by_tile)
    assert not _masked_separable_is_dense()


def test_mask_ignored_by_the_l_step_is_caught(monkeypatch):
    orig = om._l_step
    monkeypatch.setattr(om, "_l_step", lambda qb, kt, h, s, vis=None: orig(qb, kt, h, s, None))
    assert not _masked_separable_is_dense()
