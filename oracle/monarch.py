"""Plain fp64 CPU oracle for Monarch-factorised video attention (forward).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it.  It shares no code with the CUDA library
and imports nothing from the product package.

What it computes
----------------
MonarchRT (arXiv 2602.12271, "MonarchRT: Efficient Attention for Real-Time
Video Generation") replaces dense 3D self-attention softmax(S)V over a
T x H x W token grid by an attention matrix constrained to Monarch form,
M = P blockdiag(L) P^T blockdiag(R) (abstract; gist.science explainer §2
"Methodology: MonarchRT"), with blocks aligned to the video grid (§2.A
"Block Alignment") and tiled inside a frame (§2.B "Tiled Monarch
Parameterization").  L and R come from the alternating refinement of the
original MonarchAttention algorithm (§2.C "Finetuning and Efficient
Implementation": "iterative refinement", one step after finetuning).  The
pages give no equations; the reading implemented here is:

  grid -> blocks  token (t, y, x) of a frame grid with tiles th x tw maps to
                  tile  c1 = (t*(H/th) + y//th)*(W/tw) + x//tw   (block axis 1)
                  pos   c2 = (y % th)*tw + x % tw                (block axis 2)
  D1  M[(a1,a2),(c1,c2)] = L_{a2}[a1,c1] * R_{c1}[a2,c2]
  D2  scores S = s * q.k, s = 1/sqrt(d)
  D3  initial L: block identity (self-attention); for a KV cache with
      key frames Tk > query frames T, the eps -> 0 limit of
      (1-eps)[c1 == a1 + (Tk-T)P] + eps/|visible(a1)|
  D4  R step:  beta = sum_a1 L,  q~ = (sum_a1 L q)/beta,
               R_{c1}[a2,:] = softmax_c2(s q~[c1,a2].k[c1,c2])
  D5  h[c1,a2] = -sum_c2 R log R
  D6  L step:  k~ = sum_c2 R k,
               L_{a2}[a1,:] = softmax_c1(s q[a1,a2].k~[c1,a2] + h[c1,a2])
  D7  one iteration = one R step then one L step
  D8  output:  z = sum_c2 R v,  y = sum_c1 L z,  out = y scattered back to
               the grid order
  D9  frame-chunk causal mask (autoregressive training over the whole
      sequence, chunks of C frames; gist.science explainer §1 "auto-regressive
      generation"): query tile a1 sees key tile c1 iff
      frame(c1) // C <= frame(a1) // C, frames counted on the key axis.  The
      mask restricts the support of L (D6's softmax runs over visible c1 only,
      D4's sums over the a1 that see c1); R works inside a tile, one frame, so
      it is unchanged, and the block identity of D3 stays feasible.

D4 and D6 are the exact block maximisers of the variational softmax
objective F(M) = sum_rows <M_row, S_row> + H(M_row) (whose unconstrained
maximiser over row-stochastic M is softmax(S)); this is what the tests pin.

Everything here is fp64 numpy; ``np.matmul`` is the only library primitive
used as a step.  Loops run over (batch, head) so memory stays one head deep.

How it is pinned (tests/test_oracle_pins.py, test_oracle_properties.py,
test_oracle_mutations.py, test_oracle_backward.py): the grid -> block map
against a hand-written table; the factored output against M materialised
entry by entry from token coordinates (non-negative, row-stochastic, zero
outside the mask), on fixed and on randomly drawn tiny grids; separable
scores and the one-position or one-tile grids against dense softmax
attention; each block update against random feasible perturbations of F; the
backward against central finite differences of the forward and two exact
invariants.  For generic inputs no printed value exists, so the output values
are pinned through these properties only, not against a worked example.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Grid:
    """Token grid and tiling.  T query frames, Tk key frames (Tk == T is
    self-attention), frame H x W, spatial tile th x tw."""

    T: int
    H: int
    W: int
    th: int
    tw: int
    Tk: int | None = None
    chunk_frames: int = 0  # frames per causal chunk (D9); 0 = every key visible

    @property
    def Tkey(self) -> int:
        return self.T if self.Tk is None else self.Tk

    @property
    def tiles_per_frame(self) -> int:
        return (self.H // self.th) * (self.W // self.tw)

    @property
    def b2(self) -> int:
        return self.th * self.tw

    @property
    def b1q(self) -> int:
        return self.T * self.tiles_per_frame

    @property
    def b1k(self) -> int:
        return self.Tkey * self.tiles_per_frame

    @property
    def Nq(self) -> int:
        return self.T * self.H * self.W

    @property
    def Nk(self) -> int:
        return self.Tkey * self.H * self.W

    def check(self) -> None:
        if self.H % self.th or self.W % self.tw:
            raise ValueError("tile must divide the frame")
        if self.Tkey < self.T:
            raise ValueError("key frames must include the query chunk")
        if self.chunk_frames < 0:
            raise ValueError("chunk_frames must be >= 0")

    def visible(self) -> np.ndarray:
        """[b1q, b1k] bool: key tile c1 visible to query tile a1 (D9).  The
        query chunk is the last T frames of the key sequence."""
        P = self.tiles_per_frame
        vis = np.ones((self.b1q, self.b1k), dtype=bool)
        if self.chunk_frames:
            C = self.chunk_frames
            for a1 in range(self.b1q):
                tq = self.Tkey - self.T + a1 // P
                for c1 in range(self.b1k):
                    vis[a1, c1] = (c1 // P) // C <= tq // C
        return vis


def block_index(frames: int, H: int, W: int, th: int, tw: int) -> np.ndarray:
    """idx[c1, c2] = grid token index n = (t*H + y)*W + x of tile c1,
    position c2 (block alignment, gist.science explainer §2.A; tiling §2.B).

    Written as an explicit loop over grid tokens so it reads like the
    definition of the map."""
    nty, ntx = H // th, W // tw
    P = nty * ntx
    idx = np.empty((frames * P, th * tw), dtype=np.int64)
    for t in range(frames):
        for y in range(H):
            for x in range(W):
                c1 = (t * nty + y // th) * ntx + x // tw
                c2 = (y % th) * tw + x % tw
                idx[c1, c2] = (t * H + y) * W + x
    return idx


def _softmax_last(x: np.ndarray) -> np.ndarray:
    m = x.max(axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=-1, keepdims=True)


def _logsumexp_last(x: np.ndarray) -> np.ndarray:
    m = x.max(axis=-1)
    return m + np.log(np.exp(x - m[..., None]).sum(axis=-1))


def initial_qtilde(qb: np.ndarray, grid: Grid) -> np.ndarray:
    """q~ of the first R step (D3 + D4) for one head.

    qb: [b1q, b2, d] queries in block order.  Returns [b1k, b2, d].

    Self-attention: L0 is the block identity, so beta = 1 and q~[c1] = q[c1].
    KV cache (Tk > T): the query chunk is the last T frames of the key
    sequence, so query tile a1 is aligned with key tile a1 + (Tk-T)P.  With
    L0 = (1-eps)*aligned + eps*uniform-over-visible, an aligned key tile gets
    its own query tile as eps -> 0, and an earlier (cached) key tile gets the
    mean of q over the query tiles that see it, weighted by 1/|visible(a1)|.
    Every cached frame precedes the query chunk, so every query tile sees
    every key tile and the weights are uniform.  (The pages describe the
    KV-cache regime -- autoregressive chunks attending to cached frames,
    gist.science explainer §1 and §4 -- but not this initialisation.)
    """
    b1q, b2, d = qb.shape
    if grid.Tkey == grid.T:
        return qb.copy()
    off = (grid.Tkey - grid.T) * grid.tiles_per_frame
    b1k = grid.b1k
    visible = grid.visible()  # without a mask the query chunk sees all keys
    w = 1.0 / visible.sum(axis=1)  # 1/|visible(a1)|
    qt = np.empty((b1k, b2, d))
    for c1 in range(b1k):
        if c1 >= off:
            qt[c1] = qb[c1 - off]
        else:
            wa = w * visible[:, c1]
            qt[c1] = np.einsum("a,apd->pd", wa, qb) / wa.sum()
    return qt


@dataclass
class HeadState:
    """Factors and intermediates of one head after the last iteration."""

    qt: np.ndarray  # [b1k, b2, d]   q~ used by the last R step
    R: np.ndarray  # [b1k, b2, b2]  R_{c1}[a2, c2]
    h: np.ndarray  # [b1k, b2]      entropy of R_{c1}[a2, :]
    kt: np.ndarray  # [b1k, b2, d]   k~[c1, a2]
    L: np.ndarray  # [b2, b1q, b1k] L_{a2}[a1, c1]
    lse: np.ndarray  # [b2, b1q]     log-sum-exp of the last L step's rows
    z: np.ndarray  # [b1k, b2, d]   z[c1, a2] = sum_c2 R v
    y: np.ndarray  # [b1q, b2, d]   output in block order
    objective: list  # F(M) after every iteration


def _r_step(qt: np.ndarray, kb: np.ndarray, scale: float):
    """D4 + D5 for one head: qt, kb [b1k, b2, d] -> R [b1k, b2, b2], h [b1k, b2]."""
    s_r = scale * np.matmul(qt, np.swapaxes(kb, 1, 2))  # [c1, a2, c2]
    R = _softmax_last(s_r)
    h = -(R * np.log(R)).sum(axis=-1)
    return R, h


def _l_step(qb: np.ndarray, kt: np.ndarray, h: np.ndarray, scale: float, visible=None):
    """D6 for one head: qb [b1q,b2,d], kt [b1k,b2,d], h [b1k,b2] ->
    L [b2, b1q, b1k], lse [b2, b1q].  ``visible`` [b1q, b1k] (D9) restricts
    the softmax to the visible key tiles."""
    qp = np.swapaxes(qb, 0, 1)  # [a2, a1, d]
    kp = np.swapaxes(kt, 0, 1)  # [a2, c1, d]
    s_l = scale * np.matmul(qp, np.swapaxes(kp, 1, 2)) + h.T[:, None, :]
    if visible is not None:
        s_l = np.where(visible[None, :, :], s_l, -np.inf)
    return _softmax_last(s_l), _logsumexp_last(s_l)


def _column_qtilde(L: np.ndarray, qb: np.ndarray) -> np.ndarray:
    """D4's aggregation for one head: q~[c1,a2] = sum_a1 L q / sum_a1 L."""
    beta = L.sum(axis=1)  # [a2, c1]
    num = np.matmul(np.swapaxes(L, 1, 2), np.swapaxes(qb, 0, 1))  # [a2, c1, d]
    return np.swapaxes(num / beta[:, :, None], 0, 1)  # [c1, a2, d]


def head_objective(L, R, qb, kb, scale) -> float:
    """F(M) = sum_rows <M, S> + H(M) for the Monarch M of one head, written
    through the factors: M[(a1,a2),(c1,c2)] = L_{a2}[a1,c1] R_{c1}[a2,c2]."""
    S = scale * np.einsum("apd,cjd->apcj", qb, kb)
    M = np.einsum("pac,cpj->apcj", L, R)
    with np.errstate(divide="ignore", invalid="ignore"):
        ent = np.where(M > 0, -M * np.log(M), 0.0)
    return float((M * S).sum() + ent.sum())


def monarch_head(qb, kb, vb, grid: Grid, iters: int, scale: float,
                 track_objective: bool = False) -> HeadState:
    """One (batch, head): qb [b1q,b2,d], kb/vb [b1k,b2,d] in block order."""
    if iters < 1:
        raise ValueError("iters must be >= 1")
    qt = initial_qtilde(qb, grid)
    vis = grid.visible() if grid.chunk_frames else None
    obj = []
    L = None
    for it in range(iters):
        if it > 0:
            qt = _column_qtilde(L, qb)  # L of the previous iteration
        R, h = _r_step(qt, kb, scale)
        kt = np.matmul(R, kb)  # k~[c1, a2] = sum_c2 R k
        L, lse = _l_step(qb, kt, h, scale, vis)
        if track_objective:
            obj.append(head_objective(L, R, qb, kb, scale))
    z = np.matmul(R, vb)  # [c1, a2, d]
    y = np.swapaxes(np.matmul(L, np.swapaxes(z, 0, 1)), 0, 1)  # [a1, a2, d]
    return HeadState(qt=qt, R=R, h=h, kt=kt, L=L, lse=lse, z=z, y=y,
                     objective=obj)


def monarch_attention(q, k, v, grid: Grid, iters: int, scale: float | None = None,
                      heads=None, return_states: bool = False):
    """Monarch attention forward.

    q: [B, Hh, Nq, d]; k, v: [B, Hh, Nk, d], tokens in grid order (t, y, x).
    Returns out [B, Hh, Nq, d] (fp64).  ``heads`` optionally restricts the
    computation to a list of (b, h) pairs (other rows of ``out`` stay NaN);
    heads are independent, so a subset is an exact sample.
    """
    grid.check()
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hh, Nq, d = q.shape
    assert Nq == grid.Nq and k.shape[2] == grid.Nk and v.shape[2] == grid.Nk
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    iq = block_index(grid.T, grid.H, grid.W, grid.th, grid.tw)
    ik = block_index(grid.Tkey, grid.H, grid.W, grid.th, grid.tw)
    out = np.full(q.shape, np.nan)
    states = {}
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hh)]
    for b, h in todo:
        st = monarch_head(q[b, h][iq], k[b, h][ik], v[b, h][ik], grid, iters, scale)
        out[b, h][iq] = st.y
        if return_states:
            states[(b, h)] = st
    return (out, states) if return_states else out


def monarch_head_backward(qb, kb, vb, dyb, grid: Grid, scale: float):
    """Gradients of one head's output for iters = 1 (the one-step regime of
    finetuned models, gist.science explainer §2.C), self-attention.

    The forward is D4-D6 + D8 with q~ = q (D3: block identity), optionally
    under the D9 mask.  The chain rule, step by step (all per head, block order):
      L step (per position a2):  y = L z, L = softmax_c1(s q.k~ + h)
        dz = L^T dy;  dL = dy z^T;  dS = L * (dL - rowsum(L * dL))
        dq += s dS k~;  dk~ = s dS^T q;  dh = colsum(dS)
      R step (per tile c1):  k~ = R k, z = R v, h = -sum R log R,
                             R = softmax_c2(s q.k)
        dR = dk~ k^T + dz v^T - dh (log R + 1)
        dk = R^T dk~ + s dSr^T q;  dv = R^T dz;  dq += s dSr k,
        with dSr = R * (dR - rowsum(R * dR)).
    qb, kb, vb, dyb: [b1, b2, d] in block order -> dq, dk, dv [b1, b2, d]."""
    if grid.Tkey != grid.T:
        raise NotImplementedError("the backward covers self-attention")
    vis = grid.visible() if grid.chunk_frames else None
    # forward quantities
    R, h = _r_step(qb, kb, scale)                   # [c1, a2, c2], [c1, a2]
    kt = np.matmul(R, kb)                           # [c1, a2, d]
    z = np.matmul(R, vb)
    L, _ = _l_step(qb, kt, h, scale, vis)           # [a2, a1, c1]
    sw = lambda x: np.swapaxes(x, 0, 1)
    # L step backward, positions a2 as the batch axis
    dy_p, z_p, q_p, kt_p = sw(dyb), sw(z), sw(qb), sw(kt)
    dz_p = np.matmul(np.swapaxes(L, 1, 2), dy_p)    # [a2, c1, d]
    dL = np.matmul(dy_p, np.swapaxes(z_p, 1, 2))    # [a2, a1, c1]
    dS = L * (dL - (L * dL).sum(axis=-1, keepdims=True))
    dq_p = scale * np.matmul(dS, kt_p)              # [a2, a1, d]
    dkt_p = scale * np.matmul(np.swapaxes(dS, 1, 2), q_p)
    dh = dS.sum(axis=1).T                           # [c1, a2]
    dz, dkt, dq = sw(dz_p), sw(dkt_p), sw(dq_p)
    # R step backward, tiles c1 as the batch axis
    dR = (np.matmul(dkt, np.swapaxes(kb, 1, 2)) + np.matmul(dz, np.swapaxes(vb, 1, 2))
          - dh[..., None] * (np.log(R) + 1.0))      # [c1, a2, c2]
    dSr = R * (dR - (R * dR).sum(axis=-1, keepdims=True))
    dk = np.matmul(np.swapaxes(R, 1, 2), dkt) + scale * np.matmul(np.swapaxes(dSr, 1, 2), qb)
    dv = np.matmul(np.swapaxes(R, 1, 2), dz)
    dq = dq + scale * np.matmul(dSr, kb)
    return dq, dk, dv


def monarch_attention_backward(q, k, v, dy, grid: Grid, scale: float | None = None, heads=None):
    """Gradients (dq, dk, dv) of sum(dy * monarch_attention(q, k, v, grid, 1)).
    Tensors [B, Hh, N, d] in grid order; fp64.  ``heads`` as in
    monarch_attention (other heads stay NaN)."""
    grid.check()
    q, k, v, dy = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dy))
    B, Hh, N, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx = block_index(grid.T, grid.H, grid.W, grid.th, grid.tw)
    dq, dk, dv = (np.full(q.shape, np.nan) for _ in range(3))
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(Hh)]):
        gq, gk, gv = monarch_head_backward(q[b, h][idx], k[b, h][idx], v[b, h][idx], dy[b, h][idx], grid, scale)
        dq[b, h][idx], dk[b, h][idx], dv[b, h][idx] = gq, gk, gv
    return dq, dk, dv


def dense_attention(q, k, v, scale: float | None = None, mask=None):
    """Textbook softmax(s q k^T) v per (batch, head), fp64.  ``mask``
    [Nq, Nk] bool keeps only the allowed keys of each query."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = scale * np.matmul(q, np.swapaxes(k, -1, -2))
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    return np.matmul(_softmax_last(s), v)


def frame_chunk_mask(T: int, Tk: int, H: int, W: int, chunk_frames: int) -> np.ndarray:
    """Token-level [Nq, Nk] mask of D9: query token of (absolute) frame tq
    sees key token of frame tk iff tk // C <= tq // C."""
    hw = H * W
    tq = (Tk - T) + np.arange(T * hw) // hw
    tk = np.arange(Tk * hw) // hw
    return (tk[None, :] // chunk_frames) <= (tq[:, None] // chunk_frames)


def monarch_flops(grid: Grid, d: int, iters: int, B: int = 1, heads: int = 1) -> float:
    """Algorithmic FLOPs of one forward: 2*iters*F_L + (2*iters+1)*F_R per head,
    F_L = 2*b2*b1q*b1k*d (one L-sized contraction), F_R = 2*b1k*b2^2*d."""
    FL = 2.0 * grid.b2 * grid.b1q * grid.b1k * d
    FR = 2.0 * grid.b1k * grid.b2 * grid.b2 * d
    return B * heads * (2 * iters * FL + (2 * iters + 1) * FR)


def dense_flops(grid: Grid, d: int, B: int = 1, heads: int = 1) -> float:
    """FLOPs of dense attention on the same shape: 4*Nq*Nk*d per head."""
    return 4.0 * B * heads * grid.Nq * grid.Nk * d
