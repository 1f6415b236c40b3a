"""Seeded synthetic inputs for Monarch video attention.

This module only synthesises inputs; it holds none of the attention
arithmetic.  Tests, the benchmark and the oracle checks all draw their
q, k, v from here, so the CUDA path and the oracle consume the same values.

Recipe (one ``numpy.random.default_rng(seed)`` per workload, fp64 draws):
  1. noise:   for each (b, h) in order, Q[b,h] ~ N(0,1) of shape [Nq, d];
              then K[b,h] [Nk, d]; then V[b,h] [Nk, d].
  2. planted: (kinds with planted pairs) for each (b, h): 64 query tokens
              and 64 key tokens drawn uniformly, then 64 directions
              u ~ N(0, I_d) normalised; q[i] += a*u and k[j] += a*u with
              a = sqrt(8*sqrt(d)), which raises that pair's scaled logit by
              about +8 (a sparse long-range semantic match).
  3. positional: (all kinds but "iid"/"separable") Q and K gain the same
              sinusoidal (t, y, x) code with weight 1.0: d is split into
              groups (g_t, g_y, g_x) = (44, 42, 42) for d=128, (22, 22, 20)
              for d=64; in a group of size g the features (2j, 2j+1) are
              sin(c*w_j), cos(c*w_j) of the axis coordinate c with
              w_j = 10000^(-2j/g).  For a KV cache the query frames carry their
              absolute frame index (the last T of the Tk key frames).
  4. round:   the fp64 values are rounded once to the workload dtype; both
              sides consume the rounded values.

The mix (periodic positional structure + sparse semantic pairs + dense
noise) mirrors the attention structure MonarchRT describes for video DiTs:
A = D + S + eps, a separable periodic positional part, a sparse semantic
part and a residual (gist.science explainer §2.A "Structural Analysis").

"separable" draws q = [qA(token) | qB(y mod th, x mod tw)] and
k = [kA(t, y div th, x div tw) | kB(token)] (halves of d), so that the scores
split into a part constant inside a key tile plus a part that depends only on
the in-tile positions -- the case in which the Monarch form is exact.
"""

from __future__ import annotations

from dataclasses import dataclass, field, asdict

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    T: int
    H: int
    W: int
    d: int
    th: int
    tw: int
    iters: int
    dtype: str
    seed: int
    kind: str  # "iid" | "separable" | "pos" | "pos_planted"
    Tk: int = 0  # key frames; 0 means T (self-attention)
    planted: int = 64
    chunk_frames: int = 0  # frame-chunk causal mask of whole-sequence training; 0 = bidirectional

    @property
    def Tkey(self) -> int:
        return self.Tk or self.T

    @property
    def Nq(self) -> int:
        return self.T * self.H * self.W

    @property
    def Nk(self) -> int:
        return self.Tkey * self.H * self.W

    @property
    def kv_len(self) -> int:
        return self.Nk

    def to_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("toy_256_f32", 1, 2, 4, 8, 8, 64, 4, 4, 1, "f32", 0, "iid"),
        Workload("toy_256_f32_separable", 1, 2, 4, 8, 8, 64, 4, 4, 1, "f32", 1, "separable"),
        Workload("chunk_4680_bf16", 1, 12, 3, 30, 52, 128, 6, 4, 2, "bf16", 2, "pos"),
        Workload("kvcache_4680x32760_bf16", 1, 12, 3, 30, 52, 128, 6, 4, 2, "bf16", 3, "pos", Tk=21),
        Workload("full_32760_bf16", 2, 12, 21, 30, 52, 128, 6, 4, 3, "bf16", 4, "pos_planted"),
        # the same sequence in the training regime: 3-frame chunks, chunk-causal
        Workload("train_32760_bf16_causal", 2, 12, 21, 30, 52, 128, 6, 4, 3, "bf16", 4, "pos_planted",
                 chunk_frames=3),
        # the one-step regime of finetuned models (a single refinement step)
        Workload("chunk_4680_bf16_1step", 1, 12, 3, 30, 52, 128, 6, 4, 1, "bf16", 2, "pos"),
        Workload("full_32760_bf16_1step", 2, 12, 21, 30, 52, 128, 6, 4, 1, "bf16", 4, "pos_planted"),
        Workload("sweep_2048_f16", 1, 24, 8, 16, 16, 64, 8, 8, 2, "f16", 5, "pos_planted"),
        Workload("sweep_8192_f16", 1, 24, 8, 32, 32, 64, 8, 8, 2, "f16", 5, "pos_planted"),
        Workload("sweep_32768_f16", 1, 24, 8, 64, 64, 64, 8, 8, 2, "f16", 5, "pos_planted"),
    ]
}


def _groups(d: int):
    if d == 128:
        return (44, 42, 42)
    if d == 64:
        return (22, 22, 20)
    g = 2 * (d // 6)
    return (d - 2 * g, g, g)


def positional_code(frames: np.ndarray, H: int, W: int, d: int) -> np.ndarray:
    """[len(frames)*H*W, d] sinusoidal code of (t, y, x) in grid order."""
    gt, gy, gx = _groups(d)
    t = np.repeat(np.asarray(frames, dtype=np.float64), H * W)
    y = np.tile(np.repeat(np.arange(H, dtype=np.float64), W), len(frames))
    x = np.tile(np.arange(W, dtype=np.float64), len(frames) * H)
    cols = []
    for c, g in ((t, gt), (y, gy), (x, gx)):
        j = np.arange(g // 2, dtype=np.float64)
        w = 10000.0 ** (-2.0 * j / g)
        ang = c[:, None] * w[None, :]
        blk = np.empty((c.shape[0], g))
        blk[:, 0::2] = np.sin(ang)
        blk[:, 1::2] = np.cos(ang)
        cols.append(blk)
    return np.concatenate(cols, axis=1)


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(x).to(DTYPES[dtype])


def make_inputs(w: Workload):
    """Returns (q, k, v) as CPU torch tensors in the workload dtype, shapes
    [B, heads, Nq, d] and [B, heads, Nk, d], tokens in grid order (t, y, x)."""
    rng = np.random.default_rng(w.seed)
    B, Hh, d = w.B, w.heads, w.d
    tdt = DTYPES[w.dtype]
    q = torch.empty((B, Hh, w.Nq, d), dtype=tdt)
    k = torch.empty((B, Hh, w.Nk, d), dtype=tdt)
    v = torch.empty((B, Hh, w.Nk, d), dtype=tdt)

    if w.kind == "separable":
        for b in range(B):
            for h in range(Hh):
                half = d // 2
                nty, ntx = w.H // w.th, w.W // w.tw
                qa = rng.standard_normal((w.T, w.H, w.W, half))
                qb = rng.standard_normal((w.th, w.tw, half))
                ka = rng.standard_normal((w.Tkey, nty, ntx, half))
                kb = rng.standard_normal((w.Tkey, w.H, w.W, half))
                vv = rng.standard_normal((w.Nk, d))
                ys, xs = np.arange(w.H), np.arange(w.W)
                qb_full = qb[ys % w.th][:, xs % w.tw]  # [H, W, half]
                ka_full = ka[:, ys // w.th][:, :, xs // w.tw]  # [Tk, H, W, half]
                qq = np.concatenate([qa, np.broadcast_to(qb_full, qa.shape)], axis=-1)
                kk = np.concatenate([ka_full, kb], axis=-1)
                q[b, h] = _round(qq.reshape(w.Nq, d), w.dtype)
                k[b, h] = _round(kk.reshape(w.Nk, d), w.dtype)
                v[b, h] = _round(vv, w.dtype)
        return q, k, v

    noise_q = [[rng.standard_normal((w.Nq, d)) for h in range(Hh)] for b in range(B)]
    noise_k = [[rng.standard_normal((w.Nk, d)) for h in range(Hh)] for b in range(B)]
    for b in range(B):
        for h in range(Hh):
            v[b, h] = _round(rng.standard_normal((w.Nk, d)), w.dtype)
    if w.kind in ("pos", "pos_planted"):
        pos_k = positional_code(np.arange(w.Tkey), w.H, w.W, d)
        pos_q = pos_k[(w.Tkey - w.T) * w.H * w.W:]
    for b in range(B):
        for h in range(Hh):
            qq, kk = noise_q[b][h], noise_k[b][h]
            if w.kind == "pos_planted":
                qi = rng.integers(0, w.Nq, size=w.planted)
                kj = rng.integers(0, w.Nk, size=w.planted)
                u = rng.standard_normal((w.planted, d))
                u /= np.linalg.norm(u, axis=1, keepdims=True)
                a = np.sqrt(8.0 * np.sqrt(d))
                np.add.at(qq, qi, a * u)
                np.add.at(kk, kj, a * u)
            if w.kind in ("pos", "pos_planted"):
                qq = qq + pos_q
                kk = kk + pos_k
            q[b, h] = _round(qq, w.dtype)
            k[b, h] = _round(kk, w.dtype)
            noise_q[b][h] = noise_k[b][h] = None
    return q, k, v


def make_cotangent(w: Workload, dtype: str = "f32"):
    """Seeded output gradient dy for the backward: [B, heads, Nq, d] standard
    normal entries rounded to `dtype` (CPU torch tensor)."""
    rng = np.random.default_rng(w.seed + 1_000_003)
    dy = torch.empty((w.B, w.heads, w.Nq, w.d), dtype=DTYPES[dtype])
    for b in range(w.B):
        for h in range(w.heads):
            dy[b, h] = _round(rng.standard_normal((w.Nq, w.d)), dtype)
    return dy
