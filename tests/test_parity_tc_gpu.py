"""GPU checks of the tensor-core path's own pieces, below the final output:

* the grid -> block permutation on the load side, bit for bit: the first R
  step writes the queries in block-major order (the f16 copy the L step
  reads), which must equal q[b, h][block_index] converted to f16;
* a permutation probe through the whole call: inputs built so that R and L
  are both the identity (one-hot to within 2^-100), for which the exact
  output is out = v of the query's own token; a misplaced tile or position
  anywhere in the load permutation, the factor bookkeeping or the inverse
  permutation of the store would put another token's value there;
* the intermediates of the last iteration (k~, z, q~ and h as the tensor-core
  kernels store them: f16 hi/lo planes, input-type hi/lo planes, base-2
  entropy) against the oracle's HeadState.

Block order, positions and the tile map follow the MonarchRT explainers
(gist.science §2.A "Block Alignment", §2.B "Tiled Monarch
Parameterization"); the oracle's block_index is pinned to a hand-written
table on the CPU."""

import math

import numpy as np
import pytest
import torch

import structured_sparse_attention_grid_b200 as m
from oracle import monarch as om
from structured_sparse_attention_grid_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

CODE = {"f32": m.MONARCH_F32, "bf16": m.MONARCH_BF16, "f16": m.MONARCH_F16}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _custom(dtype, T, H, W, d, th, tw, iters, Tk=0, B=2, heads=3, kind="pos_planted", seed=11, C=0):
    return Workload(f"tc_{dtype}_{T}x{H}x{W}_d{d}_{th}x{tw}_it{iters}_Tk{Tk}_C{C}", B, heads, T, H, W, d,
                    th, tw, iters, dtype, seed, kind, Tk=Tk, planted=8, chunk_frames=C)


def _run_ws(w, q, k, v):
    """One forward through monarch_attn_fwd_ws with a zeroed workspace; returns
    the f32 output and the workspace (uint8) with its region offsets."""
    total, offs = m.workspace_layout(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw, w.iters, w.Nk, CODE[w.dtype])
    ws = torch.zeros(total, dtype=torch.uint8, device="cuda")
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty(qd.shape, dtype=torch.float32, device="cuda")
    m.device_error(reset=True)
    m.monarch_attn_fwd_ws(qd, kd, vd, out, ws, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert m.device_error(reset=True) == 0
    return out, ws, offs


def _region(ws, off, numel, dtype):
    nbytes = numel * torch.empty(0, dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype)


# ---------------------------------------------------------------------------
# load permutation: the block-major f16 copy of q, bit for bit

BLOCK_MAJOR = [
    WORKLOADS["chunk_4680_bf16"],
    WORKLOADS["kvcache_4680x32760_bf16"],
    _custom("f16", 2, 9, 10, 64, 3, 5, 2),           # 15 positions per tile (padded R-step rows)
    _custom("f16", 2, 12, 20, 128, 4, 4, 1, Tk=5),   # KV cache, f16: stored straight from the loaded rows
    _custom("bf16", 5, 12, 20, 128, 4, 4, 3),        # three iterations: the copy of the first step stays
]


@pytest.mark.parametrize("w", BLOCK_MAJOR, ids=[w.name for w in BLOCK_MAJOR])
def test_block_major_query_copy_is_bit_exact(w, cuda_lib):
    q, k, v = make_inputs(w)
    _, ws, offs = _run_ws(w, q, k, v)
    P = (w.H // w.th) * (w.W // w.tw)
    b2, b1q = w.th * w.tw, w.T * P
    got = _region(ws, offs[6], w.B * w.heads * b2 * b1q * w.d, torch.float16).view(w.B, w.heads, b2, b1q, w.d)
    idx = torch.from_numpy(om.block_index(w.T, w.H, w.W, w.th, w.tw))   # [b1q, b2] token of (tile, position)
    want = q.to(torch.float16)[:, :, idx.T.reshape(-1)].view(w.B, w.heads, b2, b1q, w.d)
    assert torch.equal(got.cpu().view(torch.int16), want.view(torch.int16))


# ---------------------------------------------------------------------------
# permutation probe through the whole call

ALPHA, BETA = 40.0, 64.0
MIN_GAP_BITS = 100.0   # every non-selected weight is below 2^-100 of the selected one


def _probe_inputs(w, seed=5):
    """k[token] = ALPHA e_{c2} + BETA f(c1): a one-hot code of the position c2
    in the first b2 channels and a random unit vector f of the key tile c1 in
    the others; queries are the keys of their aligned tile (the last T key
    frames).  Then, in base-2 logits, the R step sees s log2(e) ALPHA^2 between
    a query's own position and any other (the tile term is common to a tile
    and cancels), and the L step sees s log2(e) BETA^2 (1 - f(a).f(c)) between
    a query's own tile and any other: both >= MIN_GAP_BITS (checked on the
    rounded inputs), so R and L are the identity and out = v of the query's
    own token.  The KV mean query of a cached tile keeps the position code,
    and a chunk-causal mask keeps every aligned tile visible."""
    b2 = w.th * w.tw
    P = (w.H // w.th) * (w.W // w.tw)
    b1k = w.Tkey * P
    gen = torch.Generator().manual_seed(seed)
    f = torch.randn(w.B, w.heads, b1k, w.d - b2, generator=gen, dtype=torch.float64)
    f /= f.norm(dim=-1, keepdim=True)
    idx = torch.from_numpy(om.block_index(w.Tkey, w.H, w.W, w.th, w.tw))   # [b1k, b2]
    c1_of = torch.empty(w.Nk, dtype=torch.long)
    c2_of = torch.empty(w.Nk, dtype=torch.long)
    c1_of[idx.reshape(-1)] = torch.arange(b1k).repeat_interleave(b2)
    c2_of[idx.reshape(-1)] = torch.arange(b2).repeat(b1k)
    k = torch.zeros(w.B, w.heads, w.Nk, w.d, dtype=torch.float64)
    k[..., :b2] = ALPHA * torch.nn.functional.one_hot(c2_of, b2).to(torch.float64)
    k[..., b2:] = BETA * f[:, :, c1_of]
    k = k.to(TDT[w.dtype])
    q = k[:, :, w.Nk - w.Nq:].contiguous()
    v = torch.randn(w.B, w.heads, w.Nk, w.d, generator=gen, dtype=torch.float64).to(TDT[w.dtype])
    # the gaps, from the rounded tile codes
    s2 = math.log2(math.e) / math.sqrt(w.d)
    fr = k[:, :, idx[:, 0], b2:].double().cuda()                        # [B, heads, b1k, d - b2]
    gram = fr @ fr.transpose(-1, -2)
    own = gram.diagonal(dim1=-2, dim2=-1).clone()
    gram.diagonal(dim1=-2, dim2=-1).fill_(-math.inf)
    gap_l = float((s2 * (own - gram.amax(dim=-1))).min())
    gap_r = s2 * ALPHA * ALPHA
    assert gap_l >= MIN_GAP_BITS and gap_r >= MIN_GAP_BITS, (gap_l, gap_r)
    return q, k, v


PROBE = [
    WORKLOADS["chunk_4680_bf16"],
    WORKLOADS["kvcache_4680x32760_bf16"],
    WORKLOADS["full_32760_bf16"],
    WORKLOADS["train_32760_bf16_causal"],
    WORKLOADS["chunk_4680_bf16_1step"],
    _custom("bf16", 2, 9, 10, 128, 3, 5, 2),
    _custom("f16", 4, 16, 16, 64, 4, 4, 2, Tk=6),
    _custom("f32", 3, 8, 12, 128, 2, 4, 2),
    # small grids whose L step stacks positions (32 tiles: 4 a block; 64 tiles: 2)
    _custom("f16", 2, 16, 16, 64, 4, 4, 2),
    _custom("bf16", 4, 8, 8, 128, 2, 2, 2),
    _custom("bf16", 4, 8, 8, 128, 2, 2, 1),
]


@pytest.mark.parametrize("w", PROBE, ids=[w.name for w in PROBE])
def test_permutation_probe_returns_each_tokens_own_value(w, cuda_lib):
    q, k, v = _probe_inputs(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty(qd.shape, dtype=torch.float32, device="cuda")
    m.monarch_attn_fwd(qd, kd, vd, out, w.T, w.H, w.W, w.th, w.tw, w.iters, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    want = vd[:, :, w.Nk - w.Nq:].float()
    err = (out - want).abs()
    # rounding leaves a relative error near 1e-7; a value from any other token
    # differs by O(1) (v ~ N(0, 1))
    bad = err > 1e-5 * (1.0 + want.abs())
    assert not bool(bad.any()), f"{int(bad.sum())} outputs are not their own token's value (max err {float(err.max()):.3e})"


# ---------------------------------------------------------------------------
# intermediates of the tensor-core kernels against the oracle

INTER = [
    _custom("bf16", 3, 12, 20, 128, 4, 4, 1, B=1, heads=2),
    _custom("f16", 3, 12, 20, 64, 4, 4, 1, B=1, heads=2),
    _custom("bf16", 3, 12, 20, 128, 4, 4, 2, B=1, heads=2),
    _custom("f16", 3, 12, 20, 64, 3, 5, 2, B=1, heads=2),
    _custom("bf16", 2, 12, 20, 128, 4, 4, 2, Tk=4, B=1, heads=2),
    # 32 tiles a head: the L step stacks four positions in one block
    _custom("f16", 2, 16, 16, 64, 4, 4, 2, B=1, heads=2),
    # more than 256 key tiles: the separate LSE and column kernels
    _custom("bf16", 1, 12, 20, 128, 4, 4, 2, Tk=18, B=1, heads=2),
    _custom("f16", 18, 12, 20, 64, 4, 4, 2, B=1, heads=1),
]


@pytest.mark.parametrize("w", INTER, ids=[w.name for w in INTER])
def test_tensor_core_intermediates_match_the_oracle(w, cuda_lib):
    """k~ and z (f16 hi + lo), h (base 2) and, after the first iteration, q~
    (input-type hi + lo) of the last iteration against the oracle.

    Bars.  One iteration: the R step starts from the exact queries, so its
    scores are exact up to fp32 accumulation; R is rounded into the input
    type's hi/lo planes (relative 2^-16 for bf16, 2^-22 for f16) and k~, z are
    stored as f16 hi/lo (2^-22): |dk~| <= 1e-4 max|k| (and z with v), and h,
    a length-b2 fp32 sum of R (x - m) with |x - m| below 32 bits, within
    1e-3 bits.  Two or more iterations: q~ comes from the column pass, whose
    weights 2^(x - lse) take the row LSE of the one-plane (f16, relative
    2^-11) k~, so a weight is off by up to 2^-11 |x| relative; with base-2
    logits up to about 10 that is 5e-3, and each intermediate is held to 5e-3
    of its RMS (entropy: of its RMS in bits), a quarter of the output's bar."""
    q, k, v = make_inputs(w)
    _, ws, offs = _run_ws(w, q, k, v)
    g = om.Grid(w.T, w.H, w.W, w.th, w.tw, Tk=w.Tkey if w.Tk else None)
    _, states = om.monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), g, w.iters,
                                     return_states=True)
    BH, b2, b1, d = w.B * w.heads, g.b2, g.b1k, w.d
    b1p = (b1 + 3) // 4 * 4
    n = BH * b2 * b1 * d

    def planes(i, dt):
        x = _region(ws, offs[i], 2 * n, dt).view(2, BH, b2, b1, d).double().cpu()
        return (x[0] + x[1]).numpy()

    kt, z = planes(0, torch.float16), planes(1, torch.float16)
    qt = planes(2, TDT[w.dtype]) if w.iters > 1 else None
    hb = _region(ws, offs[3], BH * b2 * b1p, torch.float32).view(BH, b2, b1p)[:, :, :b1].double().cpu().numpy()
    kn, vn = k.double().numpy(), v.double().numpy()
    report = []
    for i in range(BH):
        st = states[(i // w.heads, i % w.heads)]
        checks = [("k~", kt[i], np.swapaxes(st.kt, 0, 1)), ("z", z[i], np.swapaxes(st.z, 0, 1)),
                  ("h", hb[i], st.h.T / math.log(2.0))]
        if qt is not None:
            checks.append(("q~", qt[i], np.swapaxes(st.qt, 0, 1)))
        for name, got, ref in checks:
            err = float(np.abs(got - ref).max())
            if w.iters == 1:
                bar = {"k~": 1e-4 * np.abs(kn[i // w.heads, i % w.heads]).max(),
                       "z": 1e-4 * np.abs(vn[i // w.heads, i % w.heads]).max(), "h": 1e-3}[name]
            else:
                bar = 5e-3 * float(np.sqrt((ref ** 2).mean()))
            report.append(f"{name}[{i}] {err / bar:.3f}")
            assert err <= bar, f"{w.name} head {i} {name}: max|err| {err:.3e} > bar {bar:.3e}"
    print(w.name, "err/bar:", ", ".join(report))
