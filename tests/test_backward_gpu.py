"""GPU parity of the backward (one-step forward, self-attention, optional
frame-chunk causal mask): dq, dk, dv from the C ABI against the fp64 oracle
backward on the same seeded inputs and cotangent.

Tolerance, per gradient, per head and element: |got - ref| <= tol *
RMS(ref) + (u/2) |ref|.  f32 inputs run the fp32 CUDA-core backward, tol =
1e-3: dS = L (dy.z - D) subtracts two rounded dot products of length d whose
difference is small where L is peaked, so the relative error of dS, not of
the output, sets it.  bf16/f16 inputs run the tensor-core backward, tol =
1e-2, half the forward's 2e-2 bar: its own products carry every operand as
f16 hi/lo planes, and the rest is the precision of the forward it recomputes
(R rounded to the input type in k~ = R k and z = R v, P a single f16 in
y = P z), measured at most 0.8e-2 of the RMS (a ragged 75-tile grid), so a
doubling of that error fails.
The second is the one rounding of the stored gradient (u/2 = 2^-8 for bf16,
2^-11 for f16, 0 for f32), which on peaked rows' entries of many times the RMS
is larger than any fixed fraction of the RMS.  Full-size workloads compare
sampled heads element by element and check two exact invariants on every
head: sum_tokens dv = sum_tokens dy and sum_tokens dk = 0."""

import numpy as np
import pytest
import torch

import structured_sparse_attention_grid_b200 as m
from oracle import monarch as om
from structured_sparse_attention_grid_b200.workloads import (DTYPES, WORKLOADS, Workload, make_cotangent,
                                                             make_inputs)

pytestmark = pytest.mark.gpu

TOL_GRAD = {"f32": 1e-3, "bf16": 1e-2, "f16": 1e-2}   # by input dtype
# largest relative error of one round-to-nearest store in the gradient type,
# 2^-p for p significand bits (8 for bf16, 11 for f16)
HALF_ULP = {torch.float32: 0.0, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def _wl(dtype, T, H, W, d, th, tw, C=0, B=2, heads=2, seed=7, kind="pos_planted"):
    return Workload(f"bwd_{dtype}_{T}x{H}x{W}_d{d}_{th}x{tw}_C{C}", B, heads, T, H, W, d, th, tw, 1, dtype,
                    seed, kind, planted=8, chunk_frames=C)


def _run_bwd(w, q, k, v, dy):
    qd, kd, vd, dyd = (t.cuda() for t in (q, k, v, dy))
    dq, dk, dv = (torch.empty_like(dyd) for _ in range(3))
    m.monarch_attn_bwd(qd, kd, vd, dyd, dq, dk, dv, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    return dq, dk, dv


def _grid(w):
    return om.Grid(w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)


def _compare(w, got, q, k, v, dy, heads=None):
    qn, kn, vn, dyn = (t.double().numpy() for t in (q, k, v, dy))
    ref = om.monarch_attention_backward(qn, kn, vn, dyn, _grid(w), heads=heads)
    half_ulp = HALF_ULP[got[0].dtype]
    tol = TOL_GRAD[w.dtype]
    hs = heads or [(b, h) for b in range(w.B) for h in range(w.heads)]
    worst = 0.0
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.double().cpu().numpy()
        for b, h in hs:
            rms = float(np.sqrt((r[b, h] ** 2).mean()))
            excess = np.abs(g[b, h] - r[b, h]) - half_ulp * np.abs(r[b, h])
            err = float(excess.max())
            assert err <= tol * rms, f"{w.name} {name} head {(b, h)}: max excess {err:.3e} > {tol} * rms {rms:.3e}"
            worst = max(worst, err / rms)
    return worst


def _invariants(dk, dv, dy):
    """Exact identities up to the fp32 sums and, for bf16/f16 gradients, the
    rounding of each entry (at most 2^-8 or 2^-11 relative)."""
    n = dy.shape[2]
    u = {torch.float32: 0.0, torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}[dv.dtype]
    assert torch.isfinite(dk).all() and torch.isfinite(dv).all()
    dk64, dv64, dy64 = (t.cuda().double() for t in (dk, dv, dy))
    sdv, sdy = dv64.sum(dim=2), dy64.sum(dim=2)
    tol_v = 1e-4 * dy64.abs().amax() * n ** 0.5 + u * dv64.abs().sum(dim=2)
    assert ((sdv - sdy).abs() <= tol_v).all()
    tol_k = 1e-4 * dk64.abs().amax() * n ** 0.5 + u * dk64.abs().sum(dim=2)
    assert (dk64.sum(dim=2).abs() <= tol_k).all()


CASES = [
    # (input dtype, gradient dtype, workload)
    ("f32", _wl("f32", 4, 8, 8, 64, 4, 4)),                 # the toy grid
    ("f32", _wl("bf16", 5, 12, 20, 128, 4, 4)),             # ragged: b1 = 75
    ("f32", _wl("bf16", 5, 12, 20, 128, 4, 4, C=2)),        # chunk-causal, ragged last chunk
    ("f16", _wl("f16", 3, 8, 12, 64, 2, 4)),                # gradients in the input type
    ("bf16", _wl("bf16", 6, 8, 8, 128, 4, 2, C=4)),
    ("f32", _wl("f16", 3, 12, 16, 64, 4, 4, C=1)),          # one-frame chunks
    ("f32", _wl("f32", 2, 6, 8, 64, 1, 1)),                 # b2 = 1: R = 1, dense over tiles
    ("f32", _wl("f32", 1, 6, 8, 128, 6, 8)),                # b1 = 1: one tile
    ("f32", _wl("f32", 2, 16, 16, 128, 8, 8, B=1)),         # b2 = 64, the largest tile
    ("f32", _wl("bf16", 3, 30, 52, 128, 6, 4, B=1, heads=2)),   # the 4680-token chunk grid
    ("f32", _wl("f16", 2, 16, 16, 64, 8, 8, B=1)),          # tensor cores: b2 = 64, d = 64
    ("f32", _wl("bf16", 2, 6, 8, 128, 1, 1)),               # tensor cores: b2 = 1
    ("f32", _wl("bf16", 1, 6, 8, 128, 6, 8)),               # tensor cores: b1 = 1
    ("f32", _wl("bf16", 9, 16, 16, 128, 4, 4, C=4, B=1)),   # tensor cores: several 128-tile blocks, masked
    ("f32", _wl("bf16", 2, 8, 8, 128, 4, 4, B=8, heads=12)),   # 96 head units of 8 tiles: padded blocks
    ("bf16", _wl("bf16", 6, 12, 16, 64, 4, 4, C=3, B=1)),      # tensor cores: d = 64, masked, bf16 gradients
]


@pytest.mark.parametrize("gdt,w", CASES, ids=[f"{w.name}_g{g}" for g, w in CASES])
def test_backward_matches_the_oracle(gdt, w, cuda_lib):
    q, k, v = make_inputs(w)
    dy = make_cotangent(w, gdt)
    got = _run_bwd(w, q, k, v, dy)
    assert all(t.dtype == DTYPES[gdt] for t in got)
    _invariants(got[1], got[2], dy)
    _compare(w, got, q, k, v, dy)


def test_backward_of_dense_limit_is_the_softmax_gradient(cuda_lib):
    """b2 = 1: the Monarch operator is softmax attention over the tiles."""
    w = _wl("f32", 3, 4, 6, 64, 1, 1, B=1, heads=1, kind="iid")
    q, k, v = make_inputs(w)
    dy = make_cotangent(w, "f32")
    dq, dk, dv = (t.double().cpu() for t in _run_bwd(w, q, k, v, dy))
    qq, kk, vv = (t.double().requires_grad_() for t in (q, k, v))
    y = torch.softmax(qq @ kk.transpose(-1, -2) / 8.0, dim=-1) @ vv
    y.backward(dy.double())
    for a, b in ((dq, qq.grad), (dk, kk.grad), (dv, vv.grad)):
        assert (a - b).abs().max() <= 1e-4 * b.pow(2).mean().sqrt()


@pytest.mark.parametrize("name,heads", [
    ("full_32760_bf16", [(0, 0), (1, 11)]),
    ("train_32760_bf16_causal", [(1, 5)]),
])
def test_backward_full_size_sampled_heads(name, heads, cuda_lib):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    dy = make_cotangent(w, "f32")
    got = _run_bwd(w, q, k, v, dy)
    _invariants(got[1], got[2], dy)
    _compare(w, got, q, k, v, dy, heads=heads)


def test_backward_rejects_a_kv_cache_shape(cuda_lib):
    w = _wl("bf16", 2, 8, 8, 64, 4, 4)
    q, _, _ = make_inputs(w)
    k = torch.zeros((2, 2, 3 * 64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        m.monarch_attn_bwd(q.cuda(), k, k, q.cuda().float(), *(torch.empty_like(q.cuda().float()) for _ in range(3)),
                           w.T, w.H, w.W, w.th, w.tw)


@pytest.mark.parametrize("w,gdt", [(_wl("bf16", 5, 12, 20, 128, 4, 4), "f32"),
                                   (_wl("f16", 6, 8, 8, 64, 4, 2, C=2), "f16")],
                         ids=["bf16_gf32", "f16_masked_gf16"])
def test_saved_state_pair_matches_the_recomputing_backward(w, gdt, cuda_lib):
    """monarch_attn_fwd_train writes the one-step forward's output and row LSE;
    monarch_attn_bwd_saved with them returns the gradients of monarch_attn_bwd
    bit for bit (both run the same kernels on the same values)."""
    q, k, v = (t.cuda() for t in make_inputs(w))
    dy = make_cotangent(w, gdt).cuda()
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    lse = torch.empty(m.lse_numel(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw), dtype=torch.float32,
                      device="cuda")
    m.monarch_attn_fwd_train(q, k, v, out, lse, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    ref_out = torch.empty_like(out)
    m.monarch_attn_fwd(q, k, v, ref_out, w.T, w.H, w.W, w.th, w.tw, 1, chunk_frames=w.chunk_frames)
    got = [torch.empty_like(dy) for _ in range(3)]
    ref = [torch.empty_like(dy) for _ in range(3)]
    m.monarch_attn_bwd_saved(q, k, v, out, lse, dy, *got, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    m.monarch_attn_bwd(q, k, v, dy, *ref, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    assert torch.equal(out, ref_out)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("dtype,C", [("bf16", 0), ("f32", 2)])
def test_autograd_function_gives_the_library_gradients(dtype, C, cuda_lib):
    """loss = sum(dy * monarch_attention(q, k, v)); loss.backward() yields the
    gradients of the backward entry point (f32 gradients, converted to the
    inputs' dtype by autograd)."""
    w = _wl(dtype, 4, 8, 12, 64, 2, 4, C=C)
    q, k, v = (t.cuda() for t in make_inputs(w))
    dy = make_cotangent(w, "f32").cuda()
    qg, kg, vg = (t.clone().requires_grad_() for t in (q, k, v))
    y = m.monarch_attention(qg, kg, vg, w.T, w.H, w.W, w.th, w.tw, chunk_frames=C)
    (y * dy).sum().backward()
    ref = [torch.empty_like(dy) for _ in range(3)]
    m.monarch_attn_bwd(q, k, v, dy, *ref, w.T, w.H, w.W, w.th, w.tw, chunk_frames=C)
    out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, 1, chunk_frames=C)
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), out)
    for g, r, t in zip((qg.grad, kg.grad, vg.grad), ref, (q, k, v)):
        assert g.dtype == t.dtype
        assert torch.equal(g, r.to(t.dtype))
