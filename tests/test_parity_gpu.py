"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Tolerances: fp32 max|err| <= 1e-4; bf16/f16 max|err| <= 2e-2 * RMS(oracle
output), each head against its own RMS.  Full-size workloads compare every
output of a sample of heads (heads are independent, so a head is an exact
sample) plus all-head properties (finite output, every row a convex
combination of v rows)."""

import numpy as np
import pytest
import torch

import structured_sparse_attention_grid_b200 as m
from oracle import monarch as om
from structured_sparse_attention_grid_b200.workloads import WORKLOADS, Workload, make_inputs
from tests.parity_helpers import STORE_BITS, TOL_F32, compare_per_head, grid_of, oracle_out

pytestmark = pytest.mark.gpu

_grid = grid_of


def _run_gpu(w, q, k, v, out_dtype=torch.float32):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty(qd.shape, dtype=out_dtype, device=qd.device)
    m.monarch_attn_fwd(qd, kd, vd, out, w.T, w.H, w.W, w.th, w.tw, w.iters, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    return out


def _compare(w, out_gpu, q, k, v, heads=None, store_bits=None):
    ref = oracle_out(w, q, k, v, heads=heads)
    return compare_per_head(w, out_gpu, ref, heads=heads, store_bits=store_bits)


def _all_head_properties(out, v):
    o = out.float()
    assert torch.isfinite(o).all()
    vd = v.cuda().float()
    lo = vd.amin(dim=2, keepdim=True)
    hi = vd.amax(dim=2, keepdim=True)
    slack = 1e-2 * (hi - lo) + 1e-3
    assert (o >= lo - slack).all() and (o <= hi + slack).all()


@pytest.mark.parametrize("name", ["toy_256_f32", "toy_256_f32_separable"])
def test_toy_fp32(name, cuda_lib):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _compare(w, out, q, k, v)


def test_toy_separable_matches_dense_attention(cuda_lib):
    w = WORKLOADS["toy_256_f32_separable"]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v).double().cpu().numpy()
    ref = om.dense_attention(q.double().numpy(), k.double().numpy(), v.double().numpy())
    assert np.abs(out - ref).max() <= TOL_F32


@pytest.mark.parametrize("name", ["chunk_4680_bf16", "chunk_4680_bf16_1step", "kvcache_4680x32760_bf16",
                                  "sweep_2048_f16", "sweep_8192_f16"])
def test_workload_all_heads(name, cuda_lib):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _all_head_properties(out, v)
    _compare(w, out, q, k, v)


@pytest.mark.parametrize("name,heads", [
    # six heads over both batches, among them the most peaked one (1, 5)
    ("full_32760_bf16", [(0, 0), (0, 6), (0, 11), (1, 0), (1, 5), (1, 11)]),
    ("full_32760_bf16_1step", [(1, 5)]),
    ("sweep_32768_f16", [(0, 0), (0, 13), (0, 23)]),
])
def test_workload_sampled_heads(name, heads, cuda_lib):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _all_head_properties(out, v)
    _compare(w, out, q, k, v, heads=heads)


def _custom(dtype, T, H, W, d, th, tw, iters, Tk=0, B=2, heads=3, kind="pos_planted", seed=7, C=0):
    return Workload(f"custom_{dtype}_{T}x{H}x{W}_d{d}_{th}x{tw}_it{iters}_Tk{Tk}_C{C}", B, heads, T, H, W, d,
                    th, tw, iters, dtype, seed, kind, Tk=Tk, planted=8, chunk_frames=C)


EDGE = [
    # ragged tiles (b1 = 75 not a multiple of any tile), every iteration count
    _custom("bf16", 5, 12, 20, 128, 4, 4, 1),
    _custom("bf16", 5, 12, 20, 128, 4, 4, 2),
    _custom("f16", 5, 12, 20, 64, 4, 4, 3),
    _custom("f32", 3, 8, 12, 128, 2, 4, 2),
    # KV cache with b1q != b1k and a ragged tail
    _custom("bf16", 2, 12, 20, 128, 4, 4, 2, Tk=7),
    _custom("f16", 1, 8, 8, 64, 4, 2, 3, Tk=5),
    _custom("f32", 2, 8, 8, 64, 4, 4, 2, Tk=3),
    # degenerate: one position per tile (b2 = 1) and one tile per sequence (b1 = 1)
    _custom("bf16", 2, 6, 8, 128, 1, 1, 2),
    _custom("bf16", 1, 6, 8, 128, 6, 8, 2),
    _custom("f32", 1, 6, 8, 64, 6, 8, 1),
    # largest supported tile (64 positions) and b1 exactly one 128-row block
    _custom("f16", 2, 32, 32, 64, 8, 8, 2),
    _custom("bf16", 8, 16, 16, 128, 4, 2, 2, B=1, heads=2),
    # 64 positions with d = 128 (two tiles an R-step item): the fused L step,
    # a KV cache, and 288 tiles a head (separate LSE and column passes)
    _custom("bf16", 2, 16, 16, 128, 8, 8, 2),
    _custom("bf16", 1, 16, 16, 128, 8, 8, 2, Tk=3),
    _custom("bf16", 8, 48, 48, 128, 8, 8, 2, B=1, heads=1),
    # positions per tile not a multiple of 8 (padded rows inside each stacked
    # R-step tile), with and without a KV cache, both head sizes
    _custom("bf16", 2, 9, 10, 128, 3, 5, 2),
    _custom("f16", 2, 10, 15, 64, 5, 5, 3),
    _custom("bf16", 2, 9, 10, 128, 3, 5, 2, Tk=5),
    _custom("bf16", 3, 12, 21, 64, 3, 7, 1),
    # small grids whose L step stacks positions: 32 tiles (four a block), 64
    # tiles (two), 16 tiles (eight), with one, two and three iterations
    _custom("f16", 2, 16, 16, 64, 4, 4, 2),
    _custom("bf16", 4, 8, 8, 128, 2, 2, 1),
    _custom("bf16", 1, 16, 32, 128, 4, 4, 2),
    _custom("f16", 1, 16, 16, 64, 4, 4, 3),
]


@pytest.mark.parametrize("w", EDGE, ids=[w.name for w in EDGE])
def test_edge_cases(w, cuda_lib):
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _compare(w, out, q, k, v)


def test_degenerate_grids_reduce_to_dense_attention(cuda_lib):
    for w in (_custom("f32", 2, 6, 8, 64, 1, 1, 2, kind="iid"), _custom("f32", 1, 6, 8, 64, 6, 8, 2, kind="iid")):
        q, k, v = make_inputs(w)
        out = _run_gpu(w, q, k, v).double().cpu().numpy()
        ref = om.dense_attention(q.double().numpy(), k.double().numpy(), v.double().numpy())
        assert np.abs(out - ref).max() <= TOL_F32


def test_intermediates_match_the_oracle_on_the_toy(cuda_lib):
    w = _custom("f32", 4, 8, 8, 64, 4, 4, 2, B=1, heads=2, kind="iid")
    q, k, v = make_inputs(w)
    total, offs = m.workspace_layout(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw, w.iters, w.Nk, m.MONARCH_F32)
    ws = torch.zeros(total, dtype=torch.uint8, device="cuda")
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty_like(qd)
    m.monarch_attn_fwd_ws(qd, kd, vd, out, ws, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    g = _grid(w)
    _, states = om.monarch_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), g,
                                     w.iters, return_states=True)
    b2, b1, d = g.b2, g.b1k, w.d

    def view(i, n, dt=torch.float32):
        return ws[offs[i]:offs[i] + n * 4].view(dt)

    kt = view(0, 2 * b2 * b1 * d).view(2, b2, b1, d).cpu().double().numpy()
    qt = view(2, 2 * b2 * b1 * d).view(2, b2, b1, d).cpu().double().numpy()
    b1p = (b1 + 3) // 4 * 4  # h rows are padded to a multiple of 4
    hh = view(3, 2 * b2 * b1p).view(2, b2, b1p)[:, :, :b1].cpu().double().numpy()
    for h in range(2):
        st = states[(0, h)]
        np.testing.assert_allclose(kt[h], np.swapaxes(st.kt, 0, 1), atol=1e-4)
        np.testing.assert_allclose(qt[h], np.swapaxes(st.qt, 0, 1), atol=1e-4)
        np.testing.assert_allclose(hh[h], st.h.T, atol=1e-4)


def test_output_in_input_dtype_is_the_rounded_f32_output(cuda_lib):
    for name in ("chunk_4680_bf16", "sweep_2048_f16"):
        w = WORKLOADS[name]
        q, k, v = make_inputs(w)
        o32 = _run_gpu(w, q, k, v)
        olow = _run_gpu(w, q, k, v, out_dtype=q.dtype)
        assert torch.equal(olow, o32.to(q.dtype))


@pytest.mark.parametrize("name", ["chunk_4680_bf16", "kvcache_4680x32760_bf16", "sweep_2048_f16",
                                  "sweep_8192_f16"])
def test_output_in_input_dtype_matches_the_oracle(name, cuda_lib):
    """out_dtype = the input dtype, against the oracle: the output bar plus
    one round-to-nearest store of each element (2^-8 |ref| for bf16, 2^-11
    for f16), the allowance the backward's gradients also get."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v, out_dtype=q.dtype)
    assert out.dtype == q.dtype
    _compare(w, out, q, k, v, store_bits=STORE_BITS[w.dtype])


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32", "bf16"])
def test_output_buffer_with_16_byte_alignment(out_dtype, cuda_lib):
    """The output pass stores 32 bytes at a time when the caller's buffer is
    32-byte aligned and 16 bytes at a time otherwise (the ABI asks for 16);
    both give the same bits."""
    w = _custom("bf16", 5, 12, 20, 128, 4, 4, 2)
    q, k, v = (t.cuda() for t in make_inputs(w))
    n = q.numel()
    a = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    shift = 16 // a.element_size()
    b = torch.empty(n + shift, dtype=out_dtype, device=q.device)[shift:].view(q.shape)
    assert a.data_ptr() % 32 == 0 and b.data_ptr() % 32 == 16
    for o in (a, b):
        m.monarch_attn_fwd(q, k, v, o, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    assert torch.equal(a, b)


def test_host_buffer_entry_point(cuda_lib):
    w = WORKLOADS["toy_256_f32"]
    q, k, v = make_inputs(w)
    out = torch.empty_like(q).pin_memory()
    m.monarch_attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out, w.T, w.H, w.W, w.th,
                            w.tw, w.iters)
    _compare(w, out, q, k, v)


@pytest.mark.parametrize("name", ["chunk_4680_bf16", "kvcache_4680x32760_bf16"])
def test_host_buffer_groups_match_the_device_call(name, cuda_lib):
    """The host entry point pipelines groups of (batch, head) units (1, 2, 3,
    3, 2, 1 heads for chunk_4680 and 1, 2, 2, 2, 2, 2, 1 for the KV cache);
    every row is computed by the same arithmetic, key tiles stacked the same
    way, as in one device call over all units."""
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    out = torch.empty(q.shape, dtype=torch.float32).pin_memory()
    m.monarch_attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out, w.T, w.H, w.W, w.th,
                            w.tw, w.iters)
    dev = _run_gpu(w, q, k, v).cpu()
    assert torch.equal(out, dev)


def test_host_buffer_groups_with_the_chunk_mask(cuda_lib):
    """The masked host entry point (groups of 1, 2, 2, 2, 2, 2, 1 heads)
    equals the masked device call."""
    w = _custom("bf16", 6, 30, 52, 128, 6, 4, 2, B=1, heads=12, C=2)
    q, k, v = make_inputs(w)
    out = torch.empty(q.shape, dtype=torch.float32).pin_memory()
    m.monarch_attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out, w.T, w.H, w.W, w.th,
                            w.tw, w.iters, chunk_frames=w.chunk_frames)
    dev = _run_gpu(w, q, k, v).cpu()
    assert torch.equal(out, dev)


def test_workspace_entry_point_matches_allocating_call(cuda_lib):
    w = WORKLOADS["chunk_4680_bf16"]
    q, k, v = (t.cuda() for t in make_inputs(w))
    total, _ = m.workspace_layout(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw, w.iters, w.Nk, m.MONARCH_BF16)
    ws = torch.empty(total, dtype=torch.uint8, device="cuda")
    a = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    b = torch.empty_like(a)
    m.monarch_attn_fwd(q, k, v, a, w.T, w.H, w.W, w.th, w.tw, w.iters)
    m.monarch_attn_fwd_ws(q, k, v, b, ws, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_repeated_calls_are_deterministic(cuda_lib):
    w = WORKLOADS["sweep_2048_f16"]
    q, k, v = (t.cuda() for t in make_inputs(w))
    a = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    b = torch.empty_like(a)
    m.monarch_attn_fwd(q, k, v, a, w.T, w.H, w.W, w.th, w.tw, w.iters)
    m.monarch_attn_fwd(q, k, v, b, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_invalid_call_returns_an_error_and_leaves_the_context_usable(cuda_lib):
    w = WORKLOADS["toy_256_f32"]
    q, k, v = (t.cuda() for t in make_inputs(w))
    out = torch.empty_like(q)
    with pytest.raises(m.MonarchError) as e:
        m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, 3, w.tw, w.iters)  # 3 does not divide H
    assert e.value.code == -1
    m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


def test_bf16_queries_beyond_the_f16_range_set_the_range_error(cuda_lib):
    # The L step computes in f16: a bf16 query of magnitude >= 65520 cannot be
    # represented, and the call reports it through the device error word
    # (kErrRange = 3) rather than returning infinities silently.
    w = _custom("bf16", 2, 12, 20, 128, 4, 4, 1, B=1, heads=1)
    q, k, v = (t.cuda() for t in make_inputs(w))
    q[0, 0, 17, 5] = 1.0e6
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    m.device_error(reset=True)
    m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert m.device_error(reset=True) == 3
    # the context stays usable and an in-range call is clean
    q[0, 0, 17, 5] = 0.5
    m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, w.iters)
    torch.cuda.synchronize()
    assert m.device_error(reset=True) == 0
    assert torch.isfinite(out).all()


# ---- frame-chunk causal mask (training over the whole sequence) ----------------

CAUSAL = [
    # chunk boundaries not aligned to the 64/128-tile blocks, several blocks per row
    _custom("bf16", 8, 16, 16, 128, 4, 2, 2, C=2, B=1, heads=2),
    _custom("bf16", 7, 12, 20, 128, 4, 4, 3, C=3),          # ragged last chunk
    _custom("bf16", 5, 12, 20, 128, 4, 4, 1, C=1),          # one frame per chunk, one iteration
    _custom("f16", 6, 16, 16, 64, 8, 8, 2, C=2),            # 64-position tiles
    _custom("bf16", 4, 9, 10, 128, 3, 5, 2, C=2),           # b2 not a multiple of 8
    _custom("f32", 5, 8, 12, 64, 2, 4, 2, C=2),             # CUDA-core path
    _custom("bf16", 20, 12, 20, 128, 4, 4, 2, C=3, B=1, heads=2),   # 300 tiles: separate LSE and column kernels
    _custom("bf16", 4, 8, 16, 128, 2, 4, 2, C=2),          # 64 tiles, two positions stacked, masked
    _custom("f16", 8, 8, 8, 64, 4, 4, 2, C=3),             # 32 tiles, four stacked, ragged last chunk
]


@pytest.mark.parametrize("w", CAUSAL, ids=[w.name for w in CAUSAL])
def test_chunk_causal_mask(w, cuda_lib):
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _compare(w, out, q, k, v)


def test_chunk_causal_separable_is_masked_dense_attention(cuda_lib):
    w = _custom("f32", 6, 8, 8, 64, 4, 4, 1, C=2, B=1, heads=2, kind="separable")
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v).double().cpu().numpy()
    mask = om.frame_chunk_mask(w.T, w.T, w.H, w.W, w.chunk_frames)
    ref = om.dense_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), mask=mask)
    assert np.abs(out - ref).max() <= 1e-4


def test_one_chunk_equals_the_bidirectional_call(cuda_lib):
    w0 = _custom("bf16", 4, 12, 20, 128, 4, 4, 2)
    q, k, v = make_inputs(w0)
    a = _run_gpu(w0, q, k, v)
    b = _run_gpu(_custom("bf16", 4, 12, 20, 128, 4, 4, 2, C=4), q, k, v)
    assert torch.equal(a, b)


def test_training_workload_sampled_heads(cuda_lib):
    w = WORKLOADS["train_32760_bf16_causal"]
    q, k, v = make_inputs(w)
    out = _run_gpu(w, q, k, v)
    _all_head_properties(out, v)
    _compare(w, out, q, k, v, heads=[(1, 5)])


def test_chunk_mask_with_a_kv_cache_is_unsupported(cuda_lib):
    w = WORKLOADS["kvcache_4680x32760_bf16"]
    q, k, v = (t.cuda() for t in make_inputs(w))
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    with pytest.raises(m.MonarchError) as e:
        m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, w.iters, chunk_frames=1)
    assert e.value.code == -4


ONESTEP = [
    WORKLOADS["chunk_4680_bf16_1step"],
    _custom("f16", 5, 12, 20, 64, 4, 4, 1),
    _custom("bf16", 3, 12, 21, 64, 3, 7, 1),
    _custom("bf16", 7, 12, 20, 128, 4, 4, 1, C=3),
]


@pytest.mark.parametrize("w", ONESTEP, ids=[w.name for w in ONESTEP])
def test_one_step_kernel_equals_the_two_kernel_forward(w, cuda_lib, monkeypatch):
    """iters = 1 runs the R step and the output pass as two kernels, or, with
    MONARCH_ONESTEP_KERNEL=1, as one kernel whose output items wait for the
    R-step items of their head; the training forward runs the same arithmetic
    as two kernels and also keeps the row LSE.  The three outputs agree bit
    for bit."""
    q, k, v = (t.cuda() for t in make_inputs(w))
    outs = [torch.full(q.shape, float("nan"), dtype=torch.float32, device=q.device) for _ in range(3)]
    lse = torch.empty(m.lse_numel(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw), dtype=torch.float32,
                      device=q.device)
    m.profile_enable(True)
    m.profile_read(reset=True)
    for fused, out in ((True, outs[0]), (False, outs[1])):
        if fused:
            monkeypatch.setenv("MONARCH_ONESTEP_KERNEL", "1")
        else:
            monkeypatch.delenv("MONARCH_ONESTEP_KERNEL", raising=False)
        m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, 1, chunk_frames=w.chunk_frames)
        torch.cuda.synchronize()
        prof = m.profile_read(reset=True)
        if fused:
            assert prof["onestep"][1] == 1 and prof["r_step"][1] == 0 and prof["l_out"][1] == 0
        else:
            assert prof["onestep"][1] == 0 and prof["r_step"][1] == 1 and prof["l_out"][1] == 1
    m.profile_enable(False)
    m.monarch_attn_fwd_train(q, k, v, outs[2], lse, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    assert m.device_error() == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_one_step_kernel_with_a_kv_cache(cuda_lib, monkeypatch):
    """The single one-step kernel on a KV-cache step (the mean-query kernel
    runs first, cached tiles start from it) equals the two-kernel call bit for
    bit and the oracle within the bar."""
    w = _custom("bf16", 2, 12, 20, 128, 4, 4, 1, Tk=5)
    q, k, v = make_inputs(w)
    monkeypatch.setenv("MONARCH_ONESTEP_KERNEL", "1")
    a = _run_gpu(w, q, k, v)
    monkeypatch.delenv("MONARCH_ONESTEP_KERNEL")
    b = _run_gpu(w, q, k, v)
    assert m.device_error() == 0
    assert torch.equal(a, b)
    _compare(w, a, q, k, v)
