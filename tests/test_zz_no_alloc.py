"""The allocation-free entry point, monarch_attn_fwd_noalloc.

It serves callers that cannot allocate device memory while they run (a
real-time generation loop that must not stall or fail on an allocation, or a
host application that owns all device memory): its workspace is a fixed
128 MiB array in device memory that the library holds on every device.  These
tests call it through the C ABI and check that it returns what the
allocating entry point returns, on two calls in a row (the array keeps the
previous call's contents, so the second call must not depend on them).

This file is collected last so that, in a run that stops at the first
failure, every other test has already run.
"""

import ctypes

import pytest
import torch

import structured_sparse_attention_grid_b200 as m
from structured_sparse_attention_grid_b200.workloads import WORKLOADS, Workload, make_inputs

TOL_F32 = 1e-4
TOL_LOWP = 2e-2


def _abi_call(fn, q, k, v, out, w, stream):
    code = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
    return fn(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
              ctypes.c_void_p(out.data_ptr()), w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw, w.iters,
              ctypes.c_long(w.Nk), code[q.dtype], code[out.dtype], ctypes.c_void_p(stream))


# a small KV-cache step: one query frame against three key frames
KV_SMALL = Workload("noalloc_kv_1x3", 1, 2, 1, 12, 20, 128, 4, 4, 2, "bf16", 9, "pos_planted", Tk=3, planted=4)
CASES = [(WORKLOADS["chunk_4680_bf16"], torch.float32), (WORKLOADS["toy_256_f32"], torch.float32),
         (WORKLOADS["sweep_2048_f16"], torch.float32), (KV_SMALL, torch.float32),
         (WORKLOADS["chunk_4680_bf16"], torch.bfloat16)]


@pytest.mark.gpu
@pytest.mark.parametrize("w,out_dtype", CASES, ids=[f"{w.name}-{str(dt)[6:]}" for w, dt in CASES])
def test_noalloc_matches_the_allocating_entry_point(w, out_dtype, cuda_lib):
    lib = m.load_library()
    q, k, v = (t.cuda() for t in make_inputs(w))
    stream = torch.cuda.current_stream().cuda_stream
    ref = torch.empty(q.shape, dtype=out_dtype, device="cuda")
    assert _abi_call(lib.monarch_attn_fwd, q, k, v, ref, w, stream) == 0, lib.monarch_attn_last_error().decode()
    torch.cuda.synchronize()
    rms = float(ref.double().pow(2).mean().sqrt())
    tol = TOL_F32 if w.dtype == "f32" else TOL_LOWP * rms
    for call in range(2):
        got = torch.full(q.shape, float("nan"), dtype=out_dtype, device="cuda")
        rc = _abi_call(lib.monarch_attn_fwd_noalloc, q, k, v, got, w, stream)
        assert rc == 0, lib.monarch_attn_last_error().decode()
        torch.cuda.synchronize()
        err = float((got.double() - ref.double()).abs().max())
        assert err <= tol, f"call {call}: max|err| {err:.3e} > {tol:.3e}"
    assert m.device_error() == 0


@pytest.mark.gpu
def test_noalloc_rejects_a_problem_larger_than_its_scratch(cuda_lib):
    lib = m.load_library()
    w = WORKLOADS["full_32760_bf16"]  # about 1.35 GiB of workspace
    assert lib.monarch_attn_workspace_bytes(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw, w.iters, w.Nk, 1) > (128 << 20)
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")  # never touched: the size check comes first
    rc = lib.monarch_attn_fwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), w.B, w.heads, w.T,
                                      w.H, w.W, w.d, w.th, w.tw, w.iters, w.Nk, 1, 1, None)
    assert rc == -2
    assert "scratch" in lib.monarch_attn_last_error().decode()
