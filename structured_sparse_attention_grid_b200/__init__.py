"""Python binding of the B200 Monarch video-attention library (C ABI).

Argument marshalling only: every step of the forward and backward runs in the CUDA
kernels of ``libmonarch_attn.so``.  PyTorch provides device memory and
streams.  There is no fallback: if the library is missing, calls fail.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmonarch_attn.so")

MONARCH_F32, MONARCH_BF16, MONARCH_F16 = 0, 1, 2
PHASES = ("qbar", "r_step", "l_lse", "l_out", "l_col", "bwd_prep", "bwd_dq", "bwd_dkv", "bwd_r", "onestep",
          "l_lsecol")

# Every symbol the header declares, with its ctypes signature.
_SIGS = {
    "monarch_attn_fwd": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                         + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "monarch_attn_fwd_ex": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                            + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "monarch_attn_bwd": (ctypes.c_int, [ctypes.c_void_p] * 7 + [ctypes.c_int] * 11 + [ctypes.c_void_p]),
    "monarch_attn_bwd_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 11),
    "monarch_attn_lse_bytes": (ctypes.c_size_t, [ctypes.c_int] * 8),
    "monarch_attn_fwd_train": (ctypes.c_int, [ctypes.c_void_p] * 5 + [ctypes.c_int] * 10 + [ctypes.c_void_p]),
    "monarch_attn_bwd_saved": (ctypes.c_int, [ctypes.c_void_p] * 9 + [ctypes.c_int] * 11 + [ctypes.c_void_p]),
    "monarch_attn_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 9 + [ctypes.c_long, ctypes.c_int]),
    "monarch_attn_fwd_ws": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                            + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                               ctypes.c_size_t, ctypes.c_void_p]),
    "monarch_attn_fwd_noalloc": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                                 + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "monarch_attn_fwd_host": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                              + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "monarch_attn_fwd_host_ex": (ctypes.c_int, [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9
                                 + [ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "monarch_attn_workspace_layout": (ctypes.c_size_t, [ctypes.c_int] * 9
                                      + [ctypes.c_long, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]),
    "monarch_attn_launch_count": (ctypes.c_ulonglong, []),
    "monarch_attn_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "monarch_attn_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_double),
                                                 ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int,
                                                 ctypes.c_int]),
    "monarch_attn_device_error": (ctypes.c_int, [ctypes.c_int]),
    "monarch_attn_last_error": (ctypes.c_char_p, []),
    "monarch_attn_version": (ctypes.c_int, []),
}

_lib = None


class MonarchError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"monarch_attn error {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH):
    """Loads the C-ABI library (once) and declares its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m structured_sparse_attention_grid_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _dtype_code(t) -> int:
    import torch
    codes = {torch.float32: MONARCH_F32, torch.bfloat16: MONARCH_BF16, torch.float16: MONARCH_F16}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(rc: int):
    if rc != 0:
        raise MonarchError(rc, _lib.monarch_attn_last_error().decode())


def _shape_args(q, k, T, H, W, tile_h, tile_w, iters):
    B, heads, nq, d = q.shape
    if nq != T * H * W:
        raise ValueError(f"q has {nq} tokens, grid {T}x{H}x{W} has {T * H * W}")
    return [B, heads, T, H, W, d, tile_h, tile_w, iters, int(k.shape[2])]


def _check_tensors(*ts):
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, heads, N, d]")


def monarch_attn_fwd(q, k, v, out, T, H, W, tile_h, tile_w, iters, stream=None, chunk_frames=0):
    """out <- Monarch attention of (q, k, v); CUDA tensors, contiguous
    [B, heads, N, d]; kv length = k.shape[2]; out is float32 or q's dtype.
    ``chunk_frames`` > 0 applies the frame-chunk causal mask of training
    over the whole sequence (monarch_attn_fwd_ex).  Asynchronous on ``stream``."""
    lib = load_library()
    _check_tensors(q, k, v, out)
    args = _shape_args(q, k, T, H, W, tile_h, tile_w, iters)
    if chunk_frames:
        _check(lib.monarch_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                       *args, int(chunk_frames), _dtype_code(q), _dtype_code(out),
                                       _stream_ptr(stream)))
    else:
        _check(lib.monarch_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    *args, _dtype_code(q), _dtype_code(out), _stream_ptr(stream)))
    return out


def monarch_attn_bwd(q, k, v, dy, dq, dk, dv, T, H, W, tile_h, tile_w, stream=None, chunk_frames=0):
    """dq, dk, dv <- gradients of sum(dy * out) for the one-step forward
    out = monarch_attn_fwd(q, k, v, ..., iters=1) (self-attention, optional
    frame-chunk causal mask).  q, k, v in one dtype; dy, dq, dk, dv float32 or
    q's dtype; all CUDA, contiguous [B, heads, T*H*W, d].  Asynchronous."""
    lib = load_library()
    _check_tensors(q, k, v, dy, dq, dk, dv)
    B, heads, nq, d = q.shape
    if nq != T * H * W:
        raise ValueError(f"q has {nq} tokens, grid {T}x{H}x{W} has {T * H * W}")
    for t in (k, v, dy, dq, dk, dv):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError("k, v, dy, dq, dk, dv must have q's shape (self-attention)")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share a dtype")
    g = _dtype_code(dy)
    if any(_dtype_code(t) != g for t in (dq, dk, dv)):
        raise TypeError("dy, dq, dk, dv must share a dtype")
    _check(lib.monarch_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), dy.data_ptr(), dq.data_ptr(),
                                dk.data_ptr(), dv.data_ptr(), B, heads, T, H, W, d, tile_h, tile_w,
                                int(chunk_frames), _dtype_code(q), g, _stream_ptr(stream)))
    return dq, dk, dv


def lse_numel(B, heads, T, H, W, d, tile_h, tile_w) -> int:
    """float32 elements of the row-LSE buffer of monarch_attn_fwd_train."""
    n = load_library().monarch_attn_lse_bytes(B, heads, T, H, W, d, tile_h, tile_w)
    if n == 0:
        raise MonarchError(-1, _lib.monarch_attn_last_error().decode())
    return int(n) // 4


def monarch_attn_fwd_train(q, k, v, out, lse, T, H, W, tile_h, tile_w, stream=None, chunk_frames=0):
    """One-step forward (bf16/f16 inputs) that also keeps the row LSE for
    monarch_attn_bwd_saved: out float32 [B, heads, T*H*W, d], lse float32 with
    lse_numel(...) elements (contiguous CUDA tensors).  Asynchronous."""
    lib = load_library()
    _check_tensors(q, k, v, out, lse)
    B, heads, nq, d = q.shape
    import torch
    if out.dtype != torch.float32 or lse.dtype != torch.float32:
        raise TypeError("out and lse must be float32")
    _check(lib.monarch_attn_fwd_train(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                      B, heads, T, H, W, d, tile_h, tile_w, int(chunk_frames), _dtype_code(q),
                                      _stream_ptr(stream)))
    return out, lse


def monarch_attn_bwd_saved(q, k, v, out, lse, dy, dq, dk, dv, T, H, W, tile_h, tile_w, stream=None,
                           chunk_frames=0):
    """monarch_attn_bwd with the out and lse of monarch_attn_fwd_train (no
    recompute of the output pass)."""
    lib = load_library()
    _check_tensors(q, k, v, out, lse, dy, dq, dk, dv)
    B, heads, nq, d = q.shape
    g = _dtype_code(dy)
    if any(_dtype_code(t) != g for t in (dq, dk, dv)):
        raise TypeError("dy, dq, dk, dv must share a dtype")
    _check(lib.monarch_attn_bwd_saved(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                      dy.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, heads, T, H, W,
                                      d, tile_h, tile_w, int(chunk_frames), _dtype_code(q), g, _stream_ptr(stream)))
    return dq, dk, dv


def workspace_layout(B, heads, T, H, W, d, tile_h, tile_w, iters, kv_len, dtype_code):
    lib = load_library()
    offs = (ctypes.c_size_t * 7)()
    total = lib.monarch_attn_workspace_layout(B, heads, T, H, W, d, tile_h, tile_w, iters,
                                              kv_len, dtype_code, offs)
    if total == 0:
        raise MonarchError(-1, lib.monarch_attn_last_error().decode())
    return int(total), [int(o) for o in offs]


def monarch_attn_fwd_ws(q, k, v, out, workspace, T, H, W, tile_h, tile_w, iters, stream=None):
    """As monarch_attn_fwd with a caller-owned device workspace (uint8 tensor)."""
    lib = load_library()
    _check_tensors(q, k, v, out)
    args = _shape_args(q, k, T, H, W, tile_h, tile_w, iters)
    _check(lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   *args, _dtype_code(q), _dtype_code(out), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(),
                                   _stream_ptr(stream)))
    return out


def monarch_attn_fwd_noalloc(q, k, v, out, T, H, W, tile_h, tile_w, iters, stream=None):
    """As monarch_attn_fwd, for callers that cannot allocate device memory
    while running: the library takes its workspace from a fixed 128 MiB array
    it holds on each device, so no allocation happens.  Larger problems are
    rejected; concurrent calls on one device must not overlap on the GPU."""
    lib = load_library()
    _check_tensors(q, k, v, out)
    args = _shape_args(q, k, T, H, W, tile_h, tile_w, iters)
    _check(lib.monarch_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        *args, _dtype_code(q), _dtype_code(out), _stream_ptr(stream)))
    return out


def monarch_attn_fwd_host(q, k, v, out, T, H, W, tile_h, tile_w, iters, stream=None, chunk_frames=0):
    """End-to-end call on HOST tensors (pinned for asynchronous copies): the
    library copies in, computes, copies out and synchronises the stream.
    ``chunk_frames`` > 0 applies the frame-chunk causal mask."""
    lib = load_library()
    _check_tensors(q, k, v, out)
    args = _shape_args(q, k, T, H, W, tile_h, tile_w, iters)
    if chunk_frames:
        _check(lib.monarch_attn_fwd_host_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                            *args, int(chunk_frames), _dtype_code(q), _dtype_code(out),
                                            _stream_ptr(stream)))
    else:
        _check(lib.monarch_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                         *args, _dtype_code(q), _dtype_code(out), _stream_ptr(stream)))
    return out


def launch_count() -> int:
    """Kernels launched so far by this process through the library."""
    return int(load_library().monarch_attn_launch_count())


def profile_enable(on: bool = True) -> None:
    """Bracket every library kernel with CUDA events on its stream."""
    load_library().monarch_attn_profile_enable(1 if on else 0)


def profile_read(reset: bool = True) -> dict:
    """{phase: (total_ms, launches)} accumulated since the last reset."""
    lib = load_library()
    n = len(PHASES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_ulonglong * n)()
    _check(lib.monarch_attn_profile_read(ms, cnt, n, 1 if reset else 0))
    return {p: (float(ms[i]), int(cnt[i])) for i, p in enumerate(PHASES)}


def device_error(reset: bool = False) -> int:
    """0 unless a library kernel gave up a bounded wait (see the header)."""
    return int(load_library().monarch_attn_device_error(1 if reset else 0))


def _autograd_function():
    import torch

    class MonarchAttentionFn(torch.autograd.Function):
        """One-step Monarch attention with its backward (the finetuned
        regime): forward through monarch_attn_fwd_train (bf16/f16, keeps the
        row LSE) or monarch_attn_fwd (f32); backward through
        monarch_attn_bwd_saved or monarch_attn_bwd, with f32 gradients."""

        @staticmethod
        def forward(ctx, q, k, v, T, H, W, tile_h, tile_w, chunk_frames):
            q, k, v = (t.contiguous() for t in (q, k, v))
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
            if q.dtype == torch.float32:
                monarch_attn_fwd(q, k, v, out, T, H, W, tile_h, tile_w, 1, chunk_frames=chunk_frames)
                lse = torch.empty(0, dtype=torch.float32, device=q.device)
            else:
                B, heads, _, d = q.shape
                lse = torch.empty(lse_numel(B, heads, T, H, W, d, tile_h, tile_w), dtype=torch.float32,
                                  device=q.device)
                monarch_attn_fwd_train(q, k, v, out, lse, T, H, W, tile_h, tile_w, chunk_frames=chunk_frames)
            ctx.save_for_backward(q, k, v, out, lse)
            ctx.geom = (T, H, W, tile_h, tile_w, chunk_frames)
            return out

        @staticmethod
        def backward(ctx, dy):
            q, k, v, out, lse = ctx.saved_tensors
            T, H, W, tile_h, tile_w, chunk_frames = ctx.geom
            dy = dy.contiguous()
            if dy.dtype != torch.float32:
                dy = dy.float()
            dq, dk, dv = (torch.empty_like(dy) for _ in range(3))
            if q.dtype == torch.float32:
                monarch_attn_bwd(q, k, v, dy, dq, dk, dv, T, H, W, tile_h, tile_w, chunk_frames=chunk_frames)
            else:
                monarch_attn_bwd_saved(q, k, v, out, lse, dy, dq, dk, dv, T, H, W, tile_h, tile_w,
                                       chunk_frames=chunk_frames)
            return dq, dk, dv, None, None, None, None, None, None

    return MonarchAttentionFn


_FN = None


def monarch_attention(q, k, v, T, H, W, tile_h, tile_w, chunk_frames=0):
    """Differentiable one-step Monarch attention (self-attention, optional
    frame-chunk causal mask): CUDA tensors [B, heads, T*H*W, d]; returns the
    float32 output.  Gradients flow to q, k, v (float32, converted by
    autograd to the inputs' dtype)."""
    global _FN
    if _FN is None:
        _FN = _autograd_function()
    return _FN.apply(q, k, v, T, H, W, tile_h, tile_w, chunk_frames)
