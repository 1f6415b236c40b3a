"""CPU checks of the C-ABI library: it loads without a GPU, exports every
symbol the header declares, and validates arguments on the host (no compute
call is made here)."""

import ctypes
import os
import re

import pytest

import structured_sparse_attention_grid_b200 as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \t\*]*?\b(monarch_\w+)\s*\(", src, flags=re.M)
    return names


@pytest.fixture(scope="module")
def lib():
    from structured_sparse_attention_grid_b200 import build
    build.build()
    return m.load_library()


def test_header_declares_the_entry_points():
    names = _declared_functions()
    assert "monarch_attn_fwd" in names and "monarch_attn_last_error" in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) == set(m._SIGS)


def _c_kind(decl: str):
    """(kind, bytes) of a C type: pointers (and the opaque stream handle) are
    ("ptr", 8); integers carry their sign and width."""
    t = " ".join(re.sub(r"\bconst\b", "", decl).split())
    if "*" in t or t == "cudaStream_t":
        return ("ptr", 8)
    return {"int": ("int", 4), "long": ("int", 8), "size_t": ("uint", 8), "unsigned long long": ("uint", 8),
            "unsigned": ("uint", 4), "void": ("void", 0)}[t]


def _param_type(p: str) -> str:
    """The type of one named parameter; an array parameter decays to a pointer."""
    m_ = re.match(r"^(.*?[\s\*])(\w+)\s*(\[[^\]]*\])?$", p.strip())
    assert m_, p
    return m_.group(1).strip() + ("*" if m_.group(3) else "")


def _ctypes_kind(t):
    if t is None:
        return ("void", 0)
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return ("ptr", 8)
    return ("int" if t(-1).value < 0 else "uint", ctypes.sizeof(t))


def _prototypes():
    src = open(os.path.join(ROOT, "include", "monarch_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for ret, name, params in re.findall(r"^([A-Za-z_][\w \t\*]*?)\b(monarch_\w+)\s*\(([^)]*)\)\s*;", src, flags=re.M):
        plist = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        out[name] = (ret.strip(), plist)
    return out


def test_binding_signatures_match_the_header():
    protos = _prototypes()
    assert set(protos) == set(m._SIGS)
    for name, (ret, params) in protos.items():
        res, args = m._SIGS[name]
        assert _ctypes_kind(res) == _c_kind(ret), (name, ret, res)
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (a, p) in enumerate(zip(args, params)):
            assert _ctypes_kind(a) == _c_kind(_param_type(p)), (name, i, p, a)


def test_version(lib):
    assert lib.monarch_attn_version() >= 102


CFG1 = dict(B=1, heads=12, T=3, H=30, W=52, d=128, th=6, tw=4, iters=2, kv=4680, dt=1)


def _ws(c, **kw):
    c = {**c, **kw}
    return m.load_library().monarch_attn_workspace_bytes(c["B"], c["heads"], c["T"], c["H"], c["W"], c["d"],
                                                         c["th"], c["tw"], c["iters"], c["kv"], c["dt"])


def test_workspace_bytes_counts_the_intermediates(lib):
    total, offs = m.workspace_layout(1, 12, 3, 30, 52, 128, 6, 4, 2, 4680, 1)
    big = 12 * 24 * 195 * 128 * 4  # k~, z, q~: fp32 or two f16 planes
    assert offs[0] == 0 and offs[1] >= big and offs[2] - offs[1] >= big
    assert total >= 3 * big + 12 * 24 * 195 * 4 * 2
    assert total == _ws(CFG1)


@pytest.mark.parametrize("bad,needle", [
    (dict(H=31), "tile"),
    (dict(tw=5), "tile"),
    (dict(d=96), "head_dim"),
    (dict(iters=0), "iters"),
    (dict(kv=4681), "kv_len"),
    (dict(kv=3000), "kv_len"),
    (dict(dt=7), "dtype"),
    (dict(B=0), ">= 1"),
])
def test_invalid_arguments_are_rejected_on_the_host(lib, bad, needle):
    assert _ws(CFG1, **bad) == 0
    assert needle in lib.monarch_attn_last_error().decode()


def test_oversized_tile_is_unsupported(lib):
    assert _ws(CFG1, th=30, tw=52) == 0
    assert "exceeds" in lib.monarch_attn_last_error().decode()


def test_null_pointer_is_rejected_before_any_launch(lib):
    c = CFG1
    rc = lib.monarch_attn_fwd(None, None, None, None, c["B"], c["heads"], c["T"], c["H"], c["W"], c["d"],
                              c["th"], c["tw"], c["iters"], c["kv"], c["dt"], c["dt"], None)
    assert rc == -1
    assert "null" in lib.monarch_attn_last_error().decode()


def test_bad_output_dtype_is_rejected(lib):
    c = CFG1
    rc = lib.monarch_attn_fwd(0x1000, 0x2000, 0x3000, 0x4000, c["B"], c["heads"], c["T"], c["H"], c["W"],
                              c["d"], c["th"], c["tw"], c["iters"], c["kv"], 1, 2, None)
    assert rc == -1
    assert "out_dtype" in lib.monarch_attn_last_error().decode()


def test_misaligned_pointer_is_rejected(lib):
    c = CFG1
    rc = lib.monarch_attn_fwd(0x1008, 0x2000, 0x3000, 0x4000, c["B"], c["heads"], c["T"], c["H"], c["W"],
                              c["d"], c["th"], c["tw"], c["iters"], c["kv"], c["dt"], c["dt"], None)
    assert rc == -1
    assert "aligned" in lib.monarch_attn_last_error().decode()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "structured_sparse_attention_grid_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), f
                assert not any("oracle" in inc for inc in re.findall(r"#include.*", src)), f


def _bwd(lib, ptrs=(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000), **kw):
    c = dict(B=1, heads=2, T=3, H=8, W=12, d=64, th=2, tw=4, C=0, dt=1, gdt=0)
    c.update(kw)
    return lib.monarch_attn_bwd(*ptrs, c["B"], c["heads"], c["T"], c["H"], c["W"], c["d"], c["th"], c["tw"],
                                c["C"], c["dt"], c["gdt"], None)


@pytest.mark.parametrize("bad,needle", [
    (dict(H=9), "tile"),
    (dict(d=80), "head_dim"),
    (dict(gdt=2), "grad_dtype"),     # f16 gradients of bf16 inputs
    (dict(dt=5), "dtype"),
    (dict(C=-1), "chunk_frames"),
])
def test_backward_validates_on_the_host(lib, bad, needle):
    assert _bwd(lib, **bad) == -1
    assert needle in lib.monarch_attn_last_error().decode()


def test_backward_rejects_null_and_misaligned_pointers(lib):
    assert _bwd(lib, ptrs=(0x1000, 0x2000, 0x3000, None, 0x5000, 0x6000, 0x7000)) == -1
    assert "dy is null" in lib.monarch_attn_last_error().decode()
    assert _bwd(lib, ptrs=(0x1000, 0x2000, 0x3000, 0x4000, 0x5004, 0x6000, 0x7000)) == -1
    assert "dq is not 16-byte aligned" in lib.monarch_attn_last_error().decode()


def test_backward_workspace_holds_the_gradient_intermediates(lib):
    n = lib.monarch_attn_bwd_workspace_bytes(1, 12, 3, 30, 52, 128, 6, 4, 0, 1, 0)
    big = 12 * 24 * 195 * 128 * 4   # fp32 k~, z, dqL, dk~, dz
    assert n >= 5 * big + 4 * 12 * 24 * 195 * 4
    assert lib.monarch_attn_bwd_workspace_bytes(1, 12, 3, 30, 52, 128, 6, 4, 0, 1, 2) == 0


def test_lse_bytes_and_training_pair_validation(lib):
    # 12 heads x 24 positions x b1q = 195 rounded up to 196, float32
    assert lib.monarch_attn_lse_bytes(1, 12, 3, 30, 52, 128, 6, 4) == 12 * 24 * 196 * 4
    ptrs = (0x1000, 0x2000, 0x3000, 0x4000, 0x5000)
    assert lib.monarch_attn_fwd_train(*ptrs, 1, 2, 3, 8, 12, 64, 2, 4, 0, 0, None) == -4   # f32 inputs
    assert "bf16" in lib.monarch_attn_last_error().decode()
    assert lib.monarch_attn_fwd_train(*ptrs[:4], None, 1, 2, 3, 8, 12, 64, 2, 4, 0, 1, None) == -1
    assert "lse is null" in lib.monarch_attn_last_error().decode()
    bptrs = (0x1000, 0x2000, 0x3000, 0x4000, None, 0x6000, 0x7000, 0x8000, 0x9000)
    assert lib.monarch_attn_bwd_saved(*bptrs, 1, 2, 3, 8, 12, 64, 2, 4, 0, 1, 0, None) == -1
    assert "lse is null" in lib.monarch_attn_last_error().decode()
