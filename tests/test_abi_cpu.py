"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/chipmunk.h declares, and rejects bad arguments
before touching a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "chipmunk.h")


@pytest.fixture(scope="module")
def cm():
    import torch  # noqa: F401  (loads the CUDA runtime the library links against)
    from dynamic_column_sparse_b200 import build, chipmunk
    build.build()
    return chipmunk


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:[A-Za-z_][\w \*]*?)\b(chipmunk_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("chipmunk_topk_cols", "chipmunk_mlp_delta", "chipmunk_attn_delta", "chipmunk_dense_refresh"):
        assert required in names


def test_library_exports_every_declared_symbol(cm):
    lib = cm.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(cm.EXPORTS) <= set(declared_functions())


def test_struct_layouts_match_the_header(cm, tmp_path):
    """Every field of the ctypes structs sits where a C compiler puts it for include/chipmunk.h."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    structs = {"chipmunk_mlp_args": cm.MlpArgs, "chipmunk_attn_args": cm.AttnArgs,
               "chipmunk_refresh_args": cm.RefreshArgs, "chipmunk_mlp_fp8_args": cm.MlpFp8Args}
    lines = ["#include <stddef.h>", "#include <stdio.h>", "#include \"chipmunk.h\"", "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run([gcc, "-I", inc, str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        cname, field, val = line.split()
        got[(cname, field)] = int(val)
    for cname, py in structs.items():
        assert got[(cname, "sizeof")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_version_and_status_strings(cm):
    lib = cm.load_library()
    assert cm.version() == "0.1.0"
    for st in range(8):
        assert lib.chipmunk_status_string(st)
    assert b"unknown" in lib.chipmunk_status_string(99)


def _mlp_args(cm, **kw):
    base = dict(T=256, D=128, H=512, Bt=64, k=128, x=0x1000, w1t=0x2000, b1=0x3000, w2=0x4000, b2=0x5000,
                idx=0x6000, a_cache=0x7000, y_cache=0x8000, out=0)
    base.update(kw)
    return cm.MlpArgs(**base)


@pytest.mark.parametrize("field,value,status", [
    ("D", 100, 2), ("D", 0, 2), ("Bt", 32, 2), ("k", 513, 1), ("k", -1, 1), ("T", 0, 2),
    ("x", 0, 1), ("w1t", 0x2008, 3), ("y_cache", 0, 1),
])
def test_mlp_delta_rejects_bad_arguments_on_the_host(cm, field, value, status):
    lib = cm.load_library()
    a = _mlp_args(cm, **{field: value})
    st = lib.chipmunk_mlp_delta(ctypes.byref(a), None, 0, None)
    assert st == status, lib.chipmunk_last_error()
    assert lib.chipmunk_last_error()


def test_mlp_delta_requires_workspace(cm):
    lib = cm.load_library()
    a = _mlp_args(cm)
    need = lib.chipmunk_workspace_bytes(cm.OP_MLP_DELTA, ctypes.byref(a))
    assert need == 4 * 128 * 64 * 2  # nb * round_up(k,128) * Bt bf16
    st = lib.chipmunk_mlp_delta(ctypes.byref(a), None, 0, None)
    assert st == 7


@pytest.mark.parametrize("field,value,status", [("d", 64, 2), ("Bt", 64, 2), ("k", 301, 1), ("h", 0, 2), ("q", 0, 1)])
def test_attn_delta_rejects_bad_arguments_on_the_host(cm, field, value, status):
    lib = cm.load_library()
    base = dict(T=300, h=2, d=128, Bt=128, k=40, scale=0.088, q=0x1000, kk=0x2000, v=0x3000, idx=0x4000,
                m_c=0x5000, l_c=0x6000, acc_c=0x7000, o=0x8000)
    base[field] = value
    a = cm.AttnArgs(**base)
    assert lib.chipmunk_attn_delta(ctypes.byref(a), None, 0, None) == status


def test_topk_rejects_bad_arguments_on_the_host(cm):
    lib = cm.load_library()
    assert lib.chipmunk_topk_cols(ctypes.c_void_p(0x1000), 4, 10, 10, 11, ctypes.c_void_p(0x2000), 11, None, 0, None) == 1
    assert lib.chipmunk_topk_cols(ctypes.c_void_p(0x1000), 4, 10, 9, 3, ctypes.c_void_p(0x2000), 3, None, 0, None) == 2
    assert lib.chipmunk_topk_cols(ctypes.c_void_p(0x1004), 4, 10, 10, 3, ctypes.c_void_p(0x2000), 3, None, 0, None) == 3
    # nothing to do is not an error
    assert lib.chipmunk_topk_cols(None, 0, 10, 10, 3, None, 3, None, 0, None) == 0
    assert lib.chipmunk_topk_cols(None, 4, 10, 10, 0, None, 0, None, 0, None) == 0


def test_refresh_rejects_unknown_kind(cm):
    lib = cm.load_library()
    r = cm.RefreshArgs(kind=7, scores=0x1000)
    assert lib.chipmunk_dense_refresh(ctypes.byref(r), None, 0, None) == 1
    r = cm.RefreshArgs(kind=cm.REFRESH_MLP, scores=0)
    assert lib.chipmunk_dense_refresh(ctypes.byref(r), None, 0, None) == cm.ERR_INVALID_ARG  # the MLP needs scores
    r = cm.RefreshArgs(kind=cm.REFRESH_ATTN, scores=0)
    assert lib.chipmunk_dense_refresh(ctypes.byref(r), None, 0, None) == cm.ERR_SHAPE        # T = 0


def _attn_refresh_args(cm, T, h, k, scores):
    p = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)]
    a = cm.AttnArgs(T, h, 128, 128, k, 0.088, p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7])
    return cm.RefreshArgs(cm.REFRESH_ATTN, 0, cm.MlpArgs(), a, scores)


def test_attn_refresh_workspace_without_a_mass_tensor(cm):
    """Without a mass tensor the refresh needs the row log-sum-exp plus the fused mass/top-k kernel's row
    buffers (at least one row of round_up(T, 32) fp32, from a 128-byte boundary); with one, the
    log-sum-exp only. Too small a workspace is rejected on the host."""
    lib = cm.load_library()
    T, h, k = 1001, 3, 165
    kept = cm.workspace_bytes(cm.OP_REFRESH, _attn_refresh_args(cm, T, h, k, 0x20000000))
    fused = cm.workspace_bytes(cm.OP_REFRESH, _attn_refresh_args(cm, T, h, k, None))
    assert kept == (h * T * 4 + 255) // 256 * 256
    row_bytes = (T + 31) // 32 * 128
    rows = (fused - kept - 128) // row_bytes
    assert fused - kept == 128 + rows * row_bytes and 1 <= rows <= h * ((T + 127) // 128)
    assert cm.attn_refresh_workspace_bytes(T, h, k, False) == fused
    assert cm.attn_refresh_workspace_bytes(T, h, k, True) == kept
    r = _attn_refresh_args(cm, T, h, k, None)
    ws = ctypes.c_void_p(0x40000000)
    assert lib.chipmunk_dense_refresh(ctypes.byref(r), ws, fused - 16, None) == cm.ERR_WORKSPACE
    r = _attn_refresh_args(cm, T, h, k, 0x20000004)
    assert lib.chipmunk_dense_refresh(ctypes.byref(r), ws, kept, None) == cm.ERR_ALIGNMENT   # scores misaligned


def test_noalloc_rejects_requests_beyond_its_scratch(cm):
    """The size check of the no-alloc entry point runs on the host, before any device call."""
    lib = cm.load_library()
    # nb * round_up(k,128) * Bt * 2 = 600 * 1024 * 128 * 2 bytes > 64 MiB
    a = _mlp_args(cm, T=600 * 128, D=128, H=1024, Bt=128, k=1024, b2=0)
    assert 600 * 1024 * 128 * 2 > cm.NOALLOC_SCRATCH_BYTES
    assert lib.chipmunk_mlp_delta_noalloc(ctypes.byref(a), None) == cm.ERR_WORKSPACE
    assert b"scratch" in lib.chipmunk_last_error()


def test_status_constants_match_the_header(cm):
    text = open(HEADER).read()
    for name in ("OK", "ERR_INVALID_ARG", "ERR_SHAPE", "ERR_ALIGNMENT", "ERR_CUDA", "ERR_DEVICE", "ERR_UNSUPPORTED",
                 "ERR_WORKSPACE"):
        m = re.search(rf"#define CHIPMUNK_{name}\s+(\d+)", text)
        assert m and int(m.group(1)) == getattr(cm, name), name
    m = re.search(r"#define CHIPMUNK_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", text)
    assert m and (int(m.group(1)) << int(m.group(2))) == cm.NOALLOC_SCRATCH_BYTES


def _fp8_args(cm, **kw):
    base = dict(T=300, D=256, H=700, Bt=128, k=128, x8=0x1000, sx=0x2000, w1t8=0x3000, s1=0x4000, b1=0x5000,
                w2_8=0x6000, g2=0x7000, s_delta=1e-4, idx=0x8000, a_cache=0x9000, y_cache=0xa000, out=0)
    base.update(kw)
    return cm.MlpFp8Args(**base)


@pytest.mark.parametrize("field,value,status", [
    ("D", 128, "ERR_SHAPE"), ("D", 384, "ERR_SHAPE"), ("Bt", 64, "ERR_SHAPE"), ("k", 701, "ERR_INVALID_ARG"),
    ("s_delta", 0.0, "ERR_INVALID_ARG"), ("s_delta", -1.0, "ERR_INVALID_ARG"), ("sx", 0, "ERR_INVALID_ARG"),
    ("g2", 0x7004, "ERR_ALIGNMENT"),
])
def test_mlp_delta_fp8_rejects_bad_arguments_on_the_host(cm, field, value, status):
    lib = cm.load_library()
    a = _fp8_args(cm, **{field: value})
    assert lib.chipmunk_mlp_delta_fp8(ctypes.byref(a), None, 0, None) == getattr(cm, status), lib.chipmunk_last_error()


def test_mlp_delta_fp8_workspace(cm):
    lib = cm.load_library()
    a = _fp8_args(cm)
    assert lib.chipmunk_workspace_bytes(cm.OP_MLP_DELTA_FP8, ctypes.byref(a)) == 3 * 128 * 128   # one byte per delta
    assert lib.chipmunk_mlp_delta_fp8(ctypes.byref(a), None, 0, None) == cm.ERR_WORKSPACE


def test_quantize_rejects_bad_arguments_on_the_host(cm):
    lib = cm.load_library()
    q = lib.chipmunk_quantize_e4m3_rows
    assert q(ctypes.c_void_p(0x1000), 4, 24, ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), None) == cm.ERR_SHAPE
    assert q(ctypes.c_void_p(0x1008), 4, 32, ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), None) == cm.ERR_ALIGNMENT
    assert q(None, 4, 32, ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), None) == cm.ERR_INVALID_ARG
    assert q(None, 0, 32, None, None, None) == cm.OK
