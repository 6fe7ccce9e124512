"""C-ABI library: loads, exports every declared symbol, rejects bad arguments
on the host before touching a GPU (no compute calls here)."""

import ctypes
import os
import re

import pytest

from exact_attention_136_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("fa_fwd", "fa_fwd_fp8", "fa_fwd_host", "fa_device_status", "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(_lib.SIGNATURES), "binding misses a declared entry point"


def test_status_strings_and_version():
    assert _lib.status_string(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert _lib.status_string(code) != "unknown status"
    assert _lib.lib().fa_version().decode().count(".") == 2


# a fake, 16-byte aligned address: validation must reject before any use
A = 1 << 20
MIS = A + 8


def fwd(q=A, k=A, v=A, out=A, lse=None, B=1, nq=128, nk=128, H=1, D=64, scale=0.125, causal=0,
        wl=-1, dt=_lib.FA_FP16):
    return _lib.lib().fa_fwd(q, k, v, out, lse, B, nq, nk, H, D, scale, causal, wl, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), _lib.FA_ERR_ARG),
    (dict(k=None), _lib.FA_ERR_ARG),
    (dict(out=None), _lib.FA_ERR_ARG),
    (dict(B=0), _lib.FA_ERR_ARG),
    (dict(H=0), _lib.FA_ERR_ARG),
    (dict(nq=-1), _lib.FA_ERR_ARG),
    (dict(nk=-5), _lib.FA_ERR_ARG),
    (dict(scale=0.0), _lib.FA_ERR_ARG),
    (dict(scale=-1.0), _lib.FA_ERR_ARG),
    (dict(scale=float("inf")), _lib.FA_ERR_ARG),
    (dict(scale=float("nan")), _lib.FA_ERR_ARG),
    (dict(causal=2), _lib.FA_ERR_ARG),
    (dict(wl=-2), _lib.FA_ERR_ARG),
    (dict(dt=7), _lib.FA_ERR_ARG),
    (dict(D=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(D=256), _lib.FA_ERR_UNSUPPORTED),
    (dict(D=64, dt=_lib.FA_E4M3), _lib.FA_ERR_UNSUPPORTED),
    (dict(q=MIS), _lib.FA_ERR_ALIGN),
    (dict(v=MIS), _lib.FA_ERR_ALIGN),
    (dict(out=MIS), _lib.FA_ERR_ALIGN),
    (dict(B=1 << 16, H=1 << 8, nq=1 << 16), _lib.FA_ERR_ARG),
])
def test_invalid_arguments_rejected_on_host(kw, expect):
    assert fwd(**kw) == expect


def test_empty_query_is_a_no_op():
    # N_q = 0: nothing to compute, returns before touching the GPU
    assert fwd(nq=0) == _lib.FA_OK


def test_fp8_descales_validated():
    f = _lib.lib().fa_fwd_fp8
    assert f(A, A, A, A, None, 1, 128, 128, 1, 128, 0.1, 0, -1, 0.0, 1.0, 1.0, None) == _lib.FA_ERR_ARG
    assert f(A, A, A, A, None, 1, 128, 128, 1, 128, 0.1, 0, -1, 1.0, float("nan"), 1.0, None) == _lib.FA_ERR_ARG
    assert f(A, A, A, A, None, 1, 128, 128, 1, 64, 0.1, 0, -1, 1.0, 1.0, 1.0, None) == _lib.FA_ERR_UNSUPPORTED


def test_host_entry_rejects_null_host_buffers():
    f = _lib.lib().fa_fwd_host
    rc = f(None, A, A, A, None, A, A, A, A, None, 1, 128, 128, 1, 64, 0.1, 0, -1, 0, 1.0, 1.0, 1.0, None)
    assert rc == _lib.FA_ERR_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch
    from exact_attention_136_b200 import forward
    x = torch.zeros(1, 4, 1, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        forward(x, x, x)


@pytest.mark.parametrize("H, h_kv", [(8, 0), (8, 3), (6, 4), (4, 8), (8, -1)])
def test_gqa_head_counts_validated(H, h_kv):
    """H must be a positive multiple of H_kv; rejected on the host, before any GPU work."""
    f = _lib.lib().fa_fwd_gqa
    assert f(A, A, A, A, None, 1, 128, 128, H, h_kv, 128, 0.1, 0, -1, _lib.FA_BF16, 1.0, 1.0, 1.0,
             None) == _lib.FA_ERR_ARG


def test_gqa_descales_validated():
    f = _lib.lib().fa_fwd_gqa
    assert f(A, A, A, A, None, 1, 128, 128, 8, 2, 128, 0.1, 0, -1, _lib.FA_E4M3, 1.0, 0.0, 1.0,
             None) == _lib.FA_ERR_ARG


def test_splitkv_workspace_size():
    f = _lib.lib().fa_fwd_splitkv_workspace_bytes
    # one slice (or one key block): no workspace
    assert f(1, 16, 1024, 4, 128, 1) == 0
    assert f(1, 16, 100, 4, 128, 8) == 0
    # 8 key blocks in 4 slices of 2: 4 * B * N_q * H * (D + 1) floats
    assert f(2, 16, 1024, 4, 128, 4) == 4 * 2 * 16 * 4 * 129 * 4
    # more slices than key blocks: one slice per block
    assert f(1, 3, 1024, 2, 64, 100) == 8 * 1 * 3 * 2 * 65 * 4
    # 10 blocks in "4" slices of 3 -> 4 slices; in "6" slices of 2 -> 5 slices
    assert f(1, 1, 1280, 1, 64, 4) == 4 * 65 * 4
    assert f(1, 1, 1280, 1, 64, 6) == 5 * 65 * 4
    assert f(0, 1, 1280, 1, 64, 6) == 0 and f(1, 1, 1280, 1, 64, 0) == 0


@pytest.mark.parametrize("splits, ws, nbytes", [(0, A, 1 << 30), (4, None, 1 << 30), (4, A, 16), (4, A + 16, 1 << 30)])
def test_splitkv_arguments_validated(splits, ws, nbytes):
    """Slice count and workspace are checked on the host, before any GPU work."""
    f = _lib.lib().fa_fwd_splitkv
    assert f(A, A, A, A, None, 1, 16, 1024, 4, 4, 128, 0.1, 0, -1, _lib.FA_BF16, 1.0, 1.0, 1.0, splits, ws, nbytes,
             None) == _lib.FA_ERR_ARG


@pytest.mark.parametrize("kind, mask, sb, sh, sq", [
    (0, A, 0, 0, 128), (3, A, 0, 0, 128), (_lib.FA_MASK_BOOL, None, 0, 0, 128),
    (_lib.FA_MASK_BOOL, A + 8, 0, 0, 128), (_lib.FA_MASK_BOOL, A, 0, 0, 100),     # misaligned, short row
    (_lib.FA_MASK_BOOL, A, 0, 0, 136), (_lib.FA_MASK_ADD, A, 0, 4, 128),           # strides not 16 B
    (_lib.FA_MASK_ADD, A, -128, 0, 128)])
def test_mask_arguments_validated(kind, mask, sb, sh, sq):
    """Mask kind, pointer and strides are checked on the host, before any GPU work."""
    f = _lib.lib().fa_fwd_mask
    assert f(A, A, A, A, None, 1, 16, 128, 4, 4, 128, 0.1, 0, -1, _lib.FA_BF16, 1.0, 1.0, 1.0, mask, kind, sb, sh,
             sq, None) == _lib.FA_ERR_ARG


def test_backward_workspace_size():
    f = _lib.lib().fa_bwd_workspace_bytes
    # the fp32 row term rowsum(dO * O), [B, H, N_q]
    assert f(2, 300, 4, 128) == 2 * 300 * 4 * 4
    assert f(1, 0, 1, 64) == 0
    assert f(0, 10, 1, 64) == 0 and f(1, 10, 1, 96) == 0


def _bwd(**kw):
    args = dict(q=A, k=A, v=A, out=A, dout=A, lse=A, dq=A, dk=A, dv=A, B=1, N_q=16, N_k=16, H=2, D=64,
                scale=0.125, causal=0, window_left=-1, dtype=_lib.FA_FP16, ws=A, nbytes=1 << 20)
    args.update(kw)
    return _lib.lib().fa_bwd(args["q"], args["k"], args["v"], args["out"], args["dout"], args["lse"], args["dq"],
                             args["dk"], args["dv"], args["B"], args["N_q"], args["N_k"], args["H"], args["D"],
                             args["scale"], args["causal"], args["window_left"], args["dtype"], args["ws"],
                             args["nbytes"], None)


@pytest.mark.parametrize("kw, expect", [
    (dict(dtype=_lib.FA_E4M3, D=128), _lib.FA_ERR_UNSUPPORTED),
    (dict(D=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(dout=None), _lib.FA_ERR_ARG),
    (dict(lse=None), _lib.FA_ERR_ARG),
    (dict(dq=None), _lib.FA_ERR_ARG),
    (dict(dk=None), _lib.FA_ERR_ARG),
    (dict(ws=None), _lib.FA_ERR_ARG),
    (dict(nbytes=100), _lib.FA_ERR_ARG),
    (dict(ws=A + 16), _lib.FA_ERR_ARG),
    (dict(dq=A + 8), _lib.FA_ERR_ALIGN),
    (dict(lse=A + 2), _lib.FA_ERR_ALIGN),
    (dict(scale=0.0), _lib.FA_ERR_ARG),
    (dict(window_left=-2), _lib.FA_ERR_ARG),
])
def test_backward_arguments_validated(kw, expect):
    """Backward arguments are checked on the host, before any GPU work."""
    assert _bwd(**kw) == expect


@pytest.mark.parametrize("H, H_kv, expect", [(4, 3, _lib.FA_ERR_ARG), (4, 0, _lib.FA_ERR_ARG),
                                             (2, 4, _lib.FA_ERR_ARG), (4, 2, _lib.FA_ERR_UNSUPPORTED)])
def test_backward_gqa_heads_validated(H, H_kv, expect):
    """fa_bwd_gqa checks the head grouping before any GPU work (D = 96 makes a
    valid grouping stop at the head-dim check instead of launching)."""
    D = 96 if expect == _lib.FA_ERR_UNSUPPORTED else 64
    f = _lib.lib().fa_bwd_gqa
    assert f(A, A, A, A, A, A, A, A, A, 1, 16, 16, H, H_kv, D, 0.125, 0, -1, _lib.FA_FP16, A, 1 << 20,
             None) == expect


def _prototypes():
    """{name: number of parameters} for every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"^\s*(?:const\s+)?[\w\s\*]*?\b(fa_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.M | re.S):
        params = m.group(2).strip()
        protos[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_arities_match_the_header():
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    for name, count in protos.items():
        assert len(_lib.SIGNATURES[name][1]) == count, name


def test_header_is_plain_c(tmp_path):
    """include/fa.h compiles as strict C99 (the ABI has no C++ in it)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_fa.c"
    src.write_text('#include "fa.h"\nint main(void) { fa_stream_t s = 0; (void)s; return FA_OK; }\n')
    res = subprocess.run([cc, "-std=c99", "-pedantic", "-Wall", "-Werror", "-fsyntax-only",
                          "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_c_program_links_and_calls(tmp_path):
    """A plain C program links against libfa_b200.so and calls it: version and
    status strings, and argument errors, which are answered before any GPU
    work (so this runs without a GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    src = tmp_path / "call_fa.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "fa.h"
int main(void) {
  static float buf[64];   /* a 16-byte-aligned dummy pointer; never dereferenced */
  int bad_batch = fa_fwd(buf, buf, buf, buf, NULL, 0, 16, 16, 2, 64, 0.125f, 0, -1, FA_FP16, NULL);
  int bad_dim = fa_fwd(buf, buf, buf, buf, NULL, 1, 16, 16, 2, 96, 0.125f, 0, -1, FA_FP16, NULL);
  int bad_fp8 = fa_fwd_fp8(buf, buf, buf, buf, NULL, 1, 16, 16, 2, 128, 0.1f, 0, -1, 0.0f, 1.0f, 1.0f, NULL);
  printf("%s|%d|%d|%d|%s\n", fa_version(), bad_batch, bad_dim, bad_fp8, fa_status_string(FA_ERR_ARG));
  return 0;
}
""")
    exe = tmp_path / "call_fa"
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                          "-L", lib_dir, "-lfa_b200", "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    version, bad_batch, bad_dim, bad_fp8, msg = run.stdout.strip().split("|")
    assert version and msg
    assert int(bad_batch) == _lib.FA_ERR_ARG
    assert int(bad_dim) == _lib.FA_ERR_UNSUPPORTED
    assert int(bad_fp8) == _lib.FA_ERR_ARG   # zero descale


@pytest.mark.parametrize("kw, expect", [
    (dict(B=0), _lib.FA_ERR_ARG),
    (dict(cu_q=None), _lib.FA_ERR_ARG),
    (dict(cu_k=A + 2), _lib.FA_ERR_ARG),            # int32 arrays: 4-byte aligned
    (dict(max_q=0), _lib.FA_ERR_ARG),               # rows but no row per sequence
    (dict(max_q=5000), _lib.FA_ERR_ARG),            # longer than the packed rows
    (dict(max_k=9000), _lib.FA_ERR_ARG),
    (dict(D=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(H=3, H_kv=2), _lib.FA_ERR_ARG),
])
def test_varlen_arguments_validated(kw, expect):
    """fa_fwd_varlen checks its sizes and pointers on the host, before any GPU work."""
    a = dict(q=A, k=A, v=A, out=A, lse=None, cu_q=A, cu_k=A, B=2, max_q=100, max_k=100, total_q=150, total_k=150,
             H=2, H_kv=2, D=64, scale=0.1, causal=0, wl=-1, dt=_lib.FA_FP16)
    a.update(kw)
    f = _lib.lib().fa_fwd_varlen
    assert f(a["q"], a["k"], a["v"], a["out"], a["lse"], a["cu_q"], a["cu_k"], a["B"], a["max_q"], a["max_k"],
             a["total_q"], a["total_k"], a["H"], a["H_kv"], a["D"], a["scale"], a["causal"], a["wl"], a["dt"], 1.0,
             1.0, 1.0, None) == expect


@pytest.mark.parametrize("kw, expect", [
    (dict(wr=-2), _lib.FA_ERR_ARG),
    (dict(wr=-7, causal=1), _lib.FA_ERR_ARG),
    (dict(wl=-2, wr=3), _lib.FA_ERR_ARG),
    (dict(wr=5, D=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(nq=1 << 30, nk=1 << 30, wr=4), _lib.FA_ERR_ARG),   # i + window_right would leave int range
])
def test_window_arguments_validated(kw, expect):
    """fa_fwd_window / fa_bwd_window check the right window on the host, before any GPU work."""
    a = dict(nq=128, nk=128, H=1, H_kv=1, D=64, causal=0, wl=-1, wr=0)
    a.update(kw)
    f = _lib.lib().fa_fwd_window
    assert f(A, A, A, A, None, 1, a["nq"], a["nk"], a["H"], a["H_kv"], a["D"], 0.125, a["causal"], a["wl"], a["wr"],
             _lib.FA_FP16, 1.0, 1.0, 1.0, None) == expect
    g = _lib.lib().fa_bwd_window
    assert g(A, A, A, A, A, A, A, A, A, 1, a["nq"], a["nk"], a["H"], a["H_kv"], a["D"], 0.125, a["causal"], a["wl"],
             a["wr"], _lib.FA_FP16, A, 1 << 40, None) == expect


@pytest.mark.parametrize("kw, expect", [
    (dict(B=0), _lib.FA_ERR_ARG),
    (dict(cu_q=None), _lib.FA_ERR_ARG),
    (dict(cu_k=A + 2), _lib.FA_ERR_ARG),
    (dict(max_q=0), _lib.FA_ERR_ARG),               # rows but no launched query block
    (dict(max_k=0), _lib.FA_ERR_ARG),               # keys but no launched key block
    (dict(max_q=5000), _lib.FA_ERR_ARG),
    (dict(max_k=9000), _lib.FA_ERR_ARG),
    (dict(D=96), _lib.FA_ERR_UNSUPPORTED),
    (dict(dt=_lib.FA_E4M3, D=128), _lib.FA_ERR_UNSUPPORTED),
    (dict(H=3, H_kv=2), _lib.FA_ERR_ARG),
    (dict(ws_bytes=100), _lib.FA_ERR_ARG),           # workspace below H * total_q floats
])
def test_varlen_backward_arguments_validated(kw, expect):
    """fa_bwd_varlen checks its sizes and pointers on the host, before any GPU work."""
    a = dict(cu_q=A, cu_k=A, B=2, max_q=100, max_k=100, total_q=150, total_k=150, H=2, H_kv=2, D=64, causal=0,
             wl=-1, dt=_lib.FA_FP16, ws_bytes=1 << 20)
    a.update(kw)
    f = _lib.lib().fa_bwd_varlen
    assert f(A, A, A, A, A, A, A, A, A, a["cu_q"], a["cu_k"], a["B"], a["max_q"], a["max_k"], a["total_q"],
             a["total_k"], a["H"], a["H_kv"], a["D"], 0.1, a["causal"], a["wl"], a["dt"], A, a["ws_bytes"],
             None) == expect


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes structures of fa_fwd_args / fa_bwd_args have the C compiler's size and field offsets."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = []
    for cname, py in (("fa_fwd_args", _lib.FwdArgs), ("fa_bwd_args", _lib.BwdArgs)):
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in py._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"fa.h\"\nint main(void) {\n"
                   + "\n".join(lines) + "\n  return 0;\n}\n")
    exe = tmp_path / "layout"
    res = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o",
                          str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60).stdout.split("\n")
    got = {(ln.split()[0], ln.split()[1]): int(ln.split()[2]) for ln in out if ln.strip()}
    for cname, py in (("fa_fwd_args", _lib.FwdArgs), ("fa_bwd_args", _lib.BwdArgs)):
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for field, _ in py._fields_:
            assert got[(cname, field)] == getattr(py, field).offset, (cname, field)


@pytest.mark.parametrize("kw, expect", [
    (dict(cu_q=A), _lib.FA_ERR_ARG),                 # one of the two packed-batch pointers
    (dict(wr=-2), _lib.FA_ERR_ARG),
    (dict(p=1.0), _lib.FA_ERR_ARG),
    (dict(p=0.1, dt=_lib.FA_E4M3, D=128), _lib.FA_ERR_UNSUPPORTED),
    (dict(cu_q=A, cu_k=A, total_q=150, total_k=150, Nq=0), _lib.FA_ERR_ARG),   # packed rows, no launched block
    (dict(D=96), _lib.FA_ERR_UNSUPPORTED),
])
def test_struct_entry_points_validated(kw, expect):
    """fa_fwd_ex / fa_bwd_ex check their arguments on the host, before any GPU work."""
    a = dict(B=2, Nq=100, Nk=100, H=2, D=64, wl=-1, wr=3, dt=_lib.FA_FP16, p=0.0, cu_q=None, cu_k=None,
             total_q=0, total_k=0)
    a.update(kw)
    f = _lib.FwdArgs(q=A, k=A, v=A, out=A, lse=None, B=a["B"], N_q=a["Nq"], N_k=a["Nk"], H=a["H"], H_kv=a["H"],
                     D=a["D"], scale=0.1, causal=0, window_left=a["wl"], window_right=a["wr"], dtype=a["dt"],
                     q_descale=1.0, k_descale=1.0, v_descale=1.0, cu_seqlens_q=a["cu_q"], cu_seqlens_k=a["cu_k"],
                     total_q=a["total_q"], total_k=a["total_k"], dropout_p=a["p"], seed=1, offset=0)
    assert _lib.lib().fa_fwd_ex(ctypes.byref(f), None) == expect
    b = _lib.BwdArgs(q=A, k=A, v=A, out=A, dout=A, lse=A, dq=A, dk=A, dv=A, B=a["B"], N_q=a["Nq"], N_k=a["Nk"],
                     H=a["H"], H_kv=a["H"], D=a["D"], scale=0.1, causal=0, window_left=a["wl"],
                     window_right=a["wr"], dtype=a["dt"], cu_seqlens_q=a["cu_q"], cu_seqlens_k=a["cu_k"],
                     total_q=a["total_q"], total_k=a["total_k"], dropout_p=a["p"], seed=1, offset=0, workspace=A,
                     workspace_bytes=1 << 30)
    assert _lib.lib().fa_bwd_ex(ctypes.byref(b), None) == expect
    assert _lib.lib().fa_fwd_ex(None, None) == _lib.FA_ERR_ARG
