"""The C ABI library loads, exports every declared entry point, and rejects
bad arguments on the host (no GPU needed; no compute is launched)."""

import ctypes
import os
import re

import pytest

from long_context_mean_b200 import sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_attn.h")


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(sa.LIB_PATH):
        from long_context_mean_b200 import build
        build.build()
    return sa.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sa.EXPORTS)


def test_version(lib):
    assert "sm_100a" in sa.version()


def test_missing_library_fails_loudly(tmp_path):
    saved = sa._lib
    try:
        sa._lib = None
        with pytest.raises(RuntimeError, match="no fallback"):
            sa.load(str(tmp_path / "nope.so"))
    finally:
        sa._lib = saved


FAKE = ctypes.c_void_p(4096)


def _shape(**kw):
    base = dict(B=1, Hq=2, Hkv=2, N=300, d=128, dv=128, dtype=sa.SA_BF16)
    base.update(kw)
    return sa.Shape(base["B"], base["Hq"], base["Hkv"], base["N"], base["d"], base["dv"], base["dtype"], 0)


def _mask():
    return sa.Mask(4096, 4096, 4096, 4096, 4096, 4096, 100, 0, 0, 0, 0, 0, 0)


def test_host_validation_codes(lib):
    s = _shape()
    p = sa.make_params(128, 64, 0.5)
    null = ctypes.c_void_p(None)
    m = _mask()
    # layout
    bad = sa.make_layout(0, 4, 4)
    assert lib.sa_layout_build(ctypes.byref(bad), FAKE, FAKE, null, 0, null) == sa.SA_ERR_INVALID_ARG
    big = sa.make_layout(3, 1000, 4, mode="hilbert")
    assert lib.sa_layout_build(ctypes.byref(big), FAKE, FAKE, null, 0, null) == sa.SA_ERR_UNSUPPORTED
    hil = sa.make_layout(5, 8, 8, mode="hilbert")
    assert lib.sa_layout_build(ctypes.byref(hil), FAKE, FAKE, null, 0, null) == sa.SA_ERR_WORKSPACE
    # reorder
    assert lib.sa_reorder(FAKE, FAKE, FAKE, 1, 10, 128, 0, null) == sa.SA_ERR_INVALID_ARG  # in place
    assert lib.sa_reorder(null, FAKE, ctypes.c_void_p(8192), 1, 10, 128, 0, null) == sa.SA_ERR_INVALID_ARG
    # predict
    p_bad = sa.make_params(128, 64, 0.0)
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s), ctypes.byref(p_bad), FAKE, 1 << 30,
                               ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    p_blk = sa.make_params(256, 64, 0.5)
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s), ctypes.byref(p_blk), FAKE, 1 << 30,
                               ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    s_d = _shape(d=96)
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s_d), ctypes.byref(p), FAKE, 1 << 30,
                               ctypes.byref(m), null) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s), ctypes.byref(p), FAKE, 16,
                               ctypes.byref(m), null) == sa.SA_ERR_WORKSPACE
    s_g = _shape(Hq=3, Hkv=2)
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s_g), ctypes.byref(p), FAKE, 1 << 30,
                               ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    # fused reorder + predict: perm and the copies must be given and must not overlap the inputs
    QR, KR = ctypes.c_void_p(1 << 30), ctypes.c_void_p(1 << 31)
    assert lib.sa_reorder_predict_mask(null, FAKE, FAKE, QR, KR, ctypes.byref(s), ctypes.byref(p), FAKE, 1 << 30,
                                       ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_reorder_predict_mask(FAKE, FAKE, ctypes.c_void_p(1 << 20), FAKE, KR, ctypes.byref(s),
                                       ctypes.byref(p), FAKE, 1 << 30, ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    # attention
    m2 = _mask()
    m2.bq, m2.bk, m2.nqb, m2.nkb = 128, 64, 3, 5
    WS = ctypes.c_void_p(1 << 20)
    assert lib.sa_block_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), ctypes.byref(m2), ctypes.c_float(0.5),
                                    ctypes.c_float(0), FAKE, null, null, null, WS, 256, 0, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), ctypes.byref(m2), ctypes.c_float(-1),
                                    ctypes.c_float(0), FAKE, null, null, null, null, 0, 0, null) == sa.SA_ERR_WORKSPACE
    m2.nqb = 4   # wrong for N=300, bq=128
    assert lib.sa_block_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), ctypes.byref(m2), ctypes.c_float(-1),
                                    ctypes.c_float(0), FAKE, null, null, null, WS, 256, 0, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_dense_attn(FAKE, FAKE, FAKE, ctypes.byref(s), 2, ctypes.c_float(0), FAKE, null, null, WS, 256,
                             0, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_read_status(null, null) == sa.SA_ERR_INVALID_ARG
    assert b"status" in lib.sa_last_error()
    # per-head placement, per-head reorder, sampled-row error
    assert lib.sa_head_placement(0, 2, 2, 0, FAKE, 2, 4, 4, FAKE, FAKE, null, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_head_placement(2, 2, 2, 0, null, 2, 4, 4, FAKE, FAKE, null, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_head_placement(2, 2, 2, 0, FAKE, 2, 0, 4, FAKE, FAKE, null, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_reorder_heads(FAKE, FAKE, ctypes.c_void_p(4096 + 64), 2, 10, 8, 0, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_reorder_heads(null, FAKE, ctypes.c_void_p(1 << 20), 2, 10, 8, 0, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_rows_mse(FAKE, FAKE, FAKE, 4, 2, 10, 8, 7, FAKE, null, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_rows_mse(FAKE, FAKE, null, 4, 2, 10, 8, 0, FAKE, null, null) == sa.SA_ERR_INVALID_ARG
    # 8-bit QK
    assert lib.sa_quantize_blocks(null, 2, 10, 128, 64, 0, 0, FAKE, FAKE, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_quantize_blocks(FAKE, 2, 10, 128, 64, 1, 0, FAKE, FAKE, null) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_quantize_blocks(FAKE, 2, 10, 128, 256, 0, 0, FAKE, FAKE, null) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_quantize_blocks(FAKE, 2, 10, 128, 64, 0, 5, FAKE, FAKE, null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_attn_qk8_workspace(None) == 0
    m3 = _mask()
    m3.bq, m3.bk, m3.nqb, m3.nkb, m3.col_capacity = 128, 64, 3, 5, 15
    assert lib.sa_attn_qk8_workspace(ctypes.byref(m3)) == 256 + 256
    WS8 = ctypes.c_void_p(1 << 21)
    assert lib.sa_block_sparse_attn_qk8(FAKE, FAKE, FAKE, FAKE, 0, FAKE, ctypes.byref(s), None, ctypes.c_float(-1),
                                        ctypes.c_float(0), FAKE, null, null, null, WS8, 512, 0,
                                        null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_sparse_attn_qk8(FAKE, FAKE, FAKE, FAKE, 0, FAKE, ctypes.byref(s), ctypes.byref(m3),
                                        ctypes.c_float(-1), ctypes.c_float(0), FAKE, null, null, null, WS8, 256, 0,
                                        null) == sa.SA_ERR_WORKSPACE
    assert lib.sa_block_sparse_attn_qk8(FAKE, null, FAKE, FAKE, 0, FAKE, ctypes.byref(s), ctypes.byref(m3),
                                        ctypes.c_float(-1), ctypes.c_float(0), FAKE, null, null, null, WS8, 512, 0,
                                        null) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_block_sparse_attn_qk8(FAKE, FAKE, FAKE, FAKE, 0, FAKE, ctypes.byref(s), ctypes.byref(m3),
                                        ctypes.c_float(-1), ctypes.c_float(0), FAKE, null, null, null, WS8, 512,
                                        sa.SA_FLAG_FORCE_SIMT, null) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_block_sparse_attn_qk8(FAKE, FAKE, FAKE, FAKE, 9, FAKE, ctypes.byref(s), ctypes.byref(m3),
                                        ctypes.c_float(-1), ctypes.c_float(0), FAKE, null, null, null, WS8, 512, 0,
                                        null) == sa.SA_ERR_INVALID_ARG
    # a per-head output permutation needs out_perm
    m2.nqb = 3
    assert lib.sa_block_sparse_attn(FAKE, FAKE, FAKE, ctypes.byref(s), ctypes.byref(m2), ctypes.c_float(-1),
                                    ctypes.c_float(0), FAKE, null, null, null, WS, 256,
                                    sa.SA_FLAG_OUT_PERM_PER_HEAD, null) == sa.SA_ERR_INVALID_ARG


def test_q8_scale_arrays_are_checked(lib):
    """sa_reorder_predict_mask_q8 rejects misaligned or overlapping scale
    arrays on the host with their own message."""
    null = ctypes.c_void_p(None)
    s = sa.Shape(1, 2, 1, 1024, 128, 128, sa.SA_BF16, 0)
    pr = sa.make_params(128, 64, 0.5)
    m = _mask()
    q, k = ctypes.c_void_p(1 << 24), ctypes.c_void_p(1 << 25)
    q8, k8 = ctypes.c_void_p(1 << 26), ctypes.c_void_p(1 << 27)
    qs, ks = ctypes.c_void_p(1 << 28), ctypes.c_void_p((1 << 28) + 4096)
    ws = ctypes.c_void_p(1 << 29)
    call = lambda qs_, ks_: lib.sa_reorder_predict_mask_q8(null, q, k, 0, q8, qs_, k8, ks_, ctypes.byref(s),
                                                          ctypes.byref(pr), ws, 1 << 20, ctypes.byref(m), null)
    assert call(ctypes.c_void_p((1 << 28) + 2), ks) == sa.SA_ERR_INVALID_ARG
    assert b"q_scales and k_scales must be 4-byte aligned" in lib.sa_last_error()
    # q_scales (2 heads x 8 blocks = 64 bytes) inside q
    assert call(ctypes.c_void_p((1 << 24) + 64), ks) == sa.SA_ERR_INVALID_ARG
    assert b"q_scales and k_scales" in lib.sa_last_error()
    # k_scales overlapping q_scales, and inside the workspace
    assert call(qs, ctypes.c_void_p((1 << 28) + 32)) == sa.SA_ERR_INVALID_ARG
    assert call(qs, ctypes.c_void_p((1 << 29) + 256)) == sa.SA_ERR_INVALID_ARG
    assert b"workspace" in lib.sa_last_error()


def test_forward_host_validation(lib):
    """sa_forward_host checks its arguments on the host before enqueueing:
    NULL buffers, a chunk count that does not divide B*Hkv, a shape whose N
    differs from the layout's tokens, an undersized workspace."""
    null = ctypes.c_void_p(None)
    s = sa.Shape(1, 4, 2, 64, 128, 128, sa.SA_BF16, 0)
    lay = sa.make_layout(4, 4, 4, 0, 0, "window", (2, 2, 2))
    pr = sa.make_params(16, 16, 0.5)
    assert lib.sa_forward_host_workspace(ctypes.byref(s), ctypes.byref(lay), ctypes.byref(pr), 3) == 0
    need = lib.sa_forward_host_workspace(ctypes.byref(s), ctypes.byref(lay), ctypes.byref(pr), 2)
    assert need > 0 and need % 256 == 0
    # one chunk holds the whole problem: at least the device copies of q, k, v, out (4 x 16 KB x heads)
    one = lib.sa_forward_host_workspace(ctypes.byref(s), ctypes.byref(lay), ctypes.byref(pr), 1)
    assert one >= (4 + 2 + 2 + 4) * 64 * 128 * 2
    st = (ctypes.c_void_p * 3)(None, None, None)
    H = ctypes.c_void_p(1 << 30)
    WS = ctypes.c_void_p(1 << 31)
    call = lambda q, shape, lay_, chunks, ws_bytes: lib.sa_forward_host(
        q, H, H, H, H, ctypes.byref(shape), ctypes.byref(lay_), ctypes.byref(pr), ctypes.c_float(-1.0),
        ctypes.c_float(0.0), chunks, WS, ws_bytes, FAKE, ctypes.byref(st))
    assert call(null, s, lay, 2, need) == sa.SA_ERR_INVALID_ARG
    assert call(H, s, lay, 3, need) == sa.SA_ERR_INVALID_ARG
    assert b"chunks" in lib.sa_last_error()
    s_bad = sa.Shape(1, 4, 2, 65, 128, 128, sa.SA_BF16, 0)
    assert call(H, s_bad, lay, 2, need) == sa.SA_ERR_INVALID_ARG
    assert call(H, s, lay, 2, need - 256) == sa.SA_ERR_WORKSPACE


def test_workspace_queries_are_host_only(lib):
    s = _shape(N=20506, Hq=24, Hkv=24)
    p = sa.make_params(128, 64, 0.5)
    off = sa.predict_mask_ws_layout(s, p)
    nqb, nkb = -(-20506 // 128), -(-20506 // 64)
    assert off[0] == 0 and off[1] >= 24 * nqb * 128 * 4
    assert sa.predict_mask_workspace(s, p) >= off[5] + 24 * nqb * 4
    assert all(o % 256 == 0 for o in off)
    assert sa.layout_workspace(sa.make_layout(21, 45, 80, 0, 1, "hilbert")) >= 2 * (1 << 21) // 8
    assert sa.layout_workspace(sa.make_layout(13, 30, 52, 226, 1, "window", (2, 8, 8))) == 0


def test_order_group_hint_and_check(lib):
    # K and V of one KV head under 32 MiB: one global order (image, video)
    assert sa.order_group_hint(_shape(B=2, Hq=24, Hkv=24, N=4096)) == 0
    assert sa.order_group_hint(_shape(Hq=24, Hkv=24, N=20506)) == 0
    # 38.7 MB per head: two heads (77 MB) fit in 96 MiB, four do not
    assert sa.order_group_hint(_shape(Hq=24, Hkv=24, N=75600)) == 2
    # GQA 32/8 at 131072: one KV head (67 MB) serves 4 query heads
    assert sa.order_group_hint(_shape(Hq=32, Hkv=8, N=131072)) == 4
    assert lib.sa_order_group_hint(ctypes.byref(_shape(Hq=3, Hkv=2))) == -1
    p = sa.make_params(128, 64, 0.5, order_group=-1)
    s, m, null = _shape(), _mask(), ctypes.c_void_p(None)
    assert lib.sa_predict_mask(FAKE, FAKE, ctypes.byref(s), ctypes.byref(p), FAKE, 1 << 30,
                               ctypes.byref(m), null) == sa.SA_ERR_INVALID_ARG
    assert b"order_group" in lib.sa_last_error()


def test_kernel_path_selection(lib):
    s = _shape()
    assert sa.attn_kernel_path(s, 128, 64, sa.SA_FLAG_FORCE_SIMT) == 0
    s32 = _shape(dtype=sa.SA_FP32, d=16, dv=16)
    assert sa.attn_kernel_path(s32, 16, 16) == 0
    assert sa.attn_kernel_path(s, 129, 64) == -1


def _declarations():
    """name -> list of parameter type strings, from the header's prototypes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(?:sa_status|size_t|int32_t|const char\*)\s+(sa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        # drop the parameter name; an array parameter (size_t offsets[6]) is a pointer
        out[m.group(1)] = [p.rsplit(None, 1)[0] + ("*" if "[" in p else "") for p in params]
    return out


def _category(ctype_param):
    """Compare a header parameter type with a ctypes argtype by kind and width."""
    if "*" in ctype_param:
        return "pointer"
    base = ctype_param.replace("const", "").strip()
    return {"int32_t": "i32", "int64_t": "i64", "size_t": "size", "float": "f32"}[base]


def _ctypes_category(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    return {ctypes.c_int32: "i32", ctypes.c_int64: "i64", ctypes.c_size_t: "size", ctypes.c_float: "f32"}[t]


def test_binding_signatures_match_the_header(lib):
    """Every ctypes argtype list has the header's parameter count and kinds
    (pointer, int32, int64, size_t, float), so a changed prototype cannot
    silently shift the arguments of a call."""
    decls = _declarations()
    assert set(decls) == set(sa.EXPORTS)
    for name, params in decls.items():
        argtypes = getattr(lib, name).argtypes or []
        assert len(argtypes) == len(params), (name, params, argtypes)
        for p, t in zip(params, argtypes):
            assert _category(p) == _ctypes_category(t), (name, p, t)


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99 and as C++."""
    import shutil
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "sparse_attn.h"\nint main(void) { return (int)sizeof(sa_shape) == 0; }\n')
    inc = os.path.dirname(HEADER)
    for comp, flags in (("gcc", ["-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror"]),
                        ("g++", ["-std=c++17", "-Wall", "-Werror", "-x", "c++"])):
        if shutil.which(comp) is None:
            pytest.skip(f"{comp} not installed")
        r = subprocess.run([comp, *flags, "-fsyntax-only", "-I", inc, str(src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_binding_return_types_match_the_header(lib):
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    kinds = {"sa_status": ctypes.c_int32, "size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32,
             "const char*": ctypes.c_char_p}
    found = re.findall(r"\b(sa_status|size_t|int32_t|const char\*)\s+(sa_[a-z0-9_]+)\s*\(", text)
    assert {n for _, n in found} == set(sa.EXPORTS)
    for ret, name in found:
        assert getattr(lib, name).restype is kinds[ret], (name, ret)


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "sparse_attn.h"

int main(void) {
  sa_shape s = {1, 2, 2, 300, 128, 128, SA_BF16, 0};
  sa_mask_params p;
  memset(&p, 0, sizeof p);
  p.bq = 128; p.bk = 64; p.tau = 0.5f; p.theta = 0.0f;
  if (strstr(sa_version(), "sm_100a") == NULL) return 10;
  if (sa_attn_workspace() == 0) return 11;
  if (sa_predict_mask_workspace(&s, &p) == 0) return 12;
  /* argument errors are reported before anything touches a device */
  if (sa_reorder(NULL, (void*)4096, (void*)8192, 1, 10, 128, SA_BF16, NULL) != SA_ERR_INVALID_ARG) return 13;
  if (sa_read_status(NULL, NULL) != SA_ERR_INVALID_ARG) return 14;
  if (sa_last_error()[0] == '\0') return 15;
  printf("c client ok\n");
  return 0;
}
"""


def test_plain_c_client_links_and_calls(tmp_path):
    """A C program (no Python, no torch) includes the header, links the
    shared library and gets its host-side answers."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not installed")
    if not os.path.exists(sa.LIB_PATH):
        from long_context_mean_b200 import build
        build.build()
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(sa.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                        "-L", libdir, "-l:libsparseattn.so", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c client ok" in run.stdout, (run.returncode, run.stdout, run.stderr)
