"""CPU checks of the C-ABI library: it builds for sm_100a, loads without a GPU, exports
every function include/hifa4.h declares, and its host-side validation rejects bad
arguments before any device work."""
import ctypes

import numpy as np
import pytest

from bit_flashattention_b200 import build, hifa4
from tests import _layout


@pytest.fixture(scope="module")
def L():
    build.build()
    return hifa4.lib()


def test_exports_every_declared_symbol(L):
    names = hifa4.declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n


def test_test_hooks_only_in_the_test_library(L):
    # the product library carries no probe and no fault injection; the test library holds
    # the product ABI plus every function include/hifa4_test.h declares
    from bit_flashattention_b200 import hifa4_testhooks as th
    T = th.lib()
    hooks = th.declared_functions()
    assert set(hooks) >= {"hifa4_test_attn_fwd_inject", "hifa4_probe_codec", "hifa4_probe_qk_tile",
                          "hifa4_probe_pv_tile"}
    for n in hooks:
        assert hasattr(T, n), n
        assert not hasattr(L, n), n
    for n in hifa4.declared_functions():
        assert hasattr(T, n), n
    assert not hasattr(L, "hifa4_debug_set_injection")


def test_status_strings(L):
    for code in range(7):
        assert hifa4.status_string(code).startswith("HIFA4_")
    assert hifa4.status_string(99) == "HIFA4_ERR_UNKNOWN"


def test_size_helpers(L):
    assert L.hifa4_qtensor_codes_bytes(1, 32, 4096, 128) == 32 * 4096 * 64
    assert L.hifa4_qtensor_scales_bytes(1, 32, 4096, 128, 0) == 32 * 4096 * 8
    assert L.hifa4_qtensor_scales_bytes(1, 8, 4096, 128, 1) == 8 * 4096 * 8
    assert L.hifa4_qtensor_scales_bytes(1, 8, 4096, 64, 1) == 8 * 64 * 512       # 64-channel atoms padded to 128
    assert L.hifa4_attn_workspace_bytes(1, 8, 4096, 128) >= 8 * 128 * 2048 + 8 * 4096 * 8


def test_host_validation_rejects_before_launch(L):
    st = (ctypes.c_int64 * 3)(0, 0, 128)
    qt = hifa4._QT(None, None, 1, 1, 128, 128, 0)
    # null input
    assert L.hifa4_quantize_qk(None, None, st, st, 1, 1, 1, 128, 128, None, None, ctypes.byref(qt),
                               ctypes.byref(qt), None, None) == hifa4.ERR_INVALID_ARG
    buf = np.zeros(4096, np.uint8)
    p = ctypes.c_void_p(((buf.ctypes.data + 15) // 16) * 16)
    status = ctypes.c_void_p(p.value + 2048)
    # unsupported head dim / N not a multiple of 128
    assert L.hifa4_quantize_v(p, st, 1, 1, 128, 96, ctypes.byref(qt), status, None) == hifa4.ERR_UNSUPPORTED_SHAPE
    assert L.hifa4_quantize_v(p, st, 1, 1, 100, 128, ctypes.byref(qt), status, None) == hifa4.ERR_UNSUPPORTED_SHAPE
    # misaligned stride
    bad = (ctypes.c_int64 * 3)(0, 0, 129)
    assert L.hifa4_quantize_v(p, bad, 1, 1, 128, 128, ctypes.byref(qt), status, None) == hifa4.ERR_INVALID_ARG
    # d = 256 needs the 64-key tile
    q = hifa4._QT(p, p, 1, 1, 128, 256, 0)
    v = hifa4._QT(p, p, 1, 1, 128, 256, 1)
    assert L.hifa4_attn_fwd_quantized(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v), 1, 1, 1, 128, 256, 1, 128,
                                      p, None, None, status, None) == hifa4.ERR_UNSUPPORTED_SHAPE
    # GQA head counts must divide
    assert L.hifa4_attn_fwd_quantized(ctypes.byref(q), ctypes.byref(q), ctypes.byref(v), 1, 3, 2, 128, 256, 1, 64,
                                      p, None, None, status, None) == hifa4.ERR_UNSUPPORTED_SHAPE


def test_fused_rope_quantiser_rejects_null_tables(L):
    buf = np.zeros(4096, np.uint8)
    p = ctypes.c_void_p(((buf.ctypes.data + 15) // 16) * 16)
    status = ctypes.c_void_p(p.value + 2048)
    st = (ctypes.c_int64 * 3)(0, 0, 128)
    qt = hifa4._QT(p, p, 1, 1, 128, 128, 0)
    assert L.hifa4_quantize_qk_rope(p, p, st, st, 1, 1, 1, 128, 128, None, None, None, None, ctypes.byref(qt),
                                    ctypes.byref(qt), status, None) == hifa4.ERR_INVALID_ARG
    assert L.hifa4_quantize_qk_rope(p, p, st, st, 1, 1, 1, 128, 128, p, ctypes.c_void_p(p.value + 4), None, None,
                                    ctypes.byref(qt), ctypes.byref(qt), status, None) == hifa4.ERR_INVALID_ARG


def test_binding_checks_tensors_before_the_call():
    # the binding hands raw device pointers to the library; host tensors and tensors of
    # another type are refused before any call
    import torch
    x = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        hifa4.hifa4_quantize_v(x)
    with pytest.raises(TypeError, match="bfloat16"):
        hifa4.hifa4_quantize_v(x.float())
    with pytest.raises(TypeError, match="QTensor"):
        hifa4.hifa4_attn_fwd_quantized(x, x, x)
    with pytest.raises(ValueError, match="CUDA"):
        hifa4.hifa4_read_status(torch.zeros(1, dtype=torch.int32))
    # a QTensor checks its buffers once, when it is built
    with pytest.raises(ValueError, match="CUDA"):
        hifa4.QTensor(1, 1, 128, 128, 0)
    with pytest.raises(TypeError, match="uint8"):
        hifa4.QTensor(1, 1, 128, 128, 0, codes=torch.zeros(8192, dtype=torch.int8), scales=None)


def test_attn_fwd_checks_the_attention_before_quantising_v(L):
    # hifa4_attn_fwd quantises V into its workspace and then runs the attention; a call
    # the attention would reject must be rejected before the V quantiser is launched (on a
    # machine without a GPU that launch attempt would report UNSUPPORTED_DEVICE instead)
    buf = np.zeros(1 << 16, np.uint8)
    p = ctypes.c_void_p(((buf.ctypes.data + 15) // 16) * 16)
    status = ctypes.c_void_p(p.value + 32768)
    st = (ctypes.c_int64 * 3)(0, 128 * 128, 128)
    ws = L.hifa4_attn_workspace_bytes(1, 2, 128, 128)
    q = hifa4._QT(p, p, 1, 3, 128, 128, 0)
    k = hifa4._QT(p, p, 1, 2, 128, 128, 0)
    # Hq = 3 is not a multiple of Hkv = 2
    assert L.hifa4_attn_fwd(ctypes.byref(q), ctypes.byref(k), p, st, 1, 3, 2, 128, 128, 1, 0, p, ws, p, None, None,
                            status, None) == hifa4.ERR_UNSUPPORTED_SHAPE
    # a kv tile the head dim does not support
    q = hifa4._QT(p, p, 1, 2, 128, 128, 0)
    assert L.hifa4_attn_fwd(ctypes.byref(q), ctypes.byref(k), p, st, 1, 2, 2, 128, 128, 1, 32, p, ws, p, None, None,
                            status, None) == hifa4.ERR_UNSUPPORTED_SHAPE
    # a query tensor whose shape does not match the call
    qbad = hifa4._QT(p, p, 1, 2, 256, 128, 0)
    assert L.hifa4_attn_fwd(ctypes.byref(qbad), ctypes.byref(k), p, st, 1, 2, 2, 128, 128, 1, 0, p, ws, p, None,
                            None, status, None) == hifa4.ERR_INVALID_ARG
    # a workspace too small for V^T
    assert L.hifa4_attn_fwd(ctypes.byref(q), ctypes.byref(k), p, st, 1, 2, 2, 128, 128, 1, 0, p, ws - 16, p, None,
                            None, status, None) == hifa4.ERR_INVALID_ARG


def test_noalloc_rejects_a_workload_beyond_its_scratch_before_any_cuda_call(L):
    # the allocation-free entry point checks the V^T size against its fixed 16 MiB scratch
    # first: on a machine without a GPU it answers UNSUPPORTED_SHAPE (a CUDA call would
    # have produced UNSUPPORTED_DEVICE), with host dummy pointers
    fn = L.hifa4_attn_fwd_noalloc
    P, i = ctypes.c_void_p, ctypes.c_int
    QP = ctypes.POINTER(hifa4._QT)
    fn.argtypes = [QP, QP, P, P, i, i, i, i, i, i, i, P, P, P, P, P]
    fn.restype = i
    buf = np.zeros(1 << 12, np.uint8)
    p = ctypes.c_void_p(((buf.ctypes.data + 15) // 16) * 16)
    B, Hq, Hkv, N, d = 4, 32, 8, 16384, 128                  # V^T ~37 MB
    assert L.hifa4_attn_workspace_bytes(B, Hkv, N, d) > (16 << 20)
    qt = hifa4._QT(p, p, B, Hq, N, d, 0)
    kt = hifa4._QT(p, p, B, Hkv, N, d, 0)
    st = (ctypes.c_int64 * 3)(0, 0, d)
    assert fn(ctypes.byref(qt), ctypes.byref(kt), p, st, B, Hq, Hkv, N, d, 1, 0, p, None, None, p,
              None) == hifa4.ERR_UNSUPPORTED_SHAPE
    # a workload that fits goes on to the device check, which fails here without a GPU
    B, Hq, Hkv, N = 1, 4, 2, 1024
    qt = hifa4._QT(p, p, B, Hq, N, d, 0)
    kt = hifa4._QT(p, p, B, Hkv, N, d, 0)
    assert fn(ctypes.byref(qt), ctypes.byref(kt), p, st, B, Hq, Hkv, N, d, 1, 0, p, None, None, p,
              None) == hifa4.ERR_UNSUPPORTED_DEVICE


def test_layout_permutations_roundtrip():
    rng = np.random.default_rng(0)
    B, H, N, d = 2, 3, 256, 128
    plain = rng.integers(0, 256, (B, H, N, d // 16), dtype=np.uint8)
    at = _layout.rows_scales_from_plain(plain, B, H, N, d)
    assert np.array_equal(_layout.rows_scales_to_plain(at, B, H, N, d), plain)
    # the atom byte of row r, block s really is (r%32)*16 + (r//32)*4 + s
    r, s = 77, 2
    assert at[(r % 32) * 16 + (r // 32) * 4 + s] == plain[0, 0, r, s]
    for dd in (64, 128, 256):
        pv = rng.integers(0, 256, (B, H, dd, N // 16), dtype=np.uint8)
        av = _layout.vt_scales_from_plain(pv, B, H, N, dd)
        assert np.array_equal(_layout.vt_scales_to_plain(av, B, H, N, dd), pv)


def test_rope_table_matches_float64_angles():
    # host helper, no GPU: cos/sin of position * theta^(-2i/d) in double, rounded once
    from bit_flashattention_b200 import hifa4
    N, d, theta, pos0 = 300, 128, 5e5, 9
    cos, sin = hifa4.hifa4_rope_table(theta, N, d, pos0=pos0)
    inv = theta ** (-np.arange(0, d // 2, dtype=np.float64) * 2.0 / d)
    ang = (pos0 + np.arange(N, dtype=np.float64))[:, None] * inv[None, :]
    for got, ref in ((cos, np.cos(ang)), (sin, np.sin(ang))):
        ulp = np.spacing(np.abs(ref.astype(np.float32)))
        assert np.all(np.abs(got.astype(np.float64) - ref) <= 0.5 * ulp + 1e-12)
    with pytest.raises(hifa4.Hifa4Error):
        hifa4.hifa4_rope_table(1.0, N, d)


def test_product_path_fails_loudly_without_the_library(monkeypatch):
    # no CPU fallback: with libhifa4.so absent every entry point raises instead of computing
    monkeypatch.setattr(hifa4, "LIB_PATH", "/nonexistent/libhifa4.so")
    monkeypatch.setattr(hifa4, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        hifa4.lib()
    with pytest.raises(RuntimeError, match="missing"):
        hifa4.QTensor(1, 1, 128, 128, 0, "cuda")
    with pytest.raises(RuntimeError, match="missing"):
        hifa4.status_string(0)


def test_empty_and_degenerate_shapes_are_rejected_on_the_host(L):
    # zero batch, heads, tokens or query tokens, and head counts that do not divide, are
    # refused before any device work (on a machine without a GPU a launch attempt would
    # report UNSUPPORTED_DEVICE instead)
    buf = np.zeros(1 << 16, np.uint8)
    p = ctypes.c_void_p(((buf.ctypes.data + 15) // 16) * 16)
    status = ctypes.c_void_p(p.value + 32768)
    st = (ctypes.c_int64 * 3)(0, 0, 128)
    SHAPE = hifa4.ERR_UNSUPPORTED_SHAPE
    for B, H, N in ((0, 1, 128), (1, 0, 128), (1, 1, 0)):
        qt = hifa4._QT(p, p, B, H, N, 128, 0)
        vt = hifa4._QT(p, p, B, H, N, 128, 1)
        assert L.hifa4_quantize_qk(p, p, st, st, B, H, H if H else 1, N, 128, None, None, ctypes.byref(qt),
                                   ctypes.byref(qt), status, None) == SHAPE
        assert L.hifa4_quantize_v(p, st, B, H, N, 128, ctypes.byref(vt), status, None) == SHAPE
        assert L.hifa4_quantize_qkv(p, p, p, st, st, st, B, H, H if H else 1, N, 128, None, None, ctypes.byref(qt),
                                    ctypes.byref(qt), ctypes.byref(vt), status, None) == SHAPE
        assert L.hifa4_attn_fwd_quantized(ctypes.byref(qt), ctypes.byref(qt), ctypes.byref(vt), B, H, H if H else 1,
                                          N, 128, 1, 0, p, None, None, status, None) == SHAPE
    ws = ctypes.c_size_t(1 << 15)
    q = hifa4._QT(p, p, 1, 1, 128, 128, 0)
    for nq, Nk in ((0, 256), (1, 0), (129, 256)):
        k = hifa4._QT(p, p, 1, 1, Nk, 128, 0)
        v = hifa4._QT(p, p, 1, 1, Nk, 128, 1)
        assert L.hifa4_attn_decode(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), 1, 1, 1, nq, Nk, 128, 0, 0, p,
                                   ws, p, None, None, status, None) == SHAPE
    assert L.hifa4_calibrate_smooth(p, p, st, st, 1, 1, 1, 0, 128, 0.5, p, p, p, None) == SHAPE
    assert L.hifa4_calibrate_smooth(p, p, st, st, 1, 3, 2, 16, 128, 0.5, p, p, p, None) == SHAPE
    assert L.hifa4_calibrate_smooth(p, p, st, st, 1, 1, 1, 16, 128, -0.5, p, p, p, None) == hifa4.ERR_INVALID_ARG
    # size helpers give 0 for empty tensors
    assert L.hifa4_qtensor_codes_bytes(0, 1, 128, 128) == 0 and L.hifa4_qtensor_scales_bytes(1, 1, 0, 128, 0) == 0
    assert L.hifa4_decode_workspace_bytes(1, 1, 0, 128) == 0 and L.hifa4_decode_workspace_bytes(1, 1, 65, 128) == 0


def test_header_is_plain_c_and_a_c_program_links(L, tmp_path):
    # include/hifa4.h is a C header (no torch or C++ types): a C11 program includes it,
    # links against libhifa4.so and calls a host-only entry point
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.join(root, "bit_flashattention_b200")
    src = tmp_path / "use_hifa4.c"
    src.write_text('#include "hifa4.h"\n'
                   'int main(void) {\n'
                   '  if (hifa4_qtensor_codes_bytes(1, 2, 128, 64) != 8192) return 1;\n'
                   '  if (hifa4_qtensor_scales_bytes(1, 2, 128, 64, 0) != 1024) return 2;\n'
                   '  return hifa4_status_string(HIFA4_ERR_TIMEOUT)[0] == \'H\' ? 0 : 3;\n'
                   '}\n')
    exe = tmp_path / "use_hifa4"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(root, "include"), "-I", cuda_inc,
                        str(src), "-o", str(exe), "-L", libdir, "-lhifa4", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert subprocess.run([str(exe)]).returncode == 0
