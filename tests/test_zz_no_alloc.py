"""hifa4_attn_fwd_noalloc: the attention entry point for callers that cannot allocate
device memory (their memory is all handed out up front, or they must not block on
cudaMalloc).  It keeps the 4-bit V^T in a fixed 16 MiB array inside the library instead
of a caller workspace.  Called through the C ABI, on two different inputs in a row, it
must give bit for bit what hifa4_attn_fwd gives on the same inputs (the same kernels run
on the same operands; only the V^T buffer differs), and it must reject a workload whose
scratch would not fit.  Collected last so that a failure here cannot hide others."""
import ctypes

import pytest
import torch

from bit_flashattention_b200 import configs, gen, hifa4
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = hifa4.lib().hifa4_attn_fwd_noalloc
    P, i = ctypes.c_void_p, ctypes.c_int
    QP = ctypes.POINTER(hifa4._QT)
    fn.argtypes = [QP, QP, P, P, i, i, i, i, i, i, i, P, P, P, P, P]
    fn.restype = i
    return fn


def _call_noalloc(w, qq, kq, vt_bf16):
    fn = _noalloc_fn()
    o = torch.empty(w.B, w.Hq, w.N, w.d, dtype=torch.bfloat16, device="cuda")
    m = torch.empty(w.B, w.Hq, w.N, dtype=torch.float16, device="cuda")
    l = torch.empty(w.B, w.Hq, w.N, dtype=torch.float16, device="cuda")
    st = hifa4.new_status("cuda")
    s = vt_bf16.stride()
    code = fn(qq.c(), kq.c(), ctypes.c_void_p(vt_bf16.data_ptr()), (ctypes.c_int64 * 3)(s[0], s[1], s[2]),
              w.B, w.Hq, w.Hkv, w.N, w.d, int(w.causal), w.bc, ctypes.c_void_p(o.data_ptr()),
              ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(l.data_ptr()), ctypes.c_void_p(st.data_ptr()),
              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == hifa4.OK, hifa4.status_string(code)
    assert hifa4.hifa4_read_status(st) == hifa4.OK
    return o, m, l


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [configs.scaled(configs.get("qwen3-8b-4k"), Hq=8, Hkv=2, N=1024),
             configs.scaled(configs.get("phi-32k"), Hq=6, Hkv=2, N=768)]
    for w in cases:                     # two calls in a row, on different inputs
        q, k, v = gen.inputs(w)
        s, sinv = gc.smooth_scales(w)
        qq, kq, _, vt = gc.gpu_quantize(w, q, k, v, s, sinv)
        o_ref, m_ref, l_ref, code = gc.gpu_attention(w, qq, kq, vt)
        assert code == hifa4.OK
        o, m, l = _call_noalloc(w, qq, kq, vt)
        torch.cuda.synchronize()
        assert torch.equal(m, m_ref) and torch.equal(l, l_ref)
        assert torch.equal(o, o_ref)


def test_noalloc_rejects_workload_beyond_its_scratch():
    w = configs.get("llama3.1-8b-b4-16k")           # V^T needs ~37 MB > 16 MiB
    assert hifa4.lib().hifa4_attn_workspace_bytes(w.B, w.Hkv, w.N, w.d) > (16 << 20)
    fn = _noalloc_fn()
    dummy = torch.zeros(256, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    qt = hifa4._QT(p, p, w.B, w.Hq, w.N, w.d, 0)
    kt = hifa4._QT(p, p, w.B, w.Hkv, w.N, w.d, 0)
    code = fn(ctypes.byref(qt), ctypes.byref(kt), ctypes.c_void_p(p), (ctypes.c_int64 * 3)(0, 0, w.d),
              w.B, w.Hq, w.Hkv, w.N, w.d, 1, w.bc, ctypes.c_void_p(p), None, None, ctypes.c_void_p(p), None)
    assert code == hifa4.ERR_UNSUPPORTED_SHAPE
