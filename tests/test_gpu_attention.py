"""GPU parity of the fused 4-bit attention forward against the oracle, through the C ABI:
FP16 m and l exact per row, O within max-abs 1e-2 and mean-relative 1e-3, on seeded
synthetic inputs of every workload family (reduced sizes compared on every row; full
sizes on sampled rows), plus the bounded-wait timeout path."""
import numpy as np
import pytest

from bit_flashattention_b200 import configs, gen, hifa4
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

REDUCED = [
    ("tiny", {}),
    ("tiny", dict(causal=True)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=512)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=512, bc=128)),
    ("qwen3-8b-4k", dict(Hq=4, Hkv=2, N=384, bc=128, causal=False)),
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=768, causal=False)),
    ("qwen3-8b-4k", dict(Hq=2, Hkv=1, N=256, bc=64)),
    ("gemma2-9b-8k", dict(Hq=4, Hkv=2, N=512)),
    ("gemma2-9b-8k", dict(Hq=2, Hkv=1, N=256, causal=False)),
    ("llama3.1-8b-b4-16k", dict(B=2, Hq=4, Hkv=1, N=512)),
    ("phi-32k", dict(Hq=3, Hkv=1, N=1024)),
    ("tiny", dict(d=64, bc=128, N=512, causal=True)),
]


@pytest.mark.parametrize("name,kw", REDUCED)
def test_parity_reduced_all_rows(name, kw):
    w = configs.scaled(configs.get(name), **kw)
    gc.assert_parity(gc.run_parity(w))


@pytest.mark.parametrize("name", ["tiny", "qwen3-8b-4k", "gemma2-9b-8k"])
def test_parity_full_size_sampled_rows(name):
    w = configs.get(name)
    rows = gen.sample_rows(w, per_head=4) if w.N > 256 else None
    gc.assert_parity(gc.run_parity(w, rows, check_quant=False))


def test_timeout_is_reported_and_context_survives():
    w = configs.scaled(configs.get("qwen3-8b-4k"), Hq=2, Hkv=1, N=512)
    q, k, v = gen.inputs(w)
    qq, kq, vq, vt = gc.gpu_quantize(w, q, k, v, None, None)
    hifa4.hifa4_set_wait_limit_ns(200_000_000)
    hifa4.hifa4_debug_set_injection(1)
    try:
        _, _, _, code = gc.gpu_attention(w, qq, kq, vt)
    finally:
        hifa4.hifa4_debug_set_injection(0)
        hifa4.hifa4_set_wait_limit_ns(2_000_000_000)
    assert code == hifa4.ERR_TIMEOUT
    # the context is still usable and the next call is correct
    gc.assert_parity(gc.run_parity(w))
