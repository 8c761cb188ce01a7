"""Seeded synthetic inputs (bf16 Q, K, V and the Smooth-QK calibration sample).

This module only draws random numbers and arranges them the way a post-RoPE attention
input looks; it holds none of the attention method's arithmetic, so both the CPU
oracle's tests and the CUDA path take their inputs from here.

Recipe (per workload, see ``configs.py``):
  * numpy PCG64 seeded with ``SeedSequence([cfg_id, stream, b, h])`` so every
    (batch, head) slab can be drawn on its own.  Streams: 0 = "model" parameters
    (K outlier channels, K bias), 1/2/3 = Q/K/V, 11/12/13 = calibration Q/K/V.
  * Q, K, V ~ N(0, 1) drawn in fp32.
  * RoPE (rotate-half convention, positions 0..N-1, inv_freq_i = theta^(-2i/d)) on Q
    and K when the workload has a RoPE base.
  * Then, on K only: the seeded outlier channels of each kv head are multiplied by the
    outlier factor, and a per-(kv head, channel) bias ~ N(0, 1) is added when enabled.
    Smooth-QK is calibrated on and applied to these post-RoPE tensors (the HiFA4
    abstract applies its per-channel scales after RoPE).
  * Everything is rounded to bf16 (round to nearest even) and returned as uint16 bits.

The pages measure on MMLU traces of real models; those are not available here, so these
tensors stand in for them by shape and by the outlier structure named in the workloads.
"""
import numpy as np

from .configs import Workload

STREAM_MODEL = 0
STREAM_Q, STREAM_K, STREAM_V = 1, 2, 3
STREAM_QCAL, STREAM_KCAL, STREAM_VCAL = 11, 12, 13


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(w: Workload, *words):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.cfg_id, *words])))


def model_params(w: Workload):
    """Outlier channel indices [Hkv, n_out] and K bias [Hkv, d] (zeros when disabled)."""
    rng = _rng(w, STREAM_MODEL)
    n_out = w.k_outlier_channels
    chans = np.stack([rng.choice(w.d, size=n_out, replace=False) for _ in range(w.Hkv)]) \
        if n_out > 0 else np.zeros((w.Hkv, 0), dtype=np.int64)
    bias = rng.standard_normal((w.Hkv, w.d), dtype=np.float32) if w.k_bias \
        else np.zeros((w.Hkv, w.d), dtype=np.float32)
    return chans, bias


def _rope(x: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE over positions 0..N-1 of an [N, d] fp32 slab (computed in fp64)."""
    n, d = x.shape
    half = d // 2
    inv_freq = theta ** (-np.arange(0, half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(n, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    x1 = x[:, :half].astype(np.float64)
    x2 = x[:, half:].astype(np.float64)
    out = np.empty((n, d), dtype=np.float64)
    out[:, :half] = x1 * cos - x2 * sin
    out[:, half:] = x2 * cos + x1 * sin
    return out.astype(np.float32)


def head_slab(w: Workload, which: str, b: int, h: int, calib: bool = False) -> np.ndarray:
    """One [N, d] bf16 slab (uint16 bits) of Q (h in 0..Hq-1), K or V (h in 0..Hkv-1)."""
    stream = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}[which]
    if calib:
        stream += 10
    x = _rng(w, stream, b, h).standard_normal((w.N, w.d), dtype=np.float32)
    if which in ("q", "k") and w.rope_theta is not None:
        x = _rope(x, w.rope_theta)
    if which == "k":
        chans, bias = model_params(w)
        if chans.shape[1]:
            x[:, chans[h]] *= np.float32(w.k_outlier_factor)
        x += bias[h][None, :]
    return f32_to_bf16_bits(x)


def tensor(w: Workload, which: str, calib: bool = False, batches=None) -> np.ndarray:
    """[B, H, N, d] bf16 tensor (uint16 bits) for 'q', 'k' or 'v'; with `batches` (a range of
    batch indices) only those batches, [len(batches), H, N, d], drawn exactly as in the
    full tensor."""
    H = w.Hq if which == "q" else w.Hkv
    bs = range(w.B) if batches is None else batches
    out = np.empty((len(bs), H, w.N, w.d), dtype=np.uint16)
    for i, b in enumerate(bs):
        for h in range(H):
            out[i, h] = head_slab(w, which, b, h, calib)
    return out


def inputs(w: Workload, calib: bool = False, batches=None):
    """(Q, K, V) bf16 bit tensors of the workload (or of its calibration sample); `batches`
    selects a range of batch indices."""
    return tensor(w, "q", calib, batches), tensor(w, "k", calib, batches), tensor(w, "v", calib, batches)


def sample_rows(w: Workload, per_head: int = 8, seed: int = 7, br: int = 128):
    """Seeded sample of query row ids ((b*Hq + h)*N + i) for full-size parity checks:
    per (b, h) the first and the last 128-row q-tile plus `per_head` random rows."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.cfg_id, 99, seed])))
    rows = []
    for b in range(w.B):
        for h in range(w.Hq):
            base = (b * w.Hq + h) * w.N
            sel = set(range(0, min(br, w.N)))
            sel |= set(range(max(0, w.N - br), w.N))
            sel |= set(int(i) for i in rng.integers(0, w.N, size=per_head))
            rows.extend(base + i for i in sorted(sel))
    return np.asarray(rows, dtype=np.int32)
