"""Reader of the hand-derived worked examples in tests/golden/worked_examples.txt and the
input recipe of its attention cases (shared by the oracle and GPU tests)."""
import os

import numpy as np

from bit_flashattention_b200 import gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_examples.txt")


def load():
    """{section: {key: [tokens]}} of the fixture ('#' comments dropped)."""
    sections, cur = {}, None
    for raw in open(GOLDEN):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        if line.startswith("[") and line.endswith("]"):
            cur = sections.setdefault(line[1:-1], {})
            continue
        key, val = line.split(":", 1)
        cur[key.strip()] = val.split()
    return sections


def num(s):
    return int(s, 16) if s.startswith("0x") else float(s)


# the 16 E2M1 multiples every 16-token block of a V channel holds (a rotation of them)
L = np.array([6, -6, 4, -4, 3, -3, 2, -2, 1.5, -1.5, 1, -1, 0.5, -0.5, 0, 6], np.float64)


def attn_inputs(N=256, d=64):
    """The fixture's attention inputs as bf16 bits [1, 1, N, d]: Q = 0, K any values,
    V[n, c] = 2^-(c % 4) / 4 * L[(n + c) % 16]; also V as float64 [N, d]."""
    n = np.arange(N)[:, None]
    c = np.arange(d)[None, :]
    v = np.exp2(-(c % 4)) / 4 * L[(n + c) % 16]
    k = ((7 * n + 3 * c) % 13 - 6) * 0.5              # any values: Q_hat = 0 ignores them
    q = np.zeros((N, d))
    bits = lambda a: gen.f32_to_bf16_bits(a.astype(np.float32))[None, None]
    return bits(q), bits(k), bits(v), v


def select_inputs(N=256, d=64):
    """The attn_select case: every query row (6, 0, ..., 0); key n with n % 4 == 0 zero in
    channels 0..15, the others -6 in channel 0 and zero in 1..15; channels 16.. of K any
    values; V as in attn_inputs.  bf16 bits [1, 1, N, d]."""
    _, k, v, vf = attn_inputs(N, d)
    kf = gen.bf16_bits_to_f32(k[0, 0]).copy()
    kf[:, :16] = 0.0
    kf[np.arange(N) % 4 != 0, 0] = -6.0
    q = np.zeros((N, d), np.float32)
    q[:, 0] = 6.0
    bits = lambda a: gen.f32_to_bf16_bits(a.astype(np.float32))[None, None]
    return bits(q), bits(kf), v, vf


def tie_inputs(N=256, d=64):
    """The attn_bf16_tie case: Q = 0, K as in attn_inputs, every V channel 1 except a 1.5
    at the start of each 16-token block, then a 1.5 (block 0) or a 0.5 (the others).
    bf16 bits [1, 1, N, d]."""
    q, k, _, _ = attn_inputs(N, d)
    col = np.ones(N)
    col[0::16] = 1.5
    col[1::16] = 0.5
    col[1] = 1.5
    v = np.repeat(col[:, None], d, axis=1)
    return q, k, gen.f32_to_bf16_bits(v.astype(np.float32))[None, None]
