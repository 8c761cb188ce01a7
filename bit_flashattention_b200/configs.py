"""The five attention workloads this library is measured and tested on.

Each entry fixes a shape (B, Hq, Hkv, N, d, causal), the Smooth-QK strength alpha
(None = Smooth-QK disabled, s == 1), the kv tile width Bc that is part of the
result's definition (the online-softmax state is updated once per kv tile), and the
recipe of the synthetic inputs (RoPE base, K outlier channels and factor, K bias).

The shapes follow the LLM families named in the HiFA4 abstract ("HiFA4: Training-Free
4-bit FlashAttention on Ascend HIF4 NPUs for LLM Inference", abstract: Qwen3-8B,
Gemma2-9B, LLaMA3.1-8B, Phi-4B); the pages give no trained weights or traces, so
the values are synthetic stand-ins with those shapes only.
"""
from dataclasses import dataclass
from typing import Optional


@dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    alpha: Optional[float]     # Smooth-QK exponent; None = disabled (s == 1)
    bc: int                    # kv tile width (part of the result's definition)
    rope_theta: Optional[float]
    k_outlier_channels: int
    k_outlier_factor: float
    k_bias: bool

    @property
    def flops(self) -> float:
        """Metric flops: 4*B*Hq*N^2*d, halved for causal (QK^T and PV, 2 flops/MAC)."""
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 1, 256, 64, False, 0.5, 64,
                     None, 4, 8.0, True),
    "qwen3-8b-4k": Workload("qwen3-8b-4k", 1, 1, 32, 8, 4096, 128, True, 0.5, 256,
                            1e6, 8, 10.0, True),
    "gemma2-9b-8k": Workload("gemma2-9b-8k", 2, 1, 16, 8, 8192, 256, True, 0.25, 64,
                             1e4, 8, 4.0, True),
    "llama3.1-8b-b4-16k": Workload("llama3.1-8b-b4-16k", 3, 4, 32, 8, 16384, 128, True, None, 256,
                                   5e5, 8, 10.0, False),
    "phi-32k": Workload("phi-32k", 4, 1, 24, 8, 32768, 128, True, 0.5, 256,
                        1e4, 6, 6.0, False),
}

ORDER = ["tiny", "qwen3-8b-4k", "gemma2-9b-8k", "llama3.1-8b-b4-16k", "phi-32k"]


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (used for reduced-size test cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)
