"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle checks.

This module draws random numbers and rounds them to the working dtype; it holds
none of the attention arithmetic. Recipe: one CPU ``torch.Generator`` seeded
with ``seed``; ``randn`` in float32 drawn in the order Q, K, V, then dO when a
backward is wanted; for bf16 workloads each tensor is rounded to bf16
(round-to-nearest-even). The oracle receives the same rounded values upcast to
float64, which is exact.

The named workloads are the shapes of the attention runs this library is
measured and checked on; the 8192-token, 32-head case is the one whose unfused
score matrix would exceed four gigabytes in half precision (fanfani.net
"FlashAttention", section "The bottleneck was never the arithmetic").
"""

from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    dtype: str  # "bf16" or "f32"
    causal: tuple  # causal settings run on this shape
    backward: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


WORKLOADS = {
    w.name: w
    for w in (
        Workload("fwd_f32_b1_h2_n256_d64", 1, 2, 2, 256, 64, "f32", (False,)),
        Workload("fwd_bf16_b4_h16_n2048_d64", 4, 16, 16, 2048, 64, "bf16", (False, True)),
        Workload("fwd_causal_bf16_b2_h32_n8192_d128", 2, 32, 32, 8192, 128, "bf16", (True,)),
        Workload("gqa_causal_bf16_b1_h32_kv8_n16384_d128", 1, 32, 8, 16384, 128, "bf16", (True,)),
        Workload("gqa_causal_bf16_b1_h16_kv4_n8192_d256", 1, 16, 4, 8192, 256, "bf16", (True,)),
        Workload("train_causal_bf16_b2_h16_n4096_d128", 2, 16, 16, 4096, 128, "bf16", (True,), True),
    )
}


def make_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, dtype: str = "bf16",
                seed: int = 0, grad: bool = False) -> dict:
    """Return CPU tensors ``q [B,Hq,N,d]``, ``k, v [B,Hkv,N,d]`` (and ``do``)."""
    if dtype not in ("bf16", "f32"):
        raise ValueError(f"dtype must be 'bf16' or 'f32', got {dtype!r}")
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    out = {
        "q": torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32),
        "k": torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32),
        "v": torch.randn((B, Hkv, N, d), generator=g, dtype=torch.float32),
    }
    if grad:
        out["do"] = torch.randn((B, Hq, N, d), generator=g, dtype=torch.float32)
    if dtype == "bf16":
        out = {name: t.to(torch.bfloat16) for name, t in out.items()}
    return out


def workload_inputs(w: Workload, seed: int = 0) -> dict:
    return make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, seed, grad=w.backward)


def as_f64(t: torch.Tensor):
    """Exact float64 numpy copy of a CPU or CUDA tensor (bf16 and f32 upcast exactly)."""
    return t.detach().to("cpu", torch.float64).numpy()


def make_varlen_inputs(lens_q, lens_k, Hq: int, Hkv: int, d: int, dtype: str = "bf16", seed: int = 0,
                       grad: bool = False):
    """A packed batch of sequences: ``q [sum(lens_q), Hq, d]``, ``k, v [sum(lens_k), Hkv, d]`` (CPU) and
    the int32 offsets ``cu_q``, ``cu_k`` (batch + 1 entries from 0); with ``grad`` also an upstream
    gradient ``do`` shaped like ``q``. Same recipe as :func:`make_inputs`."""
    if len(lens_q) != len(lens_k):
        raise ValueError("one query length and one key length per sequence")
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    out = {
        "q": torch.randn((tq, Hq, d), generator=g, dtype=torch.float32),
        "k": torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32),
        "v": torch.randn((tk, Hkv, d), generator=g, dtype=torch.float32),
    }
    if grad:
        out["do"] = torch.randn((tq, Hq, d), generator=g, dtype=torch.float32)
    if dtype == "bf16":
        out = {name: t.to(torch.bfloat16) for name, t in out.items()}
    cu = lambda lens: torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    out["cu_q"], out["cu_k"] = cu(lens_q), cu(lens_k)
    return out
