"""Seeded synthetic inputs for the PACE decode path.

This module is the one piece shared by the fp64 oracle (``oracle/``) and the
CUDA path (``bit_recurrent_state_pace_b200``).  It holds no arithmetic of the
method itself: it only draws random numbers and shapes them into the
per-token inputs ``(q, k, v, alpha, beta)`` of a Gated DeltaNet decode step,
plus the seeded choices a workload makes (which heads are stored as INT8,
which value channels carry outliers).

Workloads stand in for the batched decode of the hybrid 4B-35B models that
the PACE pages evaluate on ("PACE: four-bit recurrent state by rounding less
often", TL;DR).  No model weights or evaluation suites are used; every tensor
is synthetic with the distribution stated below:

* ``q, k ~ N(0, 1)``, L2-normalised over ``d_k`` per (sequence, head), then
  cast to the io dtype;
* ``v ~ N(0, 1)``; in the 4B-hybrid-like workloads four seeded value channels
  (shared by every sequence, head and token) are scaled by 8;
* ``beta = sigmoid(N(0, 1))``;
* ``alpha = exp(-0.1 * softplus(N(0, 1)))``; heads marked long-memory use
  ``-0.01`` instead of ``-0.1``;
* all of them rounded to the io dtype (bf16, or fp32 for the tiny case) before
  either side sees them.

Small tensors are drawn on the host with a CPU generator; large ones on the
GPU with a CUDA generator.  Either way the oracle is handed copies of the very
tensors the GPU consumes, so the two sides never need identical streams.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional, Sequence

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "int8_heads",
    "long_memory_heads",
    "outlier_channels",
    "head_bits",
    "token_inputs",
    "token_inputs_for_heads",
    "random_state",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one decode workload."""

    name: str
    B: int                 # concurrently decoding sequences (pool slots)
    H: int                 # value heads per layer
    d_k: int
    d_v: int
    P: int                 # period: tokens buffered between two roundings
    steps: int             # decode steps
    io_dtype: str          # "bf16" or "f32"
    int8_fraction: float   # share of heads kept at 8 bits
    long_memory_int8: bool  # INT8 heads also get the slow-decay alpha
    outliers: bool         # four value channels scaled by 8
    warmup: int            # tokens of unquantised fp32 prefill before decode
    axis: str = "col"      # "col" = one scale per key channel j

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_io_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.io_dtype == "bf16" else torch.float32


# The five workloads, numbered 0..4 as listed with the method's benchmarks.
WORKLOADS: Dict[str, Workload] = {
    # 0: exactness case, every head checked.
    "tiny": Workload("tiny", B=2, H=2, d_k=32, d_v=32, P=4, steps=16,
                     io_dtype="f32", int8_fraction=0.0, long_memory_int8=False,
                     outliers=False, warmup=0),
    # 1: one GDN layer shaped like a 4B hybrid.
    "gdn_layer_4b": Workload("gdn_layer_4b", B=64, H=32, d_k=128, d_v=128, P=8,
                             steps=256, io_dtype="bf16", int8_fraction=0.0,
                             long_memory_int8=False, outliers=True, warmup=512),
    # 2: mixed 4/8-bit heads; the INT8 heads are the long-memory heads.
    "mixed_4_8": Workload("mixed_4_8", B=256, H=32, d_k=128, d_v=128, P=8,
                          steps=512, io_dtype="bf16", int8_fraction=0.25,
                          long_memory_int8=True, outliers=True, warmup=512),
    # 3: period sweep (P is overridden per run: 1, 2, 4, 8, 16).
    "period_sweep": Workload("period_sweep", B=512, H=32, d_k=128, d_v=128, P=8,
                             steps=1024, io_dtype="bf16", int8_fraction=0.0,
                             long_memory_int8=False, outliers=True, warmup=512),
    # 4: concurrency stress, the HBM-bandwidth workload.
    "concurrency_stress": Workload("concurrency_stress", B=4096, H=48, d_k=128,
                                   d_v=128, P=8, steps=1024, io_dtype="bf16",
                                   int8_fraction=0.25, long_memory_int8=False,
                                   outliers=True, warmup=512),
}

PERIOD_SWEEP = (1, 2, 4, 8, 16)


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.replace(**overrides) if overrides else w


def _seed(*parts) -> int:
    """Stable 63-bit seed from a tuple of labels (independent of PYTHONHASHSEED)."""
    h = hashlib.sha256(repr(parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(device: torch.device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def int8_heads(w: Workload, seed: int = 0) -> List[int]:
    """Seeded choice of floor(H * int8_fraction) head indices kept at 8 bits."""
    n8 = int(w.H * w.int8_fraction)
    if n8 == 0:
        return []
    g = _gen(torch.device("cpu"), "int8_heads", w.H, n8, seed)
    perm = torch.randperm(w.H, generator=g)
    return sorted(int(x) for x in perm[:n8])


def long_memory_heads(w: Workload, seed: int = 0) -> List[int]:
    return int8_heads(w, seed) if w.long_memory_int8 else []


def head_bits(w: Workload, seed: int = 0) -> List[int]:
    """Per-head storage width (4 or 8) for the workload."""
    eight = set(int8_heads(w, seed))
    return [8 if h in eight else 4 for h in range(w.H)]


def outlier_channels(w: Workload, seed: int = 0) -> List[int]:
    """Four seeded value channels scaled by 8 (a property of the model's channels)."""
    if not w.outliers:
        return []
    g = _gen(torch.device("cpu"), "outliers", w.d_v, seed)
    perm = torch.randperm(w.d_v, generator=g)
    return sorted(int(x) for x in perm[:4])


def _alpha_coeff(w: Workload, seed: int, device) -> torch.Tensor:
    c = torch.full((w.H,), -0.1, dtype=torch.float32, device=device)
    for h in long_memory_heads(w, seed):
        c[h] = -0.01
    return c


def token_inputs(w: Workload, t: int, seed: int = 0, device="cpu",
                 phase: str = "decode") -> Dict[str, torch.Tensor]:
    """Inputs of decode token ``t`` for all B x H heads.

    Returns q, k ``[B, H, d_k]``, v ``[B, H, d_v]``, alpha, beta ``[B, H]``,
    all in the workload's io dtype on ``device``.  ``phase`` separates the
    warm-up prefill stream from the decode stream.
    """
    device = torch.device(device)
    g = _gen(device, "tok", w.name, w.B, w.H, w.d_k, w.d_v, phase, t, seed)
    f32 = torch.float32
    q = torch.randn(w.B, w.H, w.d_k, generator=g, device=device, dtype=f32)
    k = torch.randn(w.B, w.H, w.d_k, generator=g, device=device, dtype=f32)
    v = torch.randn(w.B, w.H, w.d_v, generator=g, device=device, dtype=f32)
    zb = torch.randn(w.B, w.H, generator=g, device=device, dtype=f32)
    za = torch.randn(w.B, w.H, generator=g, device=device, dtype=f32)
    q = q / q.norm(dim=-1, keepdim=True)
    k = k / k.norm(dim=-1, keepdim=True)
    ch = outlier_channels(w, seed)
    if ch:
        v[..., ch] *= 8.0
    beta = torch.sigmoid(zb)
    alpha = torch.exp(_alpha_coeff(w, seed, device)[None, :] * torch.nn.functional.softplus(za))
    dt = w.torch_io_dtype
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt),
            "alpha": alpha.to(dt), "beta": beta.to(dt)}


def token_inputs_for_heads(inputs: Dict[str, torch.Tensor],
                           heads: Sequence[tuple]) -> Dict[str, torch.Tensor]:
    """Gather the inputs of the listed (b, h) heads into host float64 tensors."""
    bs = torch.tensor([b for b, _ in heads], dtype=torch.long)
    hs = torch.tensor([h for _, h in heads], dtype=torch.long)
    out = {}
    for name, x in inputs.items():
        x = x.detach()
        sel = x[bs.to(x.device), hs.to(x.device)]
        out[name] = sel.to("cpu", torch.float64)
    return out


def random_state(n: int, d_v: int, d_k: int, seed: int = 0, device="cpu",
                 column_outliers: Optional[Sequence[int]] = None,
                 row_outliers: Optional[Sequence[int]] = None,
                 scale: float = 1.0) -> torch.Tensor:
    """``n`` seeded fp32 matrices ``[n, d_v, d_k]`` for quantiser tests."""
    device = torch.device(device)
    g = _gen(device, "state", n, d_v, d_k, seed)
    S = torch.randn(n, d_v, d_k, generator=g, device=device, dtype=torch.float32) * scale
    if column_outliers:
        S[..., list(column_outliers)] *= 8.0
    if row_outliers:
        S[..., list(row_outliers), :] *= 8.0
    return S
