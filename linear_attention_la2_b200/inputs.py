"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module only draws random numbers. It holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle may consume its output.

Recipe (one per workload): a CPU ``torch.Generator`` seeded with ``seed``
draws ``torch.randn`` in fp32, in the order Q, K, V, then dO (backward only),
each of shape ``[B, H, N, d]`` (``dv`` for V and dO). Every tensor is scaled by
``1/sqrt(d)`` and then rounded to the run's dtype. The oracle reads these exact
rounded values, upcast to float64.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, block size, dtype and seed."""

    name: str
    B: int
    H: int
    N: int
    d: int
    dv: int
    block: int
    dtype: str  # "f32" or "bf16"
    seed: int
    causal: bool = True
    backward: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def tokens(self) -> int:
        """Token-heads in one pass: B*H*N."""
        return self.B * self.H * self.N


# The five workloads of the hot path, with their seeds (workload k uses seed k-1).
WORKLOADS = {
    "fp32_small": Workload("fp32_small", 1, 1, 256, 64, 64, 64, "f32", 0),
    "bf16_b4h16_n2k": Workload("bf16_b4h16_n2k", 4, 16, 2048, 128, 128, 64, "bf16", 1),
    "bf16_sweep": Workload("bf16_sweep", 1, 32, 1024, 128, 128, 64, "bf16", 2),
    "bf16_long_512k": Workload("bf16_long_512k", 1, 8, 524288, 128, 128, 128, "bf16", 3),
    "bf16_fwdbwd_b2h32_n8k": Workload("bf16_fwdbwd_b2h32_n8k", 2, 32, 8192, 128, 128, 64, "bf16", 4,
                                      backward=True),
}

# Follow-on rows measured beside the five: grouped K/V heads (NEXT-3; ``Hkv`` K/V
# heads, query head h reads K/V head h // (H // Hkv)) and the decayed form (NEXT-4;
# one rate for every head), at the shapes of the B4 H16 N2K and B2 H32 N8K
# workloads (same seeds; K and V keep their first Hkv heads).
EXTRA_WORKLOADS = {
    "bf16_gqa_b4h16kv4_n2k": Workload("bf16_gqa_b4h16kv4_n2k", 4, 16, 2048, 128, 128, 64, "bf16", 1,
                                      extra={"Hkv": 4}),
    "bf16_gqa_fwdbwd_b2h32kv8_n8k": Workload("bf16_gqa_fwdbwd_b2h32kv8_n8k", 2, 32, 8192, 128, 128,
                                             64, "bf16", 4, backward=True, extra={"Hkv": 8}),
    "bf16_decay_b4h16_n2k": Workload("bf16_decay_b4h16_n2k", 4, 16, 2048, 128, 128, 64, "bf16", 1,
                                     extra={"decay": 0.99}),
    "bf16_decay_fwdbwd_b4h16_n2k": Workload("bf16_decay_fwdbwd_b4h16_n2k", 4, 16, 2048, 128, 128, 64,
                                            "bf16", 1, backward=True, extra={"decay": 0.99}),
}

SWEEP_N = (1024, 4096, 16384, 65536)
SWEEP_BLOCKS = (64, 128)


def sweep_workload(N: int, block: int) -> Workload:
    """The sequence-length sweep point (B=1, H=32, d=dv=128, bf16, seed 2)."""
    return Workload(f"bf16_sweep_n{N}_b{block}", 1, 32, N, 128, 128, block, "bf16", 2)


def make_inputs(w: Workload, with_grad_out: bool | None = None, device: str = "cpu"):
    """Draw Q, K, V (and dO) for workload ``w``.

    Returns a dict of tensors in the workload dtype on ``device``. The draw
    always happens on the CPU generator so the values do not depend on the
    device they end up on.
    """
    if with_grad_out is None:
        with_grad_out = w.backward
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    scale = 1.0 / math.sqrt(w.d)
    shapes = [("q", w.d), ("k", w.d), ("v", w.dv)]
    if with_grad_out:
        shapes.append(("do", w.dv))
    out = {}
    for name, last in shapes:
        t = torch.randn((w.B, w.H, w.N, last), generator=g, dtype=torch.float32)
        t.mul_(scale)
        out[name] = t.to(w.torch_dtype).to(device)
    return out


def make_custom(B, H, N, d, dv, dtype: str, seed: int, with_grad_out: bool = False,
                device: str = "cpu"):
    """Same recipe for an arbitrary shape (edge-case parity tests)."""
    w = Workload("custom", B, H, N, d, dv, 64, dtype, seed, backward=with_grad_out)
    return make_inputs(w, with_grad_out=with_grad_out, device=device)


def sample_rows(N: int, block: int, seed: int, count: int = 256, chunk: int | None = None,
                max_blocks: int = 64):
    """Rows checked one by one at full size.

    The first and last row of every block (of at most ``max_blocks`` evenly
    spaced blocks, always including the first and the last one), the first and
    last row of every chunk when ``chunk`` is given, row N-1, and ``count``
    seeded random rows.
    """
    nblk = (N + block - 1) // block
    if nblk <= max_blocks:
        blocks = range(nblk)
    else:
        step = nblk / (max_blocks - 1)
        blocks = sorted({min(nblk - 1, int(round(i * step))) for i in range(max_blocks)})
    rows = set()
    for b in blocks:
        start = b * block
        rows.add(start)
        rows.add(min(start + block, N) - 1)
    if chunk:
        for start in range(0, N, chunk):
            rows.add(start)
            rows.add(min(start + chunk, N) - 1)
    rows.add(N - 1)
    g = torch.Generator(device="cpu")
    g.manual_seed(1000 + seed)
    for r in torch.randint(0, N, (count,), generator=g).tolist():
        rows.add(int(r))
    return sorted(rows)
