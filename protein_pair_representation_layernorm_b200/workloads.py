"""Seeded synthetic workloads for the triangle attention block.

This module only draws random numbers and arranges them; it contains none of
the block's arithmetic.  Both the GPU path (tests, benchmark) and the CPU
oracle (tests only) take their inputs from here, so that the two sides see
bit-identical values.

Recipe (every draw on the CPU with ``torch.Generator().manual_seed(seed)``,
in this order):

1. Z, shape (N, N, c_z): standard normals drawn in blocks of 16 rows
   (``randn(rows, N, c_z)`` per block), float32.  Chain layouts add +1.0 to
   every channel of Z[i, j] when residues i and j belong to the same chain.
   Then Z is rounded to the storage dtype (bf16: round-to-nearest-even).
2. Wq, Wk, Wv, Wg: each (H*d, c_z) = randn * c_z**-0.5.
3. Wb: (H, c_z) = randn * c_z**-0.5.
4. Wo: (c_z, H*d) = randn * (H*d)**-0.5.
5. The key mask (only for "random" masks): residue r is masked when
   ``rand(N)[r] < p``; if that masks every residue, residue 0 is re-enabled.

LayerNorm gamma = 1, beta = 0; the gate and output biases are zero.  All
weights are rounded to the storage dtype like Z.

The five named workloads stand in for the protein lengths the pages measure
on (CASP14/CASP16 targets of 100 to 6,879 residues, and multi-chain
assemblies), which are not available here.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

C_Z, HEADS, HEAD_DIM = 128, 4, 32


@dataclass
class Workload:
    name: str
    N: int
    dtype: str                     # "f32" or "bf16"
    orientations: tuple
    seed: int
    mask: str = "none"             # "none" | "tail:<n>" | "random:<p>" | "all" | "first:<n>"
    chains: tuple = ()             # chain lengths, summing to N, for the intra-chain offset
    chain_offset: float = 1.0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    0: Workload("tiny_f32_N64", 64, "f32", ("starting",), 0),
    1: Workload("bf16_N384_tailmask38", 384, "bf16", ("starting", "ending"), 1, mask="tail:38"),
    2: Workload("bf16_N768_3chains", 768, "bf16", ("starting", "ending"), 2,
                chains=(256, 256, 256)),
    3: Workload("bf16_N1536", 1536, "bf16", ("starting", "ending"), 3),
    4: Workload("bf16_N4096_mask5pct", 4096, "bf16", ("starting", "ending"), 4,
                mask="random:0.05"),
}


@dataclass
class Inputs:
    Z: torch.Tensor          # (N, N, c_z), storage dtype, CPU
    mask: torch.Tensor | None  # (N,) uint8, 1 = valid key; None = all valid
    gamma: torch.Tensor
    beta: torch.Tensor
    Wq: torch.Tensor
    Wk: torch.Tensor
    Wv: torch.Tensor
    Wg: torch.Tensor
    bg: torch.Tensor
    Wb: torch.Tensor
    Wo: torch.Tensor
    bo: torch.Tensor

    @property
    def N(self) -> int:
        return int(self.Z.shape[0])

    @property
    def dtype(self) -> torch.dtype:
        return self.Z.dtype

    def weights(self) -> dict:
        return dict(gamma=self.gamma, beta=self.beta, Wq=self.Wq, Wk=self.Wk, Wv=self.Wv,
                    Wg=self.Wg, bg=self.bg, Wb=self.Wb, Wo=self.Wo, bo=self.bo)


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def draw_z(N: int, gen: torch.Generator, c_z: int = C_Z, block_rows: int = 16) -> torch.Tensor:
    z = torch.empty((N, N, c_z), dtype=torch.float32)
    for a0 in range(0, N, block_rows):
        a1 = min(N, a0 + block_rows)
        z[a0:a1] = torch.randn((a1 - a0, N, c_z), generator=gen, dtype=torch.float32)
    return z


def make_mask(kind: str, N: int, gen: torch.Generator) -> torch.Tensor | None:
    if kind == "none":
        return None
    m = torch.ones(N, dtype=torch.uint8)
    if kind == "all":
        m.zero_()
    elif kind.startswith("tail:"):
        n = int(kind.split(":")[1])
        m[N - n:] = 0
    elif kind.startswith("first:"):
        n = int(kind.split(":")[1])
        m[:n] = 0
    elif kind.startswith("random:"):
        p = float(kind.split(":")[1])
        drop = torch.rand(N, generator=gen) < p
        m[drop] = 0
        if int(m.sum()) == 0:
            m[0] = 1
    else:
        raise ValueError(f"unknown mask kind {kind!r}")
    return m


def make_inputs(N: int, dtype: str = "bf16", seed: int = 0, mask: str = "none",
                chains: tuple = (), chain_offset: float = 1.0, c_z: int = C_Z,
                H: int = HEADS, d: int = HEAD_DIM) -> Inputs:
    gen = torch.Generator().manual_seed(seed)
    z = draw_z(N, gen, c_z)
    if chains:
        assert sum(chains) == N, "chain lengths must sum to N"
        start = 0
        for length in chains:
            z[start:start + length, start:start + length, :] += chain_offset
            start += length
    HD = H * d
    wq = torch.randn((HD, c_z), generator=gen) * c_z ** -0.5
    wk = torch.randn((HD, c_z), generator=gen) * c_z ** -0.5
    wv = torch.randn((HD, c_z), generator=gen) * c_z ** -0.5
    wg = torch.randn((HD, c_z), generator=gen) * c_z ** -0.5
    wb = torch.randn((H, c_z), generator=gen) * c_z ** -0.5
    wo = torch.randn((c_z, HD), generator=gen) * HD ** -0.5
    m = make_mask(mask, N, gen)
    td = _torch_dtype(dtype)
    return Inputs(
        Z=z.to(td), mask=m,
        gamma=torch.ones(c_z).to(td), beta=torch.zeros(c_z).to(td),
        Wq=wq.to(td), Wk=wk.to(td), Wv=wv.to(td), Wg=wg.to(td),
        bg=torch.zeros(HD).to(td), Wb=wb.to(td), Wo=wo.to(td), bo=torch.zeros(c_z).to(td))


def workload_inputs(index: int) -> Inputs:
    w = WORKLOADS[index]
    return make_inputs(w.N, w.dtype, w.seed, w.mask, w.chains, w.chain_offset)
