"""Seeded synthetic inputs for S²-Attn workloads.

This module holds no attention arithmetic: it only draws random numbers in a
fixed order, so that the GPU path, the tests and the CPU oracle all see the
same bf16 bytes.

Recipe (the pages measure on Llama-2 attention layers, H=32, D=128; no dataset
is involved):

* ``g = torch.Generator('cpu').manual_seed(seed)``;
* Q, K, V, dO are drawn in that order, each ``torch.randn((B, N, H, D),
  dtype=float32, generator=g)`` rounded to bfloat16 (round-to-nearest-even);
* the long-context workload then draws ``idx = torch.randperm(N,
  generator=g)[:round(0.05 N)]`` and doubles K at those token positions, for
  every batch row and head (exact in bf16) to sharpen the softmax;
* the ragged workload draws all N_padded rows; rows >= n_valid are padding
  whose random values must not affect any valid output.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

STRICT, ROLLED, DENSE_CAUSAL = 0, 1, 2
VARIANT_NAMES = {STRICT: "strict", ROLLED: "rolled", DENSE_CAUSAL: "dense_causal"}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    D: int
    G: int
    variants: tuple = (STRICT,)
    n_valid: int | None = None
    sharpen_k: bool = False
    seed: int = 0
    description: str = ""

    @property
    def valid(self) -> int:
        return self.N if self.n_valid is None else self.n_valid

    def formula_flops(self, variant: int | None = None, passes: str = "fwd+bwd") -> float:
        """Useful causal FLOPs: 2·B·H·N·G·D forward, 2.5x that backward.

        N is the valid length (useful work); the dense-causal variant uses G = N.
        """
        n = self.valid
        base = 2.0 * self.B * self.H * n * self.G * self.D
        return {"fwd": base, "bwd": 2.5 * base, "fwd+bwd": 3.5 * base}[passes]


WORKLOADS = {
    "small_n1024_g256": Workload(
        "small_n1024_g256", B=1, N=1024, H=8, D=64, G=256,
        description="B=1 H=8 N=1024 D=64 G=256 (shift 128), strict"),
    "llama7b_n8192_g2048": Workload(
        "llama7b_n8192_g2048", B=1, N=8192, H=32, D=128, G=2048, variants=(STRICT, ROLLED),
        description="Llama-2-7B attention layer: B=1 H=32 D=128 N=8192 G=2048, strict and rolled"),
    "long_n32768_g8192": Workload(
        "long_n32768_g8192", B=1, N=32768, H=32, D=128, G=8192, sharpen_k=True,
        description="B=1 H=32 D=128 N=32768 G=8192, strict, K x2 on 5% of positions"),
    # the long-context workload with 8 of its 32 heads: the same per-head work,
    # a quarter of the device memory (about 2.7 GB with the stored dS), for
    # hardware-counter captures whose per-launch bytes scale by 32 / 8
    "long_n32768_g8192_h8": Workload(
        "long_n32768_g8192_h8", B=1, N=32768, H=8, D=128, G=8192, sharpen_k=True,
        description="B=1 H=8 D=128 N=32768 G=8192, strict, K x2 on 5% of positions (counter captures)"),
    # the long-context workload at head dimension 64 (the kernels' other D)
    "long_n32768_g8192_d64": Workload(
        "long_n32768_g8192_d64", B=1, N=32768, H=32, D=64, G=8192, sharpen_k=True,
        description="B=1 H=32 D=64 N=32768 G=8192, strict, K x2 on 5% of positions"),
    "sweep_n12288_g6144": Workload("sweep_n12288_g6144", B=2, N=12288, H=32, D=128, G=6144),
    "sweep_n12288_g3072": Workload("sweep_n12288_g3072", B=2, N=12288, H=32, D=128, G=3072),
    "sweep_n12288_g2048": Workload("sweep_n12288_g2048", B=2, N=12288, H=32, D=128, G=2048),
    "sweep_n12288_g1536": Workload("sweep_n12288_g1536", B=2, N=12288, H=32, D=128, G=1536),
    "sweep_n12288_full": Workload("sweep_n12288_full", B=2, N=12288, H=32, D=128, G=12288,
                                  variants=(DENSE_CAUSAL,)),
    "ragged_n100000_g8192": Workload(
        "ragged_n100000_g8192", B=1, N=106496, H=32, D=128, G=8192, n_valid=100000,
        description="B=1 H=32 D=128 N=100000 padded to 106496, G=8192, strict"),
}


def draw(B: int, N: int, H: int, D: int, seed: int = 0, sharpen_k: bool = False,
         with_dout: bool = True) -> dict:
    """Draw Q, K, V (and dO) as CPU bf16 [B, N, H, D] tensors."""
    g = torch.Generator("cpu").manual_seed(seed)
    shape = (B, N, H, D)
    out = {}
    for name in ("q", "k", "v", "dout"):
        t = torch.randn(shape, dtype=torch.float32, generator=g).to(torch.bfloat16)
        out[name] = t
    if sharpen_k:
        n_sel = int(round(0.05 * N))
        idx = torch.randperm(N, generator=g)[:n_sel]
        out["k"][:, idx] *= 2
    if not with_dout:
        del out["dout"]
    return out


def workload_inputs(name: str) -> dict:
    w = WORKLOADS[name]
    return draw(w.B, w.N, w.H, w.D, seed=w.seed, sharpen_k=w.sharpen_k)
