"""Seeded synthetic inputs for the SALA attention hot path.

This module only draws random numbers and allocates tensors; it contains none of
the method's arithmetic, so the CUDA path and the fp64 oracle can both be fed
from it.  Every tensor is drawn from a ``torch.Generator`` seeded per workload,
in a fixed documented order, as N(0, 1) in fp32 and then cast to the workload
dtype (the cast is the only transformation).  The shapes follow the workloads
the MiniCPM-SALA pages measure (64K-1M-token prefill, batched decode).

Workloads (names used by the tests and the benchmark):

* ``lightning_small``  -- Lightning prefill, B1 H2 D64 T1024, fp32, chunk 64, seed 1001
* ``lightning_32k``    -- Lightning prefill, B1 H32 D128 T32768, bf16, chunk 128, seed 1002
* ``lightning_decode`` -- decode, B64 H32 D128, fp32 state N(0,1)/64, 256 steps, seed 1003
* ``sparse_128k``      -- sparse prefill, B1 T131072 Hq32 Hkv2 D128, bf16, seed 1004
* ``hybrid``           -- 8 layers (Lightning at 0,1,3,4,5,7; sparse at 2,6),
                          B1 H32 D128 bf16, layer l drawn from seed 1005 + l
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import torch

HYBRID_SPARSE_LAYERS = (2, 6)
HYBRID_NUM_LAYERS = 8


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, gen: torch.Generator, dtype=torch.bfloat16, device="cpu", scale: float = 1.0):
    """N(0, scale^2) drawn in fp32 from `gen`, then cast to `dtype`."""
    x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


@dataclass
class LightningInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: Optional[torch.Tensor]


def lightning_inputs(B, T, H, D, seed, dtype=torch.bfloat16, device="cpu", gate=True):
    """q, k, v, g of shape [B, T, H, D], drawn in that order."""
    gen = generator(seed, device)
    q = randn((B, T, H, D), gen, dtype, device)
    k = randn((B, T, H, D), gen, dtype, device)
    v = randn((B, T, H, D), gen, dtype, device)
    g = randn((B, T, H, D), gen, dtype, device) if gate else None
    return LightningInputs(q, k, v, g)


@dataclass
class SparseInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: Optional[torch.Tensor]


def sparse_inputs(B, T, Hq, Hkv, D, seed, dtype=torch.bfloat16, device="cpu", gate=False):
    """q [B,T,Hq,D], k and v [B,T,Hkv,D], optional gate g [B,T,Hq,D], in that order."""
    gen = generator(seed, device)
    q = randn((B, T, Hq, D), gen, dtype, device)
    k = randn((B, T, Hkv, D), gen, dtype, device)
    v = randn((B, T, Hkv, D), gen, dtype, device)
    g = randn((B, T, Hq, D), gen, dtype, device) if gate else None
    return SparseInputs(q, k, v, g)


def decode_state(B, H, D, seed, device="cpu"):
    """Decode initial state S ~ N(0,1)/sqrt(4096) in fp32, [B, H, D, D]."""
    gen = generator(seed, device)
    return randn((B, H, D, D), gen, torch.float32, device, scale=1.0 / 64.0)


def decode_tokens(B, H, D, seed, step, dtype=torch.bfloat16, device="cpu"):
    """One decode step's q, k, v, g [B, H, D]; step s uses seed * 1000 + 1 + s."""
    gen = generator(int(seed) * 1000 + 1 + int(step), device)
    q = randn((B, H, D), gen, dtype, device)
    k = randn((B, H, D), gen, dtype, device)
    v = randn((B, H, D), gen, dtype, device)
    g = randn((B, H, D), gen, dtype, device)
    return q, k, v, g


def hybrid_layer_inputs(layer: int, T: int, B=1, H=32, Hkv=2, D=128, device="cpu",
                        dtype=torch.bfloat16, seed=1005):
    """Inputs for layer `layer` of the 8-layer hybrid stack (seed 1005 + layer).
    Lightning layers: q,k,v,g [B,T,H,D].  Sparse layers: q,g [B,T,H,D], k,v [B,T,Hkv,D]."""
    s = seed + layer
    if layer in HYBRID_SPARSE_LAYERS:
        return sparse_inputs(B, T, H, Hkv, D, s, dtype, device, gate=True)
    return lightning_inputs(B, T, H, D, s, dtype, device, gate=True)
