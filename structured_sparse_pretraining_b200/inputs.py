"""Seeded synthetic inputs and workload shapes.

This module only draws random numbers and describes shapes; it holds none of
the layer's arithmetic.  It is the one piece shared by the CUDA path's tests
and bench and by the CPU oracle's tests, so both sides see identical inputs.

Recipe: every tensor is drawn as float32 N(0, std) from its own
``torch.Generator`` (CPU, or CUDA for the bench's large inputs) seeded with
``seed * 1000 + 10 * layer + slot`` (slot order X=0, W=1, L=2, R=3, dY=4),
then rounded to bf16 by torch's conversion.  Shapes and standard deviations
follow the five workloads below, which mirror the model families the SLoPe
pages evaluate (GPT-2, BERT-Large, OPT; SLoPe technical summary
(gist.science), §4 "Experimental Results").  No dataset is involved.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

SLOT = {"X": 0, "W": 1, "L": 2, "R": 3, "dY": 4, "dW": 5}  # dW: a gradient fed to the optimizer step


@dataclass(frozen=True)
class Layer:
    in_features: int
    out_features: int


@dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[Layer, ...]
    tokens: int
    rank: int            # adapter rank as the workload states it
    rank_stored: int     # rank as stored on the GPU (zero-padded to a multiple of 8)
    std_x: float = 1.0
    std_w: float = 0.02
    std_l: float = 0.02
    std_r: float = 1e-3
    std_dy: float = 1e-2
    fwd_sweep: Tuple[int, ...] = field(default_factory=tuple)
    reprune_each_step: bool = False


def _L(*pairs):
    return tuple(Layer(i, o) for i, o in pairs)


WORKLOADS = {
    # single layer, CPU-seconds size
    "C1": Workload("slope-linear-512x512-T256-r8", _L((512, 512)), 256, 8, 8),
    # GPT-2-small MLP block, d=768, 8 x 1024 tokens, rank 16 (~2.1% of d)
    "C2": Workload("gpt2s-mlp-d768-T8192-r16", _L((768, 3072), (3072, 768)), 8192, 16, 16),
    # BERT-Large encoder linears, d=1024, 32 x 512 tokens, rank 64
    "C3": Workload("bertL-linears-d1024-T16384-r64",
                   _L((1024, 3072), (1024, 1024), (1024, 4096), (4096, 1024)), 16384, 64, 64),
    # OPT-13B decoder linears, d=5120, 4 x 1024 tokens, rank 64, re-prune every step
    "C4": Workload("opt13b-linears-d5120-T4096-r64",
                   _L((5120, 15360), (5120, 5120), (5120, 20480), (20480, 5120)), 4096, 64, 64,
                   std_w=0.01, reprune_each_step=True),
    # OPT-66B decoder linears, d=9216, rank 92 (1% of d) stored zero-padded to 96
    "C5": Workload("opt66b-linears-d9216-T8192-r92",
                   _L((9216, 27648), (9216, 9216), (9216, 36864), (36864, 9216)), 8192, 92, 96,
                   std_w=0.01, fwd_sweep=(1, 16, 128, 2048)),
}


def generator(seed: int, layer: int, slot: str, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + 10 * layer + SLOT[slot])
    return g


def normal_bf16(shape, std: float, seed: int, layer: int, slot: str, device="cpu") -> torch.Tensor:
    """float32 N(0, std) rounded to bf16, from a dedicated seeded generator."""
    g = generator(seed, layer, slot, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def layer_inputs(w: Workload, layer: int, seed: int = 0, tokens: Optional[int] = None,
                 rank: Optional[int] = None, device="cpu", std_r: Optional[float] = None):
    """Inputs of one layer: dict of bf16 tensors X [T,in], W [out,in], L [in,r],
    R [r,out], dY [T,out].  ``rank`` overrides the stored rank (0 = no adapter).
    ``std_r`` overrides R's spread (parity tests use a larger one so that the
    adapter term is exercised)."""
    lay = w.layers[layer]
    T = w.tokens if tokens is None else tokens
    r = w.rank if rank is None else rank
    d = dict(
        X=normal_bf16((T, lay.in_features), w.std_x, seed, layer, "X", device),
        W=normal_bf16((lay.out_features, lay.in_features), w.std_w, seed, layer, "W", device),
        dY=normal_bf16((T, lay.out_features), w.std_dy, seed, layer, "dY", device),
    )
    if r:
        d["L"] = normal_bf16((lay.in_features, r), w.std_l, seed, layer, "L", device)
        d["R"] = normal_bf16((r, lay.out_features), w.std_r if std_r is None else std_r,
                             seed, layer, "R", device)
    else:
        d["L"] = None
        d["R"] = None
    return d


def pad_rank(L: Optional[torch.Tensor], R: Optional[torch.Tensor], r_stored: int):
    """Zero-pad an adapter of rank r to r_stored columns of L / rows of R.
    The padded products are exactly zero, so the layer's outputs do not change."""
    if L is None:
        return None, None
    r = L.shape[1]
    if r == r_stored:
        return L, R
    Lp = torch.zeros(L.shape[0], r_stored, dtype=L.dtype, device=L.device)
    Rp = torch.zeros(r_stored, R.shape[1], dtype=R.dtype, device=R.device)
    Lp[:, :r] = L
    Rp[:r, :] = R
    return Lp, Rp


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (no arithmetic)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def sample_rows(n: int, count: int, seed: int = 1234) -> List[int]:
    """Deterministic sorted sample of row indices, always including the first
    and last rows (the ragged tail)."""
    if count >= n:
        return list(range(n))
    g = torch.Generator()
    g.manual_seed(seed + n)
    idx = torch.randperm(n, generator=g)[: max(count - 2, 0)].tolist()
    return sorted(set(idx) | {0, n - 1})
