"""Seeded synthetic workloads for the context-parallel attention hot path.

This module only *draws* inputs.  It holds none of the method's arithmetic
(no scores, softmax, merge or permutation), so both the CPU oracle and the
CUDA path can read the same tensors from it without sharing any code that
computes a result.

Workload shapes follow the diffusion-transformer attention the diffusers
context-parallelism guide benchmarks (FLUX.1-dev at 1024x1024: 4096 image +
512 text tokens, 24 heads of 128; see the guide's benchmark tables).  The
FLUX weights are not available, so seeded Gaussian tensors of those shapes
stand in for the activations.

Recipe (identical for every caller):
  * generator: ``torch.Generator().manual_seed(seed)`` on the CPU;
  * draw order: q, k, v as fp32 ``randn`` of shape [B, S, H, D] (layout
    BSHD), then the workload's extra structure, then one cast to the
    workload dtype;
  * structure ``"kscale"``: every key token is multiplied by one draw of
    U[0.5, 2] shared across heads and channels;
  * structure ``"outliers"``: every q and k entry is independently replaced,
    with probability 0.01, by +8 or -8 (sign equiprobable);
  * chunking: ``ring_chunk_lengths`` (ceil(S/R)-sized chunks, last shorter).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    dtype: str            # "f32" or "bf16"
    ring_degree: int      # R
    ulysses_degree: int   # U
    structure: str        # "plain", "kscale", "outliers"
    seed: int

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def flops(self) -> float:
        """Algorithmic attention FLOPs, 4*B*H*S^2*D (QK^T and PV, 2 each)."""
        return 4.0 * self.B * self.H * self.S * self.S * self.D


# The five workloads: index 0 is the small case the oracle finishes in
# seconds; index 1 is the FLUX-shaped joint attention the headline metric is
# quoted on.
WORKLOADS: Tuple[Workload, ...] = (
    Workload("tiny_ring_f32", 1, 2, 256, 64, "f32", 2, 1, "plain", 1000),
    Workload("flux_joint_ring4", 1, 24, 4608, 128, "bf16", 4, 1, "kscale", 1001),
    Workload("hires_dit_ring8", 1, 24, 16384, 128, "bf16", 8, 1, "outliers", 1002),
    Workload("video_ring_anything8", 1, 40, 32761, 128, "bf16", 8, 1, "plain", 1003),
    Workload("ulysses4_unified2x2", 2, 24, 8192, 128, "bf16", 2, 4, "plain", 1004),
)


def workload(name: str) -> Workload:
    for w in WORKLOADS:
        if w.name == name:
            return w
    raise KeyError(name)


def ring_chunk_lengths(S: int, R: int) -> List[int]:
    """Chunk lengths of a sequence of S tokens split over a ring of R ranks.

    Plain reading of the Ring Anything section of the diffusers
    context-parallelism guide (any sequence length is accepted): each rank
    holds ceil(S/R) tokens and the last ranks hold what is left, so
    S=32761, R=8 gives 7 x 4096 + 4089.  When R does not fit (e.g. S=5,
    R=4 gives 2,2,1,0) trailing ranks hold empty chunks.
    """
    if S < 0 or R < 1:
        raise ValueError("need S >= 0 and R >= 1")
    c = -(-S // R) if S > 0 else 0
    out = []
    left = S
    for _ in range(R):
        n = min(c, left)
        out.append(n)
        left -= n
    return out


def chunk_offsets(lengths: List[int]) -> List[int]:
    """Prefix offsets [0, l0, l0+l1, ...] of a list of chunk lengths."""
    offs = [0]
    for n in lengths:
        offs.append(offs[-1] + int(n))
    return offs


def make_qkv(B: int, H: int, S: int, D: int, dtype: torch.dtype, seed: int,
             structure: str = "plain", S_kv: Optional[int] = None):
    """Seeded q, k, v in layout [B, S, H, D] on the CPU.

    ``S_kv`` (default S) lets k/v have a different length from q.
    """
    S_kv = S if S_kv is None else S_kv
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn((B, S, H, D), generator=g, dtype=torch.float32)
    k = torch.randn((B, S_kv, H, D), generator=g, dtype=torch.float32)
    v = torch.randn((B, S_kv, H, D), generator=g, dtype=torch.float32)
    if structure == "kscale":
        s = torch.rand((B, S_kv, 1, 1), generator=g, dtype=torch.float32) * 1.5 + 0.5
        k = k * s
    elif structure == "outliers":
        for t in (q, k):
            hit = torch.rand(t.shape, generator=g) < 0.01
            sign = torch.where(torch.rand(t.shape, generator=g) < 0.5, -8.0, 8.0)
            t.copy_(torch.where(hit, sign, t))
    elif structure != "plain":
        raise ValueError(f"unknown structure {structure!r}")
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_workload_inputs(w: Workload):
    """q, k, v for a named workload (CPU tensors, layout [B, S, H, D])."""
    return make_qkv(w.B, w.H, w.S, w.D, w.torch_dtype, w.seed, w.structure)


def sequence_shards(x: torch.Tensor, degree: int) -> torch.Tensor:
    """Split [B, S, H, D] into the per-rank sequence shards a launcher hands
    out: rank p holds tokens [p*S/U, (p+1)*S/U).  Returned shard-major as one
    contiguous [U, B, S/U, H, D] tensor (what U ranks hold between them)."""
    B, S, H, D = x.shape
    if S % degree:
        raise ValueError("S must divide by the degree")
    return x.reshape(B, degree, S // degree, H, D).transpose(0, 1).contiguous()
