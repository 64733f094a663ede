"""Oracle: Ulysses all-to-all index map and the unified (Ulysses x Ring) path.

Test infrastructure only (see the package docstring).

Sources, by page and section:

* diffusers context-parallelism guide, §Ulysses Attention: a first
  all-to-all regroups the data so that each GPU holds every token for a
  subset of the heads; attention runs per head subset; a second all-to-all
  regroups the result by token.  The variant table requires S and H to be
  divisible by ``ulysses_degree``.
* same guide, §Unified Attention: all-to-all, then Ring Attention on the
  result, then the inverse all-to-all; the GPUs form a 2-D grid of
  ``ulysses_degree * ring_degree`` devices, each in one Ulysses group and
  one Ring group.
* diffusers parallelism API page, §ContextParallelConfig ``mesh``: the mesh
  dimensions are named ("ring", "ulysses", ...) in that order.

Readings (the pages give no index map): shards are held rank-major as one
[U, B, S/U, H, D] tensor; head group q is the contiguous heads
[q*H/U, (q+1)*H/U); the sequence is reassembled in source-rank order.  In
the unified grid, rank g = r*U + u (ring outer, Ulysses inner, following the
mesh dimension order) holds sequence shard g.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .attention import attention_partial, lse_merge

SEQ_TO_HEAD = 0
HEAD_TO_SEQ = 1


def ulysses_permute(x: np.ndarray, degree: int, direction: int) -> np.ndarray:
    """The Ulysses all-to-all, block by block.

    direction 0 (sequence shards -> head shards):
        x: [U, B, S/U, H, D]  ->  y: [U, B, S, H/U, D]
        y[q, b, p*S/U + s, h', d] = x[p, b, s, q*H/U + h', d]
    direction 1 is the exact inverse (head shards -> sequence shards).
    Pure data movement: values are copied bit for bit.
    """
    U = int(degree)
    x = np.asarray(x)
    if direction == SEQ_TO_HEAD:
        Ux, B, Sl, H, D = x.shape
        if Ux != U or H % U:
            raise ValueError("need x.shape[0] == degree and H % degree == 0")
        Hg = H // U
        y = np.empty((U, B, Sl * U, Hg, D), dtype=x.dtype)
        for q in range(U):              # destination rank: head group q
            for p in range(U):          # source rank: sequence shard p
                y[q, :, p * Sl:(p + 1) * Sl] = x[p, :, :, q * Hg:(q + 1) * Hg]
        return y
    if direction == HEAD_TO_SEQ:
        Uy, B, S, Hg, D = x.shape
        if Uy != U or S % U:
            raise ValueError("need y.shape[0] == degree and S % degree == 0")
        Sl = S // U
        out = np.empty((U, B, Sl, Hg * U, D), dtype=x.dtype)
        for p in range(U):              # destination rank: sequence shard p
            for q in range(U):          # source rank: head group q
                out[p, :, :, q * Hg:(q + 1) * Hg] = x[q, :, p * Sl:(p + 1) * Sl]
        return out
    raise ValueError("direction must be 0 (seq->head) or 1 (head->seq)")


def ulysses_permute_bruteforce(x: np.ndarray, degree: int, direction: int) -> np.ndarray:
    """Element-by-element Python loops over the same index map (tiny inputs)."""
    U = int(degree)
    x = np.asarray(x)
    if direction == SEQ_TO_HEAD:
        _, B, Sl, H, D = x.shape
        Hg = H // U
        y = np.empty((U, B, Sl * U, Hg, D), dtype=x.dtype)
        for p in range(U):
            for b in range(B):
                for s in range(Sl):
                    for h in range(H):
                        for d in range(D):
                            y[h // Hg, b, p * Sl + s, h % Hg, d] = x[p, b, s, h, d]
        return y
    _, B, S, Hg, D = x.shape
    Sl = S // U
    out = np.empty((U, B, Sl, Hg * U, D), dtype=x.dtype)
    for q in range(U):
        for b in range(B):
            for t in range(S):
                for hh in range(Hg):
                    for d in range(D):
                        out[t // Sl, b, t % Sl, q * Hg + hh, d] = x[q, b, t, hh, d]
    return out


def usp_attention(q_shards, k_shards, v_shards, ring_degree: int, ulysses_degree: int,
                  scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Unified sequence parallelism, emulated rank by rank.

    Inputs are the sequence shards of R*U ranks, [R*U, B, S/(R*U), H, D];
    rank g = r*U + u.  Steps, in the guide's order:
      1. within each Ulysses group r (ranks r*U .. r*U+U-1): all-to-all,
         sequence shards -> head groups; rank (r, u) then holds tokens
         [r*S/R, (r+1)*S/R) of head group u;
      2. within each Ring group u: rank (r, u) attends its Q to the K/V block
         of every ring peer r' (arriving in ring order r, r+1, ...), one
         partial per block, merged as it arrives;
      3. the inverse all-to-all within each Ulysses group.
    Returns the output shards [R*U, B, S/(R*U), H, D] and the lse of every
    query as one [B, H, S] array (token order), both float64.
    """
    R, U = int(ring_degree), int(ulysses_degree)
    qs, ks, vs = (np.asarray(t, dtype=np.float64) for t in (q_shards, k_shards, v_shards))
    G, B, Sg, H, D = qs.shape
    if G != R * U:
        raise ValueError("need R*U shards")
    Hg = H // U
    SR = Sg * U                              # tokens per ring block
    # step 1: Ulysses all-to-all inside every group r
    yq = [ulysses_permute(qs[r * U:(r + 1) * U], U, SEQ_TO_HEAD) for r in range(R)]
    yk = [ulysses_permute(ks[r * U:(r + 1) * U], U, SEQ_TO_HEAD) for r in range(R)]
    yv = [ulysses_permute(vs[r * U:(r + 1) * U], U, SEQ_TO_HEAD) for r in range(R)]
    # step 2: ring inside every group u
    o = [np.zeros((U, B, SR, Hg, D)) for _ in range(R)]
    lse = np.full((B, H, R * SR), -np.inf)
    for u in range(U):
        for r in range(R):
            acc_o = np.zeros((B, SR, Hg, D))
            acc_l = np.full((B, Hg, SR), -np.inf)
            for step in range(R):
                rp = (r + step) % R
                o_c, l_c = attention_partial(yq[r][u], yk[rp][u], yv[rp][u], scale)
                acc_o, acc_l = lse_merge(acc_o, acc_l, o_c, l_c)
            o[r][u] = acc_o
            lse[:, u * Hg:(u + 1) * Hg, r * SR:(r + 1) * SR] = acc_l
    # step 3: inverse all-to-all inside every group r
    out = np.concatenate([ulysses_permute(o[r], U, HEAD_TO_SEQ) for r in range(R)], axis=0)
    return out, lse
