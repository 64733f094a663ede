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
* same guide, §Ulysses Anything Attention (and ContextParallelConfig
  ``ulysses_anything``): sequence lengths and head counts that the degree
  does not divide are accepted; ring_degree must be 1.

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


# ---------------------------------------------------------------- Ulysses Anything
def uneven_offsets(n: int, degree: int):
    """Offsets [0, ..., n] of `degree` ranks holding ceil(n/degree) items
    each, the last ranks holding what is left (possibly nothing).  The guide's
    Ulysses Anything section accepts sequence lengths and head counts that
    the degree does not divide; this even-as-possible split is the plain
    reading (the same rule as the Ring Anything chunks)."""
    c = -(-n // degree) if n > 0 else 0
    offs = [0]
    for _ in range(degree):
        offs.append(min(n, offs[-1] + c))
    return offs


def ulysses_anything_permute(x, B: int, H: int, D: int, seq_offsets, head_offsets,
                             direction: int) -> np.ndarray:
    """Ulysses Anything all-to-all on flat per-rank buffers.

    Sequence side: the concatenation of U rank buffers, rank p holding
    [B, s_p, H, D] with s_p = seq_offsets[p+1] - seq_offsets[p].
    Head side: the concatenation of U rank buffers, rank q holding
    [B, S, h_q, D] (all S tokens in order) with h_q from head_offsets.
    direction 0: y[q][b, off_p + s, h', d] = x[p][b, s, hoff_q + h', d];
    direction 1 is the exact inverse.  Pure data movement.
    """
    U = len(seq_offsets) - 1
    S = seq_offsets[-1]
    x = np.asarray(x).reshape(-1)
    y = np.empty_like(x)
    for q in range(U):
        h0, h1 = head_offsets[q], head_offsets[q + 1]
        hq = h1 - h0
        ybase = B * S * h0 * D
        for p in range(U):
            s0, s1 = seq_offsets[p], seq_offsets[p + 1]
            sp = s1 - s0
            xbase = B * s0 * H * D
            seq_blk = (slice(xbase, xbase + B * sp * H * D), (B, sp, H, D))
            head_blk = (slice(ybase, ybase + B * S * hq * D), (B, S, hq, D))
            if direction == SEQ_TO_HEAD:
                src = x[seq_blk[0]].reshape(seq_blk[1])
                y[head_blk[0]].reshape(head_blk[1])[:, s0:s1] = src[:, :, h0:h1]
            else:
                src = x[head_blk[0]].reshape(head_blk[1])
                y[seq_blk[0]].reshape(seq_blk[1])[:, :, h0:h1] = src[:, s0:s1]
    return y


def ulysses_anything_attention(q_flat, k_flat, v_flat, B: int, H: int, D: int, seq_offsets,
                               head_offsets, scale: Optional[float] = None):
    """Ulysses Anything (ring_degree 1): all-to-all to uneven head groups,
    attention of every head group over the whole sequence, inverse
    all-to-all.  Returns the flat sequence-sharded output and the lse of
    every query as [B, H, S] (token order), float64."""
    S = seq_offsets[-1]
    U = len(seq_offsets) - 1
    yq, yk, yv = (ulysses_anything_permute(np.asarray(t, dtype=np.float64), B, H, D,
                                           seq_offsets, head_offsets, SEQ_TO_HEAD)
                  for t in (q_flat, k_flat, v_flat))
    yo = np.empty_like(yq)
    lse = np.full((B, H, S), -np.inf)
    for q in range(U):
        h0, h1 = head_offsets[q], head_offsets[q + 1]
        hq = h1 - h0
        sl = slice(B * S * h0 * D, B * S * h1 * D)
        o, l = attention_partial(yq[sl].reshape(B, S, hq, D), yk[sl].reshape(B, S, hq, D),
                                 yv[sl].reshape(B, S, hq, D), scale)
        yo[sl] = o.reshape(-1)
        lse[:, h0:h1] = l
    out = ulysses_anything_permute(yo, B, H, D, seq_offsets, head_offsets, HEAD_TO_SEQ)
    return out, lse
