"""Oracle: softmax attention, per-chunk partials and their merge (fp64 NumPy).

Test infrastructure only (see the package docstring).

Sources, by page and section:

* diffusers context-parallelism guide, §Ring Attention: every rank attends
  its local Q to each K/V block as the blocks travel round the ring; after a
  full round each rank has seen the K/V of every token.  The ring therefore
  computes exactly full attention, only in pieces -- so the oracle of the
  whole path is one-shot attention over the whole key sequence.
* diffusers parallelism API page, §ContextParallelConfig, ``convert_to_fp32``:
  the per-block output and LSE are converted to float32 and combined.  The
  pages print no merge equation; the plain reading is the log-sum-exp merge
  of two normalised partial softmaxes (written out in ``lse_merge``).
* same guide, §Ring Anything Attention: padded K/V is trimmed back to each
  block's true length before attention, i.e. padding never contributes.

Conventions (the pages fix none of them, plain reading):
  layout [B, S, H, D] for q/k/v/out, [B, H, S] for lse, natural-log lse,
  default scale 1/sqrt(D), non-causal, no mask.  Inputs are upcast to float64
  exactly (bf16 values are representable in float64).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

_ROW_BLOCK = 512  # query rows per block: bounds memory, changes no result


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _scale(D: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


def attention(q, k, v, scale: Optional[float] = None,
              rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One-shot softmax attention, the plain definition.

    For every batch b, head h and query i:
        s_j  = scale * sum_d q[b,i,h,d] * k[b,j,h,d]      (all keys j)
        m    = max_j s_j
        l    = sum_j exp(s_j - m)
        out  = sum_j exp(s_j - m) * v[b,j,h,:] / l
        lse  = m + ln(l)
    Returns out [B, S_q, H, D] and lse [B, H, S_q] in float64.  With no keys
    (S_kv == 0) the output is 0 and the lse is -inf (the empty softmax).

    ``rows`` (optional) restricts the computation to those query indices;
    the returned arrays then have len(rows) in place of S_q.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, S_q, H, D = q.shape
    S_kv = k.shape[1]
    sc = _scale(D, scale)
    if rows is not None:
        q = q[:, np.asarray(rows, dtype=np.int64)]
        S_q = q.shape[1]
    out = np.zeros((B, S_q, H, v.shape[3]), dtype=np.float64)
    lse = np.full((B, H, S_q), -np.inf, dtype=np.float64)
    if S_kv == 0 or S_q == 0:
        return out, lse
    for b in range(B):
        for h in range(H):
            kh = k[b, :, h, :]                   # [S_kv, D]
            vh = v[b, :, h, :]                   # [S_kv, Dv]
            for i0 in range(0, S_q, _ROW_BLOCK):
                qh = q[b, i0:i0 + _ROW_BLOCK, h, :]          # [n, D]
                s = sc * (qh @ kh.T)                          # [n, S_kv]
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                l = p.sum(axis=1, keepdims=True)
                out[b, i0:i0 + _ROW_BLOCK, h, :] = (p @ vh) / l
                lse[b, h, i0:i0 + _ROW_BLOCK] = (m + np.log(l))[:, 0]
    return out, lse


def attention_partial(q, k_chunk, v_chunk, scale: Optional[float] = None,
                      rows: Optional[np.ndarray] = None):
    """One ring step: attention of the local Q against ONE K/V chunk.

    The partial is normalised within the chunk (its own softmax) and carries
    that chunk's lse; an empty chunk gives (0, -inf), the merge identity.
    """
    D = _f64(q).shape[3]
    return attention(q, k_chunk, v_chunk, _scale(D, scale), rows=rows)


def lse_merge(out_acc, lse_acc, out_i, lse_i) -> Tuple[np.ndarray, np.ndarray]:
    """Merge two normalised partial softmax results (out [B,S,H,D], lse [B,H,S]).

    With a = lse_acc, b = lse_i per row:
        lse' = max(a, b) + ln(1 + exp(-|a - b|))
        out' = exp(a - lse') * out_acc + exp(b - lse') * out_i
    (0, -inf) is the identity; when both rows are -inf the accumulator is
    kept.  This is ln(e^a + e^b) written so that nothing overflows.
    """
    out_acc, lse_acc = _f64(out_acc), _f64(lse_acc)
    out_i, lse_i = _f64(out_i), _f64(lse_i)
    a, b = lse_acc, lse_i
    both_empty = np.isneginf(a) & np.isneginf(b)
    m = np.maximum(a, b)
    with np.errstate(invalid="ignore"):
        d = np.where(both_empty, 0.0, np.abs(a - b))
    new = m + np.log1p(np.exp(-d))
    with np.errstate(invalid="ignore"):
        wa = np.where(both_empty, 1.0, np.exp(a - new))
        wb = np.where(both_empty, 0.0, np.exp(b - new))
    new = np.where(both_empty, a, new)
    # weights are per (b, h, s); outputs are per (b, s, h, :)
    wa_o = np.transpose(wa, (0, 2, 1))[..., None]
    wb_o = np.transpose(wb, (0, 2, 1))[..., None]
    return wa_o * out_acc + wb_o * out_i, new


def ring_chunk_offsets(S: int, R: int) -> List[int]:
    """Offsets [0, ..., S] of R ring chunks of ceil(S/R) tokens, last shorter.

    The Ring Anything section accepts any sequence length; the plainest
    reading is an even split where the final ranks hold the remainder
    (S=32761, R=8 -> 7 x 4096 + 4089).  Trailing chunks may be empty.
    """
    c = -(-S // R) if S > 0 else 0
    offs = [0]
    for _ in range(R):
        offs.append(min(S, offs[-1] + c))
    return offs


def ring_attention(q, k, v, chunk_offsets: Sequence[int],
                   scale: Optional[float] = None, order: Optional[Sequence[int]] = None,
                   rows: Optional[np.ndarray] = None):
    """The literal ring walk: one partial per K/V chunk, merged in turn.

    ``order`` is the order in which chunks arrive (a ring rank r sees chunk
    r first); any order gives the same result up to rounding.
    """
    q = _f64(q)
    B, S_q, H, D = q.shape
    nq = S_q if rows is None else len(rows)
    out = np.zeros((B, nq, H, _f64(v).shape[3]))
    lse = np.full((B, H, nq), -np.inf)
    n = len(chunk_offsets) - 1
    for c in (range(n) if order is None else order):
        lo, hi = chunk_offsets[c], chunk_offsets[c + 1]
        o_c, l_c = attention_partial(q, _f64(k)[:, lo:hi], _f64(v)[:, lo:hi], scale, rows)
        out, lse = lse_merge(out, lse, o_c, l_c)
    return out, lse


def attention_bruteforce(q, k, v, scale: Optional[float] = None):
    """Pure-Python loops over every (b, h, i, j, d); for tiny inputs only.

    Uses math.fsum / math.exp / math.log (no NumPy arithmetic) so that it
    checks the vectorised oracle by an independent route.
    """
    q, k, v = _f64(q).tolist(), _f64(k).tolist(), _f64(v).tolist()
    B, S_q, H, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    S_kv = len(k[0])
    Dv = len(v[0][0][0]) if S_kv else D
    sc = _scale(D, scale)
    out = [[[[0.0] * Dv for _ in range(H)] for _ in range(S_q)] for _ in range(B)]
    lse = [[[-math.inf] * S_q for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            for i in range(S_q):
                if S_kv == 0:
                    continue
                s = [sc * math.fsum(q[b][i][h][d] * k[b][j][h][d] for d in range(D))
                     for j in range(S_kv)]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                l = math.fsum(w)
                for d in range(Dv):
                    out[b][i][h][d] = math.fsum(w[j] * v[b][j][h][d] for j in range(S_kv)) / l
                lse[b][h][i] = m + math.log(l)
    return np.array(out, dtype=np.float64), np.array(lse, dtype=np.float64)
