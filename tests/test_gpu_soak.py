"""Randomised soak of the attention entry points: 320 seeded ragged shapes
(bf16 and fp32, D 64 and 128, up to 6 chunks with empty ones, 1 to 1500
query rows).  For every shape the four call paths a ring rank can take -- the
fused ring walk, the per-chunk walk with the merge in the epilogue, the
gathered Ring Anything layout (NaN padding) and, for one chunk, the single
partial call -- must agree with each other; every 20th shape is also
compared with the CPU fp64 oracle.  The ring computes full attention at any
chunking (diffusers context-parallelism guide, §Ring Attention and §Ring
Anything), so the paths share one answer up to rounding order.
"""
import numpy as np
import pytest
import torch

import oracle
import context_attention_dits_cp_b200 as cp
from context_attention_dits_cp_b200 import workloads as wl

pytestmark = pytest.mark.gpu

# The method's tolerances.  Between two call paths the bf16 P is rounded
# against different running maxima, so the paths differ by up to the same
# amount each of them may differ from the exact result.
ORACLE = {torch.bfloat16: (2e-2, 1e-3), torch.float32: (1e-4, 1e-4)}
CROSS = ORACLE


def _cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        dtype = torch.float32 if rng.integers(0, 5) == 0 else torch.bfloat16
        D = int(rng.choice([64, 128]))
        B, H = int(rng.integers(1, 4)), int(rng.integers(1, 6))
        Sq = int(rng.choice([1, int(rng.integers(2, 257)), int(rng.integers(257, 1500))]))
        R = int(rng.integers(1, 7))
        Skv = int(rng.integers(1, 2000))
        cuts = np.sort(rng.integers(0, Skv + 1, size=R - 1))
        out.append((i, dtype, D, B, H, Sq, [0] + [int(c) for c in cuts] + [Skv]))
    return out


def _gather(t, lens, L):
    B, _, H, D = t.shape
    g = torch.full((len(lens), B, L, H, D), float("nan"), dtype=t.dtype, device=t.device)
    o = 0
    for c, n in enumerate(lens):
        g[c, :, :n] = t[:, o:o + n]
        o += n
    return g


def _close(a, b, tol):
    return (a.float() - b.float()).abs().max().item() <= tol


@pytest.mark.parametrize("block", range(8))
def test_call_paths_agree_on_random_shapes(cuda_ok, block):
    for i, dtype, D, B, H, Sq, offs in _cases(40, 4000 + block):
        R = len(offs) - 1
        q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 7000 + 40 * block + i, "kscale", S_kv=offs[-1])
        dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
        fo, fl = cp.ring_attention(dq, dk, dv, offs)
        wo = torch.zeros(B, Sq, H, D, device="cuda")
        wl_ = torch.full((B, H, Sq), -float("inf"), device="cuda")
        for c in range(R):
            cp.attn_partial_merge(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]], wo, wl_)
        lens = [offs[c + 1] - offs[c] for c in range(R)]
        go, gl = cp.ring_attention_gathered(dq, _gather(dk, lens, max(lens)),
                                            _gather(dv, lens, max(lens)), lens)
        po, pl = cp.attn_partial(dq, dk, dv)
        torch.cuda.synchronize()
        assert cp.last_device_error() == 0, (block, i)
        to, tl = CROSS[dtype]
        for name, (o, l) in (("walk", (wo, wl_)), ("gathered", (go, gl)), ("one chunk", (po, pl))):
            assert torch.isfinite(o).all(), (block, i, name)
            assert _close(o, fo, to) and _close(l, fl, tl), (block, i, name, offs)
        if i % 20 == 0:
            ro, rl = oracle.attention(*(t.float().numpy().astype(np.float64) for t in (q, k, v)))
            to, tl = ORACLE[dtype]
            assert np.abs(fo.cpu().double().numpy() - ro).max() <= to, (block, i)
            assert np.abs(fl.cpu().double().numpy() - rl).max() <= tl, (block, i)
