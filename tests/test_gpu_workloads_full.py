"""The five workloads at full size, in the launch configuration the benchmark
times, compared element by element with the CPU fp64 oracle.

* tiny ring (fp32, 2 chunks), FLUX joint attention (the plain ring walk with
  fp32 and with bf16 output, the literal per-chunk walk and the gathered Ring
  Anything layout) and both
  Ulysses / unified paths (R 1 x U 4 and R 2 x U 2): every query row of every
  head.
* the head-dim-64 case the benchmark also times (FLUX token count, 48 heads
  of 64): every row of every head.
* high-res 16k (8 chunks, +-8 outliers) and video 32761 (7 x 4096 + 4089):
  the oracle would need minutes for every row, so each head is checked on a
  seeded stratified sample -- four rows in every 128-row query tile (16k),
  three in every tile (video) -- plus every row of the first and of the last
  query tile, which is where the ragged tail lies.  Rows are independent,
  so the check is exact for the rows it covers.

Tolerances are those of the method's statement: fp32 inputs 1e-4 max-abs on
out and lse; bf16 inputs 2e-2 on out and 1e-3 on lse (diffusers
context-parallelism guide, §Ring Attention: the ring computes full
attention, so one-shot attention is the reference at any chunking).

The oracle runs head by head on a thread pool (NumPy releases the GIL in
its matmul and ufunc loops; BLAS is held to one thread per worker), which
changes nothing it computes.
"""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch
from threadpoolctl import threadpool_limits

import oracle
import context_attention_dits_cp_b200 as cp
from context_attention_dits_cp_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {torch.float32: (1e-4, 1e-4), torch.bfloat16: (2e-2, 1e-3)}


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def oracle_by_head(q, k, v, rows=None):
    """oracle.attention over [B, S, H, D] float64 arrays, one (b, h) per task."""
    B, S, H, D = q.shape
    n = S if rows is None else len(rows)
    out = np.empty((B, n, H, v.shape[3]))
    lse = np.empty((B, H, n))

    def job(bh):
        b, h = divmod(bh, H)
        o, l = oracle.attention(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h:h + 1],
                                v[b:b + 1, :, h:h + 1], rows=rows)
        out[b, :, h] = o[0, :, 0]
        lse[b, h] = l[0, 0]

    workers = max(1, len(os.sched_getaffinity(0)))
    with threadpool_limits(1):
        with cf.ThreadPoolExecutor(workers) as ex:
            list(ex.map(job, range(B * H)))
    return out, lse


def stratified_rows(S, per_tile, seed, tile=128):
    """per_tile seeded rows of every `tile`-row query tile, plus every row of
    the first and the last tile (the ragged tail)."""
    rng = np.random.default_rng(seed)
    rows = [np.arange(0, min(tile, S))]
    last0 = ((S - 1) // 256) * 256          # the last 256-row unit of the kernel
    rows.append(np.arange(last0, S))
    for t0 in range(0, S, tile):
        n = min(tile, S - t0)
        rows.append(t0 + rng.choice(n, size=min(per_tile, n), replace=False))
    return np.unique(np.concatenate(rows))


def check(out, lse, ref_out, ref_lse, dtype, rows=None):
    tol_o, tol_l = TOL[dtype]
    o, lz = _np(out), _np(lse)
    if rows is not None:
        o, lz = o[:, rows], lz[:, :, rows]
    assert o.shape == ref_out.shape and lz.shape == ref_lse.shape
    assert np.isfinite(o).all() and np.isfinite(lz).all()
    eo = np.abs(o - ref_out).max()
    el = np.abs(lz - ref_lse).max()
    assert eo <= tol_o, f"out max-abs {eo:.3e} > {tol_o}"
    assert el <= tol_l, f"lse max-abs {el:.3e} > {tol_l}"
    return eo, el


_REF = {}


def _inputs(name):
    w = wl.workload(name)
    q, k, v = wl.make_workload_inputs(w)
    return w, q, k, v


def _full_reference(name):
    """One-shot oracle over every row and head of a workload (cached: the
    FLUX and Ulysses references serve several call paths)."""
    if name not in _REF:
        _, q, k, v = _inputs(name)
        _REF[name] = oracle_by_head(_np(q), _np(k), _np(v))
    return _REF[name]


def _padded_gather(t, lengths, L, pad):
    B, _, H, D = t.shape
    g = torch.full((len(lengths), B, L, H, D), pad, dtype=t.dtype)
    o = 0
    for c, n in enumerate(lengths):
        g[c, :, :n] = t[:, o:o + n]
        o += n
    return g


# ---------------------------------------------------------------- tiny, fp32
def test_tiny_ring_f32_every_row(cuda_ok):
    w, q, k, v = _inputs("tiny_ring_f32")
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    assert offs == [0, 128, 256]
    out, lse = cp.ring_attention(q.cuda(), k.cuda(), v.cuda(), offs)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    check(out, lse, ro, rl, torch.float32)


# ---------------------------------------------------------------- FLUX joint attention
def test_flux_ring4_every_row(cuda_ok):
    w, q, k, v = _inputs("flux_joint_ring4")
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    out, lse = cp.ring_attention(q.cuda(), k.cuda(), v.cuda(), offs)
    torch.cuda.synchronize()
    ro, rl = _full_reference(w.name)
    check(out, lse, ro, rl, w.torch_dtype)


def test_flux_ring4_bf16_out_every_row(cuda_ok):
    """The same walk with the output cast to bf16 in the epilogue (lse stays
    fp32); the cast adds at most half a bf16 ulp of |out| to the error."""
    w, q, k, v = _inputs("flux_joint_ring4")
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    out = torch.empty((w.B, w.S, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    out, lse = cp.ring_attention(q.cuda(), k.cuda(), v.cuda(), offs, out=out)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16
    ro, rl = _full_reference(w.name)
    check(out, lse, ro, rl, w.torch_dtype)


def test_flux_literal_per_chunk_walk_every_row(cuda_ok):
    """Chunk 0 with cp_attn_partial, chunks 1-3 folded in with
    cp_attn_partial_merge: the calls a ring rank makes as chunks arrive."""
    w, q, k, v = _inputs("flux_joint_ring4")
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out, lse = cp.attn_partial(dq, dk[:, offs[0]:offs[1]], dv[:, offs[0]:offs[1]])
    for c in range(1, w.ring_degree):
        cp.attn_partial_merge(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]], out, lse)
    torch.cuda.synchronize()
    ro, rl = _full_reference(w.name)
    check(out, lse, ro, rl, w.torch_dtype)


def test_flux_gathered_uneven_every_row(cuda_ok):
    """The FLUX keys in Ring Anything shards of 1172, 1172, 1172, 1092 padded
    to 1172: own chunk first from local memory, then the three other slots
    of the padded all-gather folded in by one gathered launch.  The padding
    holds NaN, which must never reach the result."""
    w, q, k, v = _inputs("flux_joint_ring4")
    lens = [1172, 1172, 1172, 1092]
    kg = _padded_gather(k, lens, 1172, float("nan")).cuda()
    vg = _padded_gather(v, lens, 1172, float("nan")).cuda()
    dq = q.cuda()
    out, lse = cp.attn_partial(dq, kg[0, :, :lens[0]], vg[0, :, :lens[0]])
    cp.ring_attention_gathered(dq, kg, vg, lens, skip_chunk=0, out=out, lse=lse, accumulate=True)
    torch.cuda.synchronize()
    ro, rl = _full_reference(w.name)
    check(out, lse, ro, rl, w.torch_dtype)


# ---------------------------------------------------------------- long sequences, sampled rows
@pytest.mark.parametrize("name,per_tile,seed", [("hires_dit_ring8", 4, 2),
                                                ("video_ring_anything8", 3, 3)])
def test_long_workloads_stratified_rows(cuda_ok, name, per_tile, seed):
    w, q, k, v = _inputs(name)
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    out, lse = cp.ring_attention(q.cuda(), k.cuda(), v.cuda(), offs)
    torch.cuda.synchronize()
    rows = stratified_rows(w.S, per_tile, seed)
    assert len(rows) >= 512
    out, lse = out.cpu(), lse.cpu()
    ro, rl = oracle_by_head(_np(q), _np(k), _np(v), rows=rows)
    check(out, lse, ro, rl, w.torch_dtype, rows=rows)


# ---------------------------------------------------------------- Ulysses / unified
@pytest.mark.parametrize("R,U", [(1, 4), (2, 2)])
def test_ulysses_and_unified_every_row(cuda_ok, R, U):
    w, q, k, v = _inputs("ulysses4_unified2x2")
    G = R * U
    sh = lambda t: wl.sequence_shards(t, G).cuda()
    out, lse = cp.usp_attention(sh(q), sh(k), sh(v), R, U)
    torch.cuda.synchronize()
    o_full = out.cpu().transpose(0, 1).reshape(w.B, w.S, w.H, w.D)   # back to token order
    del out
    ro, rl = _full_reference(w.name)
    check(o_full, lse.cpu(), ro, rl, torch.bfloat16)


# ---------------------------------------------------------------- head dim 64
def test_head_dim_64_flux_tokens_every_row(cuda_ok):
    """The benchmark's head-dim-64 case: the FLUX token count (4608, four
    chunks of 1152) with 48 heads of 64, every row of every head."""
    q, k, v = wl.make_qkv(1, 48, 4608, 64, torch.bfloat16, 1201, "kscale")
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(4608, 4))
    out, lse = cp.ring_attention(q.cuda(), k.cuda(), v.cuda(), offs)
    torch.cuda.synchronize()
    ro, rl = oracle_by_head(_np(q), _np(k), _np(v))
    check(out, lse, ro, rl, torch.bfloat16)
