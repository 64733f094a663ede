"""Parity of the CUDA path (through the C-ABI) with the CPU fp64 oracle.

Tolerances: fp32 inputs, max-abs 1e-4 on out and lse; bf16 inputs, max-abs
2e-2 on out and 1e-3 on lse; the Ulysses permutation is compared bit for bit.
Small cases span several 128-row tiles with ragged tails.  The five
full-size workloads are in test_gpu_workloads_full.py.
"""
import numpy as np
import pytest
import torch

import oracle
import context_attention_dits_cp_b200 as cp
from context_attention_dits_cp_b200 import workloads as wl
from test_gpu_workloads_full import oracle_by_head

pytestmark = pytest.mark.gpu

TOL = {torch.float32: (1e-4, 1e-4), torch.bfloat16: (2e-2, 1e-3)}


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def _dev(*ts):
    return [t.cuda() for t in ts]


def _check(out, lse, ref_out, ref_lse, dtype, rows=None):
    tol_o, tol_l = TOL[dtype]
    o = _np(out)
    lz = _np(lse)
    if rows is not None:
        o = o[:, rows]
        lz = lz[:, :, rows]
    assert np.isfinite(o).all() and np.isfinite(lz).all()
    eo = np.abs(o - ref_out).max()
    el = np.abs(lz - ref_lse).max()
    assert eo <= tol_o, f"out max-abs {eo:.3e} > {tol_o}"
    assert el <= tol_l, f"lse max-abs {el:.3e} > {tol_l}"
    return eo, el


# ---------------------------------------------------------------- Ulysses permute
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("U,B,S,H,D", [(2, 1, 8, 4, 64), (4, 2, 64, 8, 128), (3, 1, 30, 6, 64)])
def test_ulysses_permute_bit_exact(cuda_ok, dtype, U, B, S, H, D):
    x = torch.randn(U, B, S // U, H, D).to(dtype)
    y = cp.ulysses_permute(x.cuda(), U, cp.SEQ_TO_HEAD)
    torch.cuda.synchronize()
    bits = lambda t: t.cpu().view(torch.int16 if dtype == torch.bfloat16 else torch.int32).numpy()
    assert np.array_equal(bits(y), oracle.ulysses_permute(bits(x), U, 0))
    x2 = cp.ulysses_permute(y, U, cp.HEAD_TO_SEQ)
    assert np.array_equal(bits(x2), bits(x))


def test_ulysses_permute_full_size_roundtrip(cuda_ok):
    w = wl.workload("ulysses4_unified2x2")
    q, _, _ = wl.make_workload_inputs(w)
    x = wl.sequence_shards(q, 4)
    y = cp.ulysses_permute(x.cuda(), 4, cp.SEQ_TO_HEAD)
    bits = lambda t: t.cpu().view(torch.int16).numpy()
    assert np.array_equal(bits(y), oracle.ulysses_permute(bits(x), 4, 0))
    x2 = cp.ulysses_permute(y, 4, cp.HEAD_TO_SEQ)
    assert torch.equal(x2.cpu().view(torch.int16), x.view(torch.int16))


def test_ulysses_permute_into_strided_view(cuda_ok):
    U, B, S, H, D = 2, 2, 16, 4, 64
    x = torch.randn(U, B, S // U, H, D).to(torch.bfloat16).cuda()
    big = torch.zeros(U, B, 2 * S, H // U, D, dtype=torch.bfloat16, device="cuda")
    view = big[:, :, S:]
    cp.ulysses_permute(x, U, cp.SEQ_TO_HEAD, y=view)
    bits = lambda t: t.cpu().view(torch.int16).numpy()
    assert np.array_equal(bits(view), oracle.ulysses_permute(bits(x), U, 0))
    assert torch.count_nonzero(big[:, :, :S]).item() == 0


# ---------------------------------------------------------------- LSE merge
def test_lse_merge_full_size_flux_shape(cuda_ok):
    """The merge at the benchmark's shape ([1, 4608, 24, 128] fp32), every
    element compared with the oracle."""
    g = torch.Generator().manual_seed(9)
    shape, lshape = (1, 4608, 24, 128), (1, 24, 4608)
    oa, oi = torch.randn(shape, generator=g), torch.randn(shape, generator=g)
    la, li = torch.randn(lshape, generator=g) * 4, torch.randn(lshape, generator=g) * 4
    ref_o, ref_l = oracle.lse_merge(_np(oa), _np(la), _np(oi), _np(li))
    da, dla = oa.cuda(), la.cuda()
    cp.lse_merge(da, dla, oi.cuda(), li.cuda())
    torch.cuda.synchronize()
    assert np.abs(_np(da) - ref_o).max() <= 1e-5
    assert np.abs(_np(dla) - ref_l).max() <= 1e-5


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("in_dtype", [torch.float32, torch.bfloat16])
def test_lse_merge(cuda_ok, D, in_dtype):
    B, S, H = 2, 77, 3
    g = torch.Generator().manual_seed(5)
    oa = torch.randn(B, S, H, D, generator=g)
    la = torch.randn(B, H, S, generator=g) * 3
    oi = torch.randn(B, S, H, D, generator=g).to(in_dtype)
    li = torch.randn(B, H, S, generator=g) * 3
    # identity rows: empty partial on either side, and both empty
    la[0, 0, :5] = -float("inf")
    oa[0, :5, 0] = 0
    li[1, 2, 10:15] = -float("inf")
    la[1, 1, 20:23] = -float("inf")
    li[1, 1, 20:23] = -float("inf")
    oa[1, 20:23, 1] = 0
    ref_o, ref_l = oracle.lse_merge(_np(oa), _np(la), _np(oi), _np(li))
    da, dla = oa.cuda(), la.cuda()
    cp.lse_merge(da, dla, oi.cuda(), li.cuda())
    torch.cuda.synchronize()
    assert np.abs(_np(da) - ref_o).max() <= 1e-5
    lz = _np(dla)
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(lz), np.isneginf(ref_l))
    assert np.abs(lz[fin] - ref_l[fin]).max() <= 1e-5


# ---------------------------------------------------------------- attention, small
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Skv", [(1, 1), (37, 200), (300, 333), (513, 129)])
def test_attn_partial_fp32(cuda_ok, D, Sq, Skv):
    q, k, v = wl.make_qkv(2, 3, Sq, D, torch.float32, 11, S_kv=Skv)
    ro, rl = oracle.attention_partial(_np(q), _np(k), _np(v))
    out, lse = cp.attn_partial(*_dev(q, k, v))
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, torch.float32)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Skv", [(1, 1), (128, 128), (256, 384), (300, 333), (700, 129),
                                    (255, 1000)])
def test_attn_partial_bf16(cuda_ok, D, Sq, Skv):
    q, k, v = wl.make_qkv(1, 3, Sq, D, torch.bfloat16, 12, S_kv=Skv)
    ro, rl = oracle.attention_partial(_np(q), _np(k), _np(v))
    out, lse = cp.attn_partial(*_dev(q, k, v))
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_attn_partial_bf16_out_and_scale(cuda_ok, dtype):
    q, k, v = wl.make_qkv(1, 2, 200, 128, dtype, 13, S_kv=260)
    ro, rl = oracle.attention_partial(_np(q), _np(k), _np(v), scale=0.3)
    out, lse = cp.attn_partial(*_dev(q, k, v), scale=0.3, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_partial_never_reads_past_its_chunk(cuda_ok, dtype):
    """Ring Anything trims padded K/V: rows after the chunk hold NaN/1e30
    and must not leak into the partial."""
    q, k, v = wl.make_qkv(1, 2, 150, 128, dtype, 14, S_kv=300)
    kp, vp = k.clone(), v.clone()
    kp[:, 201:] = float("nan")
    vp[:, 201:] = 1e30
    ro, rl = oracle.attention_partial(_np(q), _np(k[:, :201]), _np(v[:, :201]))
    dk, dv = kp.cuda(), vp.cuda()
    out, lse = cp.attn_partial(q.cuda(), dk[:, :201], dv[:, :201])
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_empty_chunk_is_identity(cuda_ok, dtype):
    q, k, v = wl.make_qkv(1, 2, 40, 64, dtype, 15, S_kv=0)
    out, lse = cp.attn_partial(*_dev(q, k, v))
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
    assert torch.isneginf(lse).all()


# ---------------------------------------------------------------- ring walk, small
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("offs", [[0, 128, 256, 500], [0, 100, 100, 357, 500], [0, 500],
                                  [0, 1, 2, 3, 250, 499, 500], [0, 0, 500, 500]])
def test_ring_uneven_chunks(cuda_ok, dtype, offs):
    q, k, v = wl.make_qkv(1, 2, 260, 128, dtype, 16, S_kv=500)
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    out, lse = cp.ring_attention(*_dev(q, k, v), offs)
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fused_ring_matches_literal_walk(cuda_ok, dtype):
    """cp_ring_attention (fused merge) against cp_attn_partial + cp_lse_merge
    per chunk, in two different arrival orders."""
    q, k, v = wl.make_qkv(2, 2, 333, 64, dtype, 17, S_kv=700)
    dq, dk, dv = _dev(q, k, v)
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(700, 3))
    fo, fl = cp.ring_attention(dq, dk, dv, offs)
    for order in ([0, 1, 2], [2, 0, 1]):
        acc = torch.zeros(2, 333, 2, 64, device="cuda")
        lacc = torch.full((2, 2, 333), -float("inf"), device="cuda")
        for c in order:
            oc, lc = cp.attn_partial(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]])
            cp.lse_merge(acc, lacc, oc, lc)
        torch.cuda.synchronize()
        tol_o, tol_l = TOL[dtype]
        assert (acc - fo).abs().max().item() <= tol_o
        assert (lacc - fl).abs().max().item() <= tol_l


@pytest.mark.parametrize("B,H,Sq,Skv,D,out_dtype", [(3, 2, 300, 200, 128, torch.float32),
                                                    (2, 5, 129, 640, 64, torch.bfloat16),
                                                    (1, 1, 1000, 3, 128, torch.bfloat16),
                                                    (1, 3, 1, 1, 128, torch.float32),
                                                    (2, 1, 1, 257, 64, torch.float32)])
def test_ring_tensor_core_shapes(cuda_ok, B, H, Sq, Skv, D, out_dtype):
    """Batches, S_q != S_kv, a query view whose heads are strided (every other
    head of a wider tensor), bf16 output, no lse output, and the smallest
    cases: one query against one key, one query against a ragged tail."""
    g = torch.Generator().manual_seed(B * 100 + H)
    wide = torch.randn(B, Sq, 2 * H, D, generator=g).bfloat16()
    q = wide[:, :, ::2]                       # head stride 2*D: TMA reads it in place
    k = torch.randn(B, Skv, H, D, generator=g).bfloat16()
    v = torch.randn(B, Skv, H, D, generator=g).bfloat16()
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(Skv, 3))
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    dq = wide.cuda()[:, :, ::2]
    assert not dq.is_contiguous()
    out, lse = cp.ring_attention(dq, k.cuda(), v.cuda(), offs, out_dtype=out_dtype)
    out2, none = cp.ring_attention(dq, k.cuda(), v.cuda(), offs, out_dtype=out_dtype,
                                   want_lse=False)
    torch.cuda.synchronize()
    assert none is None
    _check(out, lse, ro, rl, torch.bfloat16)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 128)])
def test_partial_merge_walk_equals_oneshot_and_literal(cuda_ok, dtype, D):
    """A ring walk made only of cp_attn_partial_merge calls (chunks arriving
    in ring order from rank 1, with an empty chunk) equals one-shot attention
    and the partial + standalone-merge walk."""
    B, H, Sq, Skv = 2, 3, 333, 700
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 43, S_kv=Skv)
    dq, dk, dv = _dev(q, k, v)
    offs = [0, 250, 250, 500, 700]
    acc = torch.zeros(B, Sq, H, D, device="cuda")
    lacc = torch.full((B, H, Sq), -float("inf"), device="cuda")
    lit = acc.clone()
    llit = lacc.clone()
    for c in (1, 2, 3, 0):
        kc, vc = dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]]
        cp.attn_partial_merge(dq, kc, vc, acc, lacc)
        oc, lc = cp.attn_partial(dq, kc, vc)
        cp.lse_merge(lit, llit, oc, lc)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    _check(acc, lacc, ro, rl, dtype)
    tol_o, tol_l = TOL[dtype]
    assert (acc - lit).abs().max().item() <= tol_o
    assert (lacc - llit).abs().max().item() <= tol_l


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_partial_merge_into_strided_views(cuda_ok, dtype):
    """The accumulator may be a view: every other head of a wider output and
    an LSE whose rows are padded.  Entries outside the views stay untouched."""
    B, H, Sq, Skv, D = 1, 2, 300, 384, 128
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 47, S_kv=Skv)
    dq, dk, dv = _dev(q, k, v)
    big = torch.full((B, Sq, 2 * H, D), 7.0, device="cuda")
    acc = big[:, :, ::2]
    acc.zero_()
    lbig = torch.full((B, H, Sq + 20), 3.0, device="cuda")
    lacc = lbig[:, :, 10:10 + Sq]
    lacc.fill_(-float("inf"))
    for lo, hi in ((256, 384), (0, 256)):
        cp.attn_partial_merge(dq, dk[:, lo:hi], dv[:, lo:hi], acc, lacc)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    _check(acc, lacc, ro, rl, dtype)
    assert bool((big[:, :, 1::2] == 7.0).all())
    assert bool((lbig[:, :, :10] == 3.0).all()) and bool((lbig[:, :, 10 + Sq:] == 3.0).all())


def _padded_gather(t, lengths, L, pad):
    """[R, B, L, H, D] slots of a padded all-gather of the chunks of t
    (rank order), padding rows set to `pad`."""
    B, _, H, D = t.shape
    g = torch.full((len(lengths), B, L, H, D), pad, dtype=t.dtype)
    o = 0
    for c, n in enumerate(lengths):
        g[c, :, :n] = t[:, o:o + n]
        o += n
    return g


@pytest.mark.parametrize("vpad", [float("nan"), float("inf"), 1e30])
@pytest.mark.parametrize("dtype,D,B", [(torch.bfloat16, 128, 1), (torch.bfloat16, 64, 2),
                                       (torch.float32, 128, 2)])
def test_gathered_ring_trims_padding_in_place(cuda_ok, dtype, D, B, vpad):
    """Ring Anything over a padded all-gather: chunk c is the first
    lengths[c] rows of slot c; the padding (NaN in K; NaN, Inf or 1e30 in V)
    never contributes.  Whole walk, and own chunk first then the rest merged
    in."""
    lengths, L, H, Sq = [300, 0, 257, 128], 320, 3, 290
    Skv = sum(lengths)
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 61, "kscale", S_kv=Skv)
    kg = _padded_gather(k, lengths, L, float("nan")).cuda()
    vg = _padded_gather(v, lengths, L, vpad).cuda()
    dq = q.cuda()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    out, lse = cp.ring_attention_gathered(dq, kg, vg, lengths)
    torch.cuda.synchronize()
    _check(out, lse, ro, rl, dtype)
    # rank 2 folds in its own chunk first, then the others from the gather
    r = 2
    o0 = sum(lengths[:r])
    acc, lacc = cp.attn_partial(dq, k[:, o0:o0 + lengths[r]].cuda(), v[:, o0:o0 + lengths[r]].cuda())
    cp.ring_attention_gathered(dq, kg, vg, lengths, skip_chunk=r, out=acc, lse=lacc,
                               accumulate=True)
    torch.cuda.synchronize()
    _check(acc, lacc, ro, rl, dtype)


def test_gathered_ring_empty_cases(cuda_ok):
    """No chunk left: accumulate leaves the accumulator alone, otherwise the
    result is attention to no keys (0, -inf)."""
    q, k, v = wl.make_qkv(1, 2, 130, 128, torch.bfloat16, 62, S_kv=40)
    kg = _padded_gather(k, [40, 0], 64, 0.0).cuda()
    vg = _padded_gather(v, [40, 0], 64, 0.0).cuda()
    acc = torch.randn(1, 130, 2, 128, device="cuda")
    lacc = torch.randn(1, 2, 130, device="cuda")
    a0, l0 = acc.clone(), lacc.clone()
    cp.ring_attention_gathered(q.cuda(), kg, vg, [40, 0], skip_chunk=0, out=acc, lse=lacc,
                               accumulate=True)
    out, lse = cp.ring_attention_gathered(q.cuda(), kg, vg, [40, 0], skip_chunk=0)
    torch.cuda.synchronize()
    assert torch.equal(acc, a0) and torch.equal(lacc, l0)
    assert bool((out == 0).all()) and bool(torch.isneginf(lse).all())


def test_constant_v_and_zero_q_closed_forms(cuda_ok):
    g = torch.Generator().manual_seed(18)
    S = 400
    k = torch.randn(1, S, 2, 128, generator=g).bfloat16()
    c = torch.randn(128, generator=g).bfloat16()
    v = c.expand(1, S, 2, 128).contiguous()
    q = torch.randn(1, 300, 2, 128, generator=g).bfloat16()
    out, _ = cp.ring_attention(*_dev(q, k, v), [0, 150, 400])
    assert (out.cpu() - c.float()).abs().max().item() <= 2e-2
    qz = torch.zeros_like(q)
    out, lse = cp.ring_attention(*_dev(qz, k, torch.randn(1, S, 2, 128, generator=g).bfloat16()),
                                 [0, 400])
    assert (lse.cpu() - np.log(S)).abs().max().item() <= 1e-3


# ---------------------------------------------------------------- unified, small
@pytest.mark.parametrize("S,D,dtype", [(512, 128, torch.bfloat16),    # shards of 128: fused
                                       (600, 64, torch.bfloat16),     # shards of 150: permute path
                                       (1000, 128, torch.bfloat16),   # shards of 250: permute path
                                       (264, 64, torch.float32)])     # fp32: permute path
def test_unified_small_matches_oracle_usp(cuda_ok, S, D, dtype):
    """The emulated grid against the oracle's own rank-by-rank emulation,
    through both the fused (tensor-map) path and the permute path."""
    B, H, R, U = 2, 8, 2, 2
    q, k, v = wl.make_qkv(B, H, S, D, dtype, 19)
    sh = lambda t: wl.sequence_shards(t, R * U)
    out, lse = cp.usp_attention(*_dev(sh(q), sh(k), sh(v)), R, U)
    torch.cuda.synchronize()
    ro, rl = oracle.usp_attention(_np(sh(q)), _np(sh(k)), _np(sh(v)), R, U)
    tol_o, tol_l = TOL[dtype]
    assert np.abs(_np(out) - ro).max() <= tol_o
    assert np.abs(_np(lse) - rl).max() <= tol_l


# ---------------------------------------------------------------- Ulysses Anything
def _flat(full, offs):
    return torch.cat([full[:, offs[p]:offs[p + 1]].reshape(-1) for p in range(len(offs) - 1)])


def _unflat(flat, offs, B, H, D):
    parts, pos = [], 0
    for p in range(len(offs) - 1):
        n = B * (offs[p + 1] - offs[p]) * H * D
        parts.append(flat[pos:pos + n].reshape(B, offs[p + 1] - offs[p], H, D))
        pos += n
    return torch.cat(parts, dim=1)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,S,H,D,U", [(1, 4481, 24, 128, 4),   # FLUX at 1008x1008
                                       (2, 37, 24, 64, 5),      # uneven heads 5,5,5,5,4
                                       (1, 10, 3, 64, 4)])      # an empty head group
def test_ulysses_anything_permute_bit_exact(cuda_ok, dtype, B, S, H, D, U):
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    x = _flat(torch.randn(B, S, H, D).to(dtype), so)
    y = cp.ulysses_anything_permute(x.cuda(), B, H, D, so, ho, cp.SEQ_TO_HEAD)
    torch.cuda.synchronize()
    iv = torch.int16 if dtype == torch.bfloat16 else torch.int32
    bits = lambda t: t.cpu().view(iv).numpy()
    assert np.array_equal(bits(y), oracle.ulysses_anything_permute(bits(x), B, H, D, so, ho, 0))
    x2 = cp.ulysses_anything_permute(y, B, H, D, so, ho, cp.HEAD_TO_SEQ)
    assert np.array_equal(bits(x2), bits(x))


def test_ulysses_anything_attention_1008px_every_row(cuda_ok):
    """FLUX at 1008x1008: 3969 image + 512 text tokens on 4 ranks, where the
    guide's plain Ulysses fails and Ulysses Anything runs."""
    B, S, H, D, U = 1, 4481, 24, 128, 4
    q, k, v = wl.make_qkv(B, H, S, D, torch.bfloat16, 41, "kscale")
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    out, lse = cp.ulysses_anything_attention(*(_flat(t, so).cuda() for t in (q, k, v)),
                                             B, H, D, so, ho)
    torch.cuda.synchronize()
    o_full = _unflat(out.cpu(), so, B, H, D)
    ro, rl = oracle_by_head(_np(q), _np(k), _np(v))     # every row of every head
    _check(o_full, lse.cpu(), ro, rl, torch.bfloat16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("S,H,U", [(300, 6, 4), (129, 24, 5)])
def test_ulysses_anything_attention_matches_oracle(cuda_ok, dtype, S, H, U):
    B, D = 2, 64
    q, k, v = wl.make_qkv(B, H, S, D, dtype, 42)
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    fq, fk, fv = (_flat(t, so) for t in (q, k, v))
    out, lse = cp.ulysses_anything_attention(fq.cuda(), fk.cuda(), fv.cuda(), B, H, D, so, ho)
    torch.cuda.synchronize()
    ro, rl = oracle.ulysses_anything_attention(_np(fq), _np(fk), _np(fv), B, H, D, so, ho)
    tol_o, tol_l = TOL[dtype]
    assert np.abs(_np(out) - ro).max() <= tol_o
    assert np.abs(_np(lse) - rl).max() <= tol_l


# ---------------------------------------------------------------- failure surfacing
def test_bounded_wait_reports_timeout(cuda_ok):
    assert cp.last_device_error() == 0
    st = cp.selftest_wait_timeout(4096)
    assert cp.binding.STATUS[st] == "CP_ERR_TIMEOUT"
    assert cp.last_device_error() == 0   # cleared
    # the context is still usable
    q, k, v = wl.make_qkv(1, 1, 64, 64, torch.bfloat16, 20)
    out, _ = cp.attn_partial(*_dev(q, k, v))
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()


# ---------------------------------------------------------------- seeded random sweep
def _sweep_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        dtype = [torch.bfloat16, torch.float32][int(rng.integers(0, 4) == 0)]
        D = int(rng.choice([64, 128]))
        B, H = int(rng.integers(1, 4)), int(rng.integers(1, 5))
        Sq = int(rng.choice([1, int(rng.integers(2, 129)), int(rng.integers(129, 700))]))
        R = int(rng.integers(1, 6))
        cuts = np.sort(rng.integers(0, int(rng.integers(1, 900)) + 1, size=R - 1))
        Skv = int(cuts[-1]) if R > 1 and rng.random() < 0.3 else int(rng.integers(1, 900))
        cuts = np.clip(cuts, 0, Skv)
        offs = [0] + [int(c) for c in cuts] + [Skv]
        path = ["ring", "walk", "merge_walk", "gathered"][i % 4]
        cases.append((i, dtype, D, B, H, Sq, offs, path))
    return cases


@pytest.mark.parametrize("case", _sweep_cases(24, 2026), ids=lambda c: f"{c[0]}-{c[7]}")
def test_seeded_random_sweep(cuda_ok, case):
    """Random shapes, chunkings (empty chunks included) and call paths, each
    against one-shot attention."""
    i, dtype, D, B, H, Sq, offs, path = case
    Skv = offs[-1]
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 500 + i, "kscale", S_kv=Skv)
    dq, dk, dv = _dev(q, k, v)
    R = len(offs) - 1
    if path == "ring":
        out, lse = cp.ring_attention(dq, dk, dv, offs)
    elif path == "walk":
        out = torch.zeros(B, Sq, H, D, device="cuda")
        lse = torch.full((B, H, Sq), -float("inf"), device="cuda")
        for c in range(R):
            oc, lc = cp.attn_partial(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]])
            cp.lse_merge(out, lse, oc, lc)
    elif path == "merge_walk":
        out = torch.zeros(B, Sq, H, D, device="cuda")
        lse = torch.full((B, H, Sq), -float("inf"), device="cuda")
        for c in reversed(range(R)):
            cp.attn_partial_merge(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]],
                                  out, lse)
    else:
        lens = [offs[c + 1] - offs[c] for c in range(R)]
        L = max(max(lens), 1)
        kg = _padded_gather(k, lens, L, float("nan")).cuda()
        vg = _padded_gather(v, lens, L, [float("nan"), float("inf")][i % 8 // 4]).cuda()
        out, lse = cp.ring_attention_gathered(dq, kg, vg, lens)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    if Skv == 0:
        assert bool((out == 0).all()) and bool(torch.isneginf(lse).all())
        return
    _check(out, lse, ro, rl, dtype)
