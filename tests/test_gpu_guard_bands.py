"""Guard bands around every output of every entry point, on small ragged
shapes (1 to 300 tokens): each output lives inside a larger buffer filled
with a NaN of a distinctive bit pattern, and after the call every element
outside the output (before it, after it, and between the heads of a
head-strided view) must still hold that exact pattern.  Workspaces are
guarded the same way past the size the library asks for.

The same checks run twice: on the release library in this process, and on
the bounds-checking build (libcpattn_debug.so, every device-side index
tested against its tensor's extent) in a child process, where in addition
no bounds check may fire.  compute-sanitizer is not available on this
hardware pool; these two together stand in for it.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import context_attention_dits_cp_b200 as cp
from context_attention_dits_cp_b200 import binding as bd
from context_attention_dits_cp_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GUARD = 4160          # guard elements on each side (keeps the outputs 16-byte aligned)
POISON = {torch.float32: (torch.int32, 0x7FC0BEEF), torch.bfloat16: (torch.int16, 0x7FC1)}
TOL = {torch.float32: (1e-4, 1e-4), torch.bfloat16: (2e-2, 1e-3)}


class Guarded:
    """A tensor of `shape` inside a poisoned buffer.  `every` > 1 places the
    tensor's heads (dim 2 of a 4-D [B, S, H, D] output) every `every` heads
    of a wider row, so the gaps between them are guarded too."""

    def __init__(self, shape, dtype, every=1, fill=None):
        self.dtype = dtype
        ib, pat = POISON[dtype]
        shape = list(shape)
        if every > 1:
            wide = shape[:2] + [shape[2] * every] + shape[3:]
            n = int(np.prod(wide))
        else:
            n = int(np.prod(shape))
        self.buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
        self.buf.view(ib).fill_(pat)
        body = self.buf[GUARD:GUARD + n]
        if every > 1:
            self.view = body.view(wide)[:, :, ::every]
        else:
            self.view = body.view(shape)
        self.mask = torch.ones(n + 2 * GUARD, dtype=torch.bool, device="cuda")
        # the elements the view covers are not guard
        idx = torch.arange(n, device="cuda").view(wide if every > 1 else shape)
        if every > 1:
            idx = idx[:, :, ::every]
        self.mask[GUARD + idx.reshape(-1)] = False
        if fill is not None:
            self.view.fill_(fill)

    def intact(self):
        ib, pat = POISON[self.dtype]
        g = self.buf.view(ib)[self.mask]
        return bool((g == pat).all())


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def _close(out, lse, ro, rl, dtype):
    tol_o, tol_l = TOL[dtype]
    o = _np(out)
    assert np.isfinite(o).all()
    assert np.abs(o - ro).max() <= tol_o
    if lse is not None:
        assert np.abs(_np(lse) - rl).max() <= tol_l


def _no_device_error():
    st = cp.last_device_error()
    assert st == 0, bd.STATUS.get(st, st)


CASES = [(torch.bfloat16, 128, 1, 37), (torch.bfloat16, 64, 129, 300),
         (torch.float32, 64, 300, 129), (torch.bfloat16, 128, 300, 1)]


@pytest.mark.parametrize("dtype,D,Sq,Skv", CASES)
def test_ring_partial_and_merge_outputs_stay_inside(cuda_ok, dtype, D, Sq, Skv):
    B, H = 2, 3
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 90 + Sq, "kscale", S_kv=Skv)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(Skv, 3))
    for out_dtype in (torch.float32, torch.bfloat16):
        o = Guarded((B, Sq, H, D), out_dtype, every=2)
        l = Guarded((B, H, Sq), torch.float32)
        cp.ring_attention(dq, dk, dv, offs, out=o.view, lse=l.view)
        torch.cuda.synchronize()
        assert o.intact() and l.intact()
        _close(o.view, l.view, ro, rl, torch.bfloat16 if out_dtype == torch.bfloat16 else dtype)
        o = Guarded((B, Sq, H, D), out_dtype)
        l = Guarded((B, H, Sq), torch.float32)
        cp.attn_partial(dq, dk, dv, out=o.view, lse=l.view)
        torch.cuda.synchronize()
        assert o.intact() and l.intact()
    # the per-chunk walk into a guarded fp32 accumulator
    acc = Guarded((B, Sq, H, D), torch.float32, every=3, fill=0.0)
    lacc = Guarded((B, H, Sq), torch.float32, fill=-float("inf"))
    for c in (2, 0, 1):
        cp.attn_partial_merge(dq, dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]],
                              acc.view, lacc.view)
    torch.cuda.synchronize()
    assert acc.intact() and lacc.intact()
    _close(acc.view, lacc.view, ro, rl, dtype)
    _no_device_error()


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_gathered_ring_outputs_stay_inside(cuda_ok, dtype, D):
    B, H, Sq = 1, 2, 130
    lengths, L = [77, 0, 130, 1], 131
    q, k, v = wl.make_qkv(B, H, Sq, D, dtype, 95, S_kv=sum(lengths))
    kg = torch.full((len(lengths), B, L, H, D), float("nan"), dtype=dtype)
    vg = torch.full((len(lengths), B, L, H, D), float("nan"), dtype=dtype)
    o0 = 0
    for c, n in enumerate(lengths):
        kg[c, :, :n] = k[:, o0:o0 + n]
        vg[c, :, :n] = v[:, o0:o0 + n]
        o0 += n
    dq, kg, vg = q.cuda(), kg.cuda(), vg.cuda()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    o = Guarded((B, Sq, H, D), torch.float32, every=2)
    l = Guarded((B, H, Sq), torch.float32)
    cp.ring_attention_gathered(dq, kg, vg, lengths, out=o.view, lse=l.view)
    torch.cuda.synchronize()
    assert o.intact() and l.intact()
    _close(o.view, l.view, ro, rl, dtype)
    acc = Guarded((B, Sq, H, D), torch.float32, fill=0.0)
    lacc = Guarded((B, H, Sq), torch.float32, fill=-float("inf"))
    cp.ring_attention_gathered(dq, kg, vg, lengths, out=acc.view, lse=lacc.view, accumulate=True)
    torch.cuda.synchronize()
    assert acc.intact() and lacc.intact()
    _close(acc.view, lacc.view, ro, rl, dtype)
    _no_device_error()


@pytest.mark.parametrize("D,S", [(64, 1), (128, 37), (64, 300)])
def test_lse_merge_stays_inside(cuda_ok, D, S):
    B, H = 2, 3
    g = torch.Generator().manual_seed(S)
    oa = torch.randn(B, S, H, D, generator=g)
    la = torch.randn(B, H, S, generator=g)
    oi = torch.randn(B, S, H, D, generator=g)
    li = torch.randn(B, H, S, generator=g)
    ro, rl = oracle.lse_merge(_np(oa), _np(la), _np(oi), _np(li))
    acc = Guarded((B, S, H, D), torch.float32, every=2)
    acc.view.copy_(oa)
    lacc = Guarded((B, H, S), torch.float32)
    lacc.view.copy_(la)
    cp.lse_merge(acc.view, lacc.view, oi.cuda(), li.cuda())
    torch.cuda.synchronize()
    assert acc.intact() and lacc.intact()
    assert np.abs(_np(acc.view) - ro).max() <= 1e-5
    assert np.abs(_np(lacc.view) - rl).max() <= 1e-5
    _no_device_error()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("U,B,S,H,D", [(2, 1, 2, 2, 64), (3, 2, 150, 6, 64), (4, 1, 300, 8, 128)])
def test_permutes_stay_inside(cuda_ok, dtype, U, B, S, H, D):
    x = torch.randn(U, B, S // U, H, D).to(dtype).cuda()
    y = Guarded((U, B, S, H // U, D), dtype)
    cp.ulysses_permute(x, U, cp.SEQ_TO_HEAD, y=y.view)
    x2 = Guarded((U, B, S // U, H, D), dtype)
    cp.ulysses_permute(y.view, U, cp.HEAD_TO_SEQ, y=x2.view)
    torch.cuda.synchronize()
    assert y.intact() and x2.intact()
    assert torch.equal(x2.view, x)
    # the uneven permutation on flat rank buffers
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    n = B * S * H * D
    xf = torch.randn(n).to(dtype).cuda()
    yf = Guarded((n,), dtype)
    cp.ulysses_anything_permute(xf, B, H, D, so, ho, cp.SEQ_TO_HEAD, y=yf.view)
    xb = Guarded((n,), dtype)
    cp.ulysses_anything_permute(yf.view, B, H, D, so, ho, cp.HEAD_TO_SEQ, y=xb.view)
    torch.cuda.synchronize()
    assert yf.intact() and xb.intact()
    assert torch.equal(xb.view, xf)
    _no_device_error()


@pytest.mark.parametrize("S,D,dtype", [(512, 128, torch.bfloat16),   # fused: no workspace
                                       (300, 64, torch.bfloat16),    # shards of 75
                                       (264, 64, torch.float32)])
def test_unified_and_workspace_stay_inside(cuda_ok, S, D, dtype):
    B, H, R, U = 2, 4, 2, 2
    q, k, v = wl.make_qkv(B, H, S, D, dtype, 97, S_kv=S)
    sh = [wl.sequence_shards(t, R * U).cuda() for t in (q, k, v)]
    ro, rl = oracle.usp_attention(*(_np(wl.sequence_shards(t, R * U)) for t in (q, k, v)), R, U)
    need = cp.usp_workspace_bytes(B, S, H, D, dtype, torch.float32, R, U)
    wbuf = torch.empty(need + 2 * 4096, dtype=torch.uint8, device="cuda")
    wbuf.fill_(0xA5)
    o = Guarded(tuple(sh[0].shape), torch.float32)
    l = Guarded((B, H, S), torch.float32)
    cp.usp_attention(*sh, R, U, out=o.view, lse=l.view,
                     workspace=wbuf[4096:4096 + need] if need else None)
    torch.cuda.synchronize()
    assert o.intact() and l.intact()
    assert bool((wbuf[:4096] == 0xA5).all()) and bool((wbuf[4096 + need:] == 0xA5).all())
    assert np.abs(_np(o.view) - ro).max() <= TOL[dtype][0]
    assert np.abs(_np(l.view) - rl).max() <= TOL[dtype][1]
    # the allocation-free variant writes the same outputs, nothing around them
    o2 = Guarded(tuple(sh[0].shape), torch.float32)
    l2 = Guarded((B, H, S), torch.float32)
    bd.usp_attention_static(*sh, R, U, out=o2.view, lse=l2.view)
    torch.cuda.synchronize()
    assert o2.intact() and l2.intact()
    assert (o2.view - o.view).abs().max().item() <= TOL[dtype][0]
    _no_device_error()


@pytest.mark.parametrize("B", [1, 2])
def test_ulysses_anything_attention_stays_inside(cuda_ok, B):
    S, H, D, U, dtype = 131, 6, 64, 4, torch.bfloat16
    q, k, v = wl.make_qkv(B, H, S, D, dtype, 98)
    so, ho = oracle.uneven_offsets(S, U), oracle.uneven_offsets(H, U)
    flat = lambda t: torch.cat([t[:, so[p]:so[p + 1]].reshape(-1) for p in range(U)])
    fq, fk, fv = (flat(t) for t in (q, k, v))
    ro, rl = oracle.ulysses_anything_attention(_np(fq), _np(fk), _np(fv), B, H, D, so, ho)
    need = bd.lib().cp_ulysses_anything_workspace_bytes(B, S, H, D, bd.CP_BF16, bd.CP_F32)
    wbuf = torch.full((need + 2 * 4096,), 0x5A, dtype=torch.uint8, device="cuda")
    o = Guarded((fq.numel(),), torch.float32)
    l = Guarded((B, H, S), torch.float32)
    cp.ulysses_anything_attention(fq.cuda(), fk.cuda(), fv.cuda(), B, H, D, so, ho, out=o.view,
                                  lse=l.view, workspace=wbuf[4096:4096 + need] if need else None)
    torch.cuda.synchronize()
    assert o.intact() and l.intact()
    assert bool((wbuf[:4096] == 0x5A).all()) and bool((wbuf[4096 + need:] == 0x5A).all())
    assert np.abs(_np(o.view) - ro).max() <= 2e-2
    assert np.abs(_np(l.view) - rl).max() <= 1e-3
    _no_device_error()


@pytest.mark.skipif(os.environ.get("CPATTN_GUARD_CHILD") == "1" or
                    os.environ.get("CPATTN_DEBUG") == "1",
                    reason="the bounds-checking build is loaded")
def test_bounds_selftest_is_silent_in_the_release_build(cuda_ok):
    assert not cp.is_debug_build()
    assert cp.selftest_bounds_check() == 0


@pytest.mark.skipif(os.environ.get("CPATTN_GUARD_CHILD") == "1" or
                    os.environ.get("CPATTN_DEBUG") == "1",
                    reason="no grandchildren; the whole run already uses the bounds-checking build")
def test_every_guard_band_again_on_the_bounds_checking_build(cuda_ok):
    """This file, rerun in a child process on libcpattn_debug.so: the checks
    are live (the self-test's deliberate failure is reported), and none of
    the calls above trips one."""
    path = os.path.join(ROOT, "context_attention_dits_cp_b200", "libcpattn_debug.so")
    assert os.path.exists(path)
    env = dict(os.environ, CPATTN_DEBUG="1", CPATTN_GUARD_CHILD="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p",
                        "no:cacheprovider", __file__, "-k", "not bounds_checking_build"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.skipif(os.environ.get("CPATTN_GUARD_CHILD") != "1",
                    reason="runs in the debug-build child only")
def test_debug_build_reports_a_failed_bounds_check(cuda_ok):
    assert cp.is_debug_build()
    assert bd.STATUS[cp.selftest_bounds_check()] == "CP_ERR_BOUNDS"
    assert cp.last_device_error() == 0      # read and cleared
