"""cp_usp_attention_static: the unified attention for callers that cannot
allocate device memory (for example a plugin running inside another engine's
execute hook, where a cudaMalloc would synchronise the device and is not
allowed).  Its workspace is the library's fixed device array instead of a
caller buffer, so it must give the same results as cp_usp_attention, call
after call, with the array keeping the previous call's contents.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import context_attention_dits_cp_b200 as cp
from context_attention_dits_cp_b200 import binding as bd
from context_attention_dits_cp_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL_OUT, TOL_LSE = 2e-2, 1e-3   # the bf16 tolerances of the parity tests


def _shards(seed, B, S, H, D, G):
    q, k, v = wl.make_qkv(B, H, S, D, torch.bfloat16, seed)
    return [wl.sequence_shards(t, G).cuda() for t in (q, k, v)]


def test_static_scratch_matches_workspace_version_twice(cuda_ok):
    # shards of 250 tokens: not a multiple of 128, so the composition goes
    # through its workspace (the fixed array for the static entry point)
    B, S, H, D, R, U = 2, 1000, 8, 128, 2, 2
    need = bd.usp_workspace_bytes(B, S, H, D, torch.bfloat16, torch.float32, R, U)
    assert 0 < need <= bd.USP_STATIC_SCRATCH_BYTES
    # two calls in a row on different inputs: the second must not see the
    # first call's leftovers in the shared array
    for seed in (31, 32):
        q, k, v = _shards(seed, B, S, H, D, R * U)
        ref_o, ref_l = cp.usp_attention(q, k, v, R, U)
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        bd.usp_attention_static(q, k, v, R, U, out=out, lse=lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all() and torch.isfinite(lse).all()
        assert (out - ref_o).abs().max().item() <= TOL_OUT
        assert (lse - ref_l).abs().max().item() <= TOL_LSE
    assert cp.last_device_error() == 0


def _np(t):
    return t.detach().cpu().float().numpy().astype(np.float64)


def test_static_scratch_empty_call_is_the_set_up(cuda_ok):
    """A call with no batch does only the per-device set-up and launches
    nothing: the way to make the first call outside a capture or hook."""
    e = torch.empty((4, 0, 64, 8, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((4, 0, 64, 8, 128), dtype=torch.float32, device="cuda")
    bd.usp_attention_static(e, e, e, 2, 2, out=o, lse=None)
    torch.cuda.synchronize()
    assert cp.last_device_error() == 0


@pytest.mark.parametrize("B,S,H,R,U", [(1, 1024, 8, 2, 2),    # shards of 256: no workspace
                                       (1, 6000, 8, 2, 2)])   # shards of 1500: 92 % of the array
def test_static_scratch_fused_and_near_limit(cuda_ok, B, S, H, R, U):
    D = 128
    need = bd.usp_workspace_bytes(B, S, H, D, torch.bfloat16, torch.float32, R, U)
    assert need <= bd.USP_STATIC_SCRATCH_BYTES
    assert (need == 0) == (S // (R * U) % 128 == 0)
    q, k, v = wl.make_qkv(B, H, S, D, torch.bfloat16, 33, "kscale")
    sh = [wl.sequence_shards(t, R * U).cuda() for t in (q, k, v)]
    ref_o, ref_l = cp.usp_attention(*sh, R, U)
    for _ in range(2):
        out = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        bd.usp_attention_static(*sh, R, U, out=out, lse=lse)
        torch.cuda.synchronize()
        assert (out - ref_o).abs().max().item() <= TOL_OUT
        assert (lse - ref_l).abs().max().item() <= TOL_LSE
    # and against the oracle, back in token order
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    o_tok = out.cpu().transpose(0, 1).reshape(B, S, H, D)
    assert np.abs(_np(o_tok) - ro).max() <= TOL_OUT
    assert np.abs(_np(lse) - rl).max() <= TOL_LSE
    assert cp.last_device_error() == 0
