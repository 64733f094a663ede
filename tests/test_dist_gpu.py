"""The multi-rank module on the GPU with real NCCL and the CUDA kernels, as a
single rank (one GPU per rank; a one-GPU machine holds one rank): the all-gather,
the local-chunk-first merge, the Ulysses packing and all-to-alls all run,
and the results match one-shot attention.  The two-rank host logic is
covered on CPU ranks in test_dist_gloo.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from context_attention_dits_cp_b200 import dist as cpd
from context_attention_dits_cp_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def one_rank(cuda_ok):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    cpu = dist.new_group(backend="gloo")
    yield cpu
    dist.destroy_process_group()


def _np(t):
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_ring_allgather_one_rank(one_rank, dtype):
    q, k, v = wl.make_qkv(1, 3, 200, 128, dtype, 81, "kscale", S_kv=333)
    out, lse = cpd.ring_attention_allgather(q.cuda(), k.cuda(), v.cuda(), cpu_group=one_rank)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    tol = (2e-2, 1e-3) if dtype == torch.bfloat16 else (1e-4, 1e-4)
    assert np.abs(_np(out) - ro).max() <= tol[0] and np.abs(_np(lse) - rl).max() <= tol[1]


def test_ulysses_all_to_all_one_rank(one_rank):
    q, k, v = wl.make_qkv(2, 4, 256, 64, torch.bfloat16, 82)
    out, lse = cpd.ulysses_attention_all_to_all(q.cuda(), k.cuda(), v.cuda(), cpu_group=one_rank,
                                                want_lse=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(_np(q), _np(k), _np(v))
    assert np.abs(_np(out) - ro).max() <= 2e-2 and np.abs(_np(lse) - rl).max() <= 1e-3


def test_unified_2d_one_rank(one_rank):
    q, k, v = wl.make_qkv(2, 4, 300, 128, torch.bfloat16, 83)
    g = dist.group.WORLD
    out = cpd.usp_attention_2d(q.cuda(), k.cuda(), v.cuda(), g, g, one_rank, one_rank)
    torch.cuda.synchronize()
    ro, _ = oracle.attention(_np(q), _np(k), _np(v))
    assert np.abs(_np(out) - ro).max() <= 2e-2
