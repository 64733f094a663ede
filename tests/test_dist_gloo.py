"""Multi-rank context parallelism (context_attention_dits_cp_b200.dist) as
world-size-2 gloo ranks on the CPU.

The host logic runs unchanged: the shard-length exchange, the Ring Anything
padding and all-gather, the skip of the local chunk, the Ulysses packing,
all-to-alls and unpacking.  The kernel calls go to a stand-in built from the
oracle (this file), since the CUDA kernels need a GPU; the GPU side of the
same calls is covered by the parity tests.  Results are compared with
one-shot attention over the whole sequence."""
import os
import socket
import sys
import traceback

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The kernel entry points dist.py calls, computed by the fp64 oracle on
    CPU tensors (results stored as fp32, like the kernels' outputs)."""

    def __init__(self, oracle):
        self.o = oracle

    @staticmethod
    def _np(t):
        return t.detach().double().numpy()

    def attn_partial(self, q, k, v, scale=None):
        out, lse = self.o.attention_partial(self._np(q), self._np(k), self._np(v), scale)
        return torch.from_numpy(out).float(), torch.from_numpy(lse).float()

    def attn_partial_merge(self, q, k, v, out, lse, scale=None):
        oc, lc = self.o.attention_partial(self._np(q), self._np(k), self._np(v), scale)
        acc, lacc = self.o.lse_merge(self._np(out), self._np(lse), oc, lc)
        out.copy_(torch.from_numpy(acc))
        lse.copy_(torch.from_numpy(lacc))
        return out, lse

    def ring_attention_gathered(self, q, kg, vg, lengths, skip_chunk=-1, scale=None, out=None,
                                lse=None, accumulate=False):
        assert accumulate and out is not None and lse is not None
        acc, lacc = self._np(out), self._np(lse)
        for c, n in enumerate(lengths):
            if c == skip_chunk or n == 0:
                continue
            oc, lc = self.o.attention_partial(self._np(q), self._np(kg[c, :, :n]),
                                              self._np(vg[c, :, :n]), scale)
            acc, lacc = self.o.lse_merge(acc, lacc, oc, lc)
        out.copy_(torch.from_numpy(acc))
        lse.copy_(torch.from_numpy(lacc))
        return out, lse

    def ulysses_anything_permute(self, x, B, H, D, seq_off, head_off, direction, y=None):
        r = self.o.ulysses_anything_permute(x.numpy(), B, H, D, seq_off, head_off, direction)
        y.copy_(torch.from_numpy(np.ascontiguousarray(r)).reshape(y.shape))
        return y

    def ulysses_anything_attention(self, q, k, v, B, H, D, seq_off, head_off, scale=None,
                                   out=None, lse=None, want_lse=True):
        o, l = self.o.ulysses_anything_attention(self._np(q), self._np(k), self._np(v), B, H, D,
                                                 seq_off, head_off, scale)
        out.copy_(torch.from_numpy(o))
        if lse is not None:
            lse.copy_(torch.from_numpy(l))
        return out, lse

    def usp_attention(self, qs, ks, vs, R, U, scale=None, out=None, lse=None, want_lse=True):
        o, l = self.o.usp_attention(self._np(qs), self._np(ks), self._np(vs), R, U, scale)
        out.copy_(torch.from_numpy(o))
        if lse is not None:
            lse.copy_(torch.from_numpy(l))
        return out, lse


def _worker(rank, world, port, case, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=5 if case == "rank_leaves"
                                                           else 60))
        import oracle
        from context_attention_dits_cp_b200 import dist as cpd
        from context_attention_dits_cp_b200 import workloads as wl
        ops = OracleOps(oracle)
        if case in ("ring", "ring3"):
            # Ring Anything: uneven shards (and an uneven query split); over
            # three ranks one rank holds no keys at all.  Both exchanges: one
            # broadcast per slot (pipelined) and one all-gather.
            if case == "ring":
                kv_len, q_len, H, D = [37, 29], [20, 33], 3, 16
            else:
                kv_len, q_len, H, D = [21, 0, 17], [9, 12, 5], 2, 8
            qa, ka, va = wl.make_qkv(2, H, sum(q_len), D, torch.float32, 71, S_kv=sum(kv_len))
            qo, ko = sum(q_len[:rank]), sum(kv_len[:rank])
            ql = qa[:, qo:qo + q_len[rank]]
            kl = ka[:, ko:ko + kv_len[rank]].contiguous()
            vl = va[:, ko:ko + kv_len[rank]].contiguous()
            ro, rl = oracle.attention(qa.double().numpy(), ka.double().numpy(),
                                      va.double().numpy())
            eo = el = 0.0
            for pipeline in ("slots", "gather"):
                out, lse = cpd.ring_attention_allgather(ql, kl, vl, ops=ops, pipeline=pipeline)
                eo = max(eo, float(np.abs(out.numpy() - ro[:, qo:qo + q_len[rank]]).max()))
                el = max(el, float(np.abs(lse.numpy() - rl[:, :, qo:qo + q_len[rank]]).max()))
            q.put((rank, "ok", eo, el))
        elif case == "ring_order":
            # the per-slot pipeline's issue order, as this rank sees it
            trace = []
            real = dist.broadcast

            def logged(t, src, group=None, async_op=False):
                trace.append(("issue", src))
                return real(t, src, group=group, async_op=async_op)

            dist.broadcast = logged
            qa, ka, va = wl.make_qkv(1, 2, 4 * world, 8, torch.float32, 77)
            sl = slice(4 * rank, 4 * rank + 4)
            cpd.ring_attention_allgather(qa[:, sl], ka[:, sl].contiguous(),
                                         va[:, sl].contiguous(), ops=ops, trace=trace)
            dist.broadcast = real
            q.put((rank, "ok", trace, 0.0))
        elif case == "ulysses":
            B, S, H, D = 2, 10, 4, 8
            qa, ka, va = wl.make_qkv(B, H, S, D, torch.float32, 72)
            Sl = S // world
            sl = slice(rank * Sl, (rank + 1) * Sl)
            out, lse = cpd.ulysses_attention_all_to_all(qa[:, sl].contiguous(),
                                                        ka[:, sl].contiguous(),
                                                        va[:, sl].contiguous(), ops=ops,
                                                        want_lse=True)
            ro, rl = oracle.attention(qa.double().numpy(), ka.double().numpy(),
                                      va.double().numpy())
            Hg = H // world
            eo = float(np.abs(out.numpy() - ro[:, sl]).max())
            el = float(np.abs(lse.numpy() - rl[:, rank * Hg:(rank + 1) * Hg]).max())
            q.put((rank, "ok", eo, el))
        elif case == "ulysses_uneven":
            # Ulysses Anything over 3 ranks: 5, 4 and 3 tokens; 4 heads split
            # 2, 2, 0 (ceil rule), so the last rank attends no heads at all
            B, H, D, lens = 2, 4, 8, [5, 4, 3]
            qa, ka, va = wl.make_qkv(B, H, sum(lens), D, torch.float32, 75)
            o0 = sum(lens[:rank])
            sl = slice(o0, o0 + lens[rank])
            out, lse = cpd.ulysses_attention_all_to_all(qa[:, sl].contiguous(),
                                                        ka[:, sl].contiguous(),
                                                        va[:, sl].contiguous(), ops=ops,
                                                        want_lse=True)
            ro, rl = oracle.attention(qa.double().numpy(), ka.double().numpy(),
                                      va.double().numpy())
            h0, h1 = [0, 2, 4, 4][rank], [0, 2, 4, 4][rank + 1]
            eo = float(np.abs(out.numpy() - ro[:, sl]).max())
            el = float(np.abs(lse.numpy() - rl[:, h0:h1]).max()) if h1 > h0 else 0.0
            assert lse.shape == (B, h1 - h0, sum(lens))
            q.put((rank, "ok", eo, el))
        elif case == "usp_2d":
            # R = 2 ring ranks x U = 2 Ulysses ranks, rank g = r * U + u holds
            # sequence shard g; uneven shards everywhere (5, 4, 6, 3 tokens)
            R, U, B, H, D, lens = 2, 2, 2, 4, 8, [5, 4, 6, 3]
            uly = [dist.new_group([r * U + u for u in range(U)]) for r in range(R)]
            ring = [dist.new_group([r * U + u for r in range(R)]) for u in range(U)]
            r_me, u_me = divmod(rank, U)
            qa, ka, va = wl.make_qkv(B, H, sum(lens), D, torch.float32, 76)
            o0 = sum(lens[:rank])
            sl = slice(o0, o0 + lens[rank])
            out = cpd.usp_attention_2d(qa[:, sl].contiguous(), ka[:, sl].contiguous(),
                                       va[:, sl].contiguous(), ring[u_me], uly[r_me], ops=ops)
            ro, _ = oracle.attention(qa.double().numpy(), ka.double().numpy(),
                                     va.double().numpy())
            q.put((rank, "ok", float(np.abs(out.numpy() - ro[:, sl]).max()), 0.0))
        elif case == "rank_leaves":
            # rank 1 leaves between steps without joining the exchange: rank 0's
            # metadata all-gather must end with an error within the group's
            # timeout instead of waiting for good
            if rank == 1:
                q.put((rank, "left", 0.0, 0.0))
                q.close()
                q.join_thread()
                os._exit(0)
            import time
            qa, ka, va = wl.make_qkv(1, 2, 8, 16, torch.float32, 74)
            t0 = time.monotonic()
            try:
                cpd.ring_attention_allgather(qa, ka, va, ops=ops)
                q.put((rank, "no error", 0.0, 0.0))
            except RuntimeError:
                q.put((rank, "raised", time.monotonic() - t0, 0.0))
            q.close()
            q.join_thread()
            os._exit(0)
        elif case == "mismatch":
            # rank 1 holds a different number of heads: every rank must raise
            H = 3 if rank == 0 else 4
            qa, ka, va = wl.make_qkv(1, H, 8, 16, torch.float32, 73)
            try:
                cpd.ring_attention_allgather(qa, ka, va, ops=ops)
                q.put((rank, "no error", 0.0, 0.0))
            except cpd.ShardMismatch:
                q.put((rank, "raised", 0.0, 0.0))
        dist.destroy_process_group()
    except Exception:
        q.put((rank, "crash: " + traceback.format_exc(), 0.0, 0.0))
        raise


def _run(case, world=2, allow_exit=False):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
    res = sorted(q.get(timeout=5) for _ in range(world))
    assert all(p.exitcode == 0 for p in procs), res
    return res


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    res = _run("rank_leaves")
    assert res[1][1] == "left"
    assert res[0][1] == "raised", res
    assert res[0][2] < 60.0          # bounded by the group's 5 s timeout, not a hang


def test_ring_allgather_uneven_shards_equals_oneshot():
    for rank, status, eo, el in _run("ring"):
        assert status == "ok", status
        assert eo <= 1e-5 and el <= 1e-5, (rank, eo, el)


def test_ring_allgather_three_ranks_one_without_keys():
    for rank, status, eo, el in _run("ring3", world=3):
        assert status == "ok", status
        assert eo <= 1e-5 and el <= 1e-5, (rank, eo, el)


def test_ring_slot_pipeline_issue_order():
    """Every slot's broadcast is issued before any attention; then the local
    chunk is attended, and slot c's attention comes right after the wait for
    slot c, before the wait for the next slot."""
    world = 3
    for rank, status, trace, _ in _run("ring_order", world=world):
        assert status == "ok", status
        want = [("issue", c) for c in range(world)] + [("attend", rank)]
        for c in range(world):
            if c != rank:
                want += [("wait", c), ("attend", c)]
        assert [tuple(e) for e in trace] == want, (rank, trace)


def test_ulysses_all_to_all_equals_oneshot():
    for rank, status, eo, el in _run("ulysses"):
        assert status == "ok", status
        assert eo <= 1e-5 and el <= 1e-5, (rank, eo, el)


def test_ulysses_anything_uneven_shards_and_heads_over_three_ranks():
    for rank, status, eo, el in _run("ulysses_uneven", world=3):
        assert status == "ok", status
        assert eo <= 1e-5 and el <= 1e-5, (rank, eo, el)


def test_unified_2d_mesh_over_four_ranks():
    for rank, status, eo, _ in _run("usp_2d", world=4):
        assert status == "ok", status
        assert eo <= 1e-5, (rank, eo)


def test_shape_mismatch_raises_on_every_rank():
    res = _run("mismatch")
    assert [r[1] for r in res] == ["raised", "raised"], res
