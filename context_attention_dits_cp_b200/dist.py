"""Context-parallel attention across ranks (one process per GPU).

The single-GPU calls of this package walk the ring and permute the Ulysses
layout inside one device.  This module runs the same computation with the
sequence really sharded over the ranks of a process group, following the
diffusers context-parallelism guide (§Ring Attention with an all-gather of
K/V, §Ring Anything for uneven shards, §Ulysses Attention):

* ``ring_attention_allgather`` -- every rank holds its own sequence shard of
  q, k, v, of any length (Ring Anything).  The shard lengths travel over a
  CPU group first, so no device synchronisation is needed for metadata.  Each
  rank pads K/V to the longest shard and the padded shards are exchanged,
  by default as one asynchronous broadcast per slot: the local chunk is
  attended while they travel, then each slot's chunk as soon as that slot
  has landed, while later slots are still in flight.  The padding is
  trimmed by the chunk extents: no call ever attends it.
* ``ulysses_attention_all_to_all`` -- every rank holds its tokens of all H
  heads.  The heads are packed into U groups, exchanged with one all-to-all
  so that every rank holds all tokens of its head group, attended, and sent
  back with the inverse all-to-all.  Equal shards with H % U == 0 are the
  guide's Ulysses (attended in the shard layout in place); anything else is
  Ulysses Anything (§Ulysses Anything): uneven shards, heads split as
  ceil(H/U) per rank, exchanged with uneven all-to-all splits.

The kernels are reached through ``ops`` (by default the C-ABI binding of this
package), so the host-side logic can be exercised on CPU ranks.  Every rank
issues the same collectives in the same order, also on the error paths:
a shape mismatch is detected from the exchanged metadata, which every rank
sees in full, and all ranks raise together.
"""
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import binding

_DTYPE_CODES = {torch.float32: 0, torch.bfloat16: 1}


class ShardMismatch(ValueError):
    """The ranks' shards disagree on batch, heads, head dim or dtype."""


def exchange_shard_meta(q: torch.Tensor, k: torch.Tensor, group=None) -> List[List[int]]:
    """All ranks' (kv_len, q_len, B, H, D, dtype) rows, gathered over ``group``
    (a CPU group: the rows are host integers).  Raises ShardMismatch on every
    rank when B, H, D or the dtype differ, or when q and k of one rank do."""
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, S, H, D]")
    code = _DTYPE_CODES.get(q.dtype, -1)
    bad = int(tuple(k.shape[0:1]) + tuple(k.shape[2:]) != tuple(q.shape[0:1]) + tuple(q.shape[2:])
              or k.dtype != q.dtype)
    meta = torch.tensor([k.shape[1], q.shape[1], q.shape[0], q.shape[2], q.shape[3], code, bad],
                        dtype=torch.int64)
    world = dist.get_world_size(group)
    # a CPU group keeps this off the device; over NCCL it costs one sync
    dev = (torch.device("cuda", torch.cuda.current_device())
           if dist.get_backend(group) == "nccl" else torch.device("cpu"))
    meta = meta.to(dev)
    rows = torch.empty(world * meta.numel(), dtype=torch.int64, device=dev)
    dist.all_gather_into_tensor(rows, meta, group=group)
    table = rows.view(world, -1).cpu().tolist()
    if any(r[6] for r in table):
        raise ShardMismatch(f"q and k disagree on some rank: {table}")
    if any(r[2:6] != table[0][2:6] for r in table):
        raise ShardMismatch(f"ranks disagree on (B, H, D, dtype): {[r[2:6] for r in table]}")
    return [r[:6] for r in table]


def ring_attention_allgather(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group=None,
                             cpu_group=None, scale: Optional[float] = None, ops=None,
                             pipeline: str = "slots", trace: Optional[list] = None):
    """Attention of this rank's queries to the whole sharded sequence.

    q, k, v: this rank's shard [B, s_r, H, D]; s_r may differ across ranks.
    group:   the device group (NCCL) that carries K/V; cpu_group: the group
             that carries the shard lengths (gloo; defaults to ``group``).
    pipeline:
      ``"slots"``  (default) the padded all-gather is split into one
                   broadcast per slot (slot c = rank c's padded [K; V]),
                   all issued at once and asynchronous.  The local chunk is
                   attended while they travel; then slot after slot, each
                   chunk's attention is issued as soon as its own transfer
                   has completed, folded into the accumulator by
                   cp_attn_partial_merge, while the later slots are still in
                   flight (the guide's ring: K/V move while the block in hand
                   is attended).
      ``"gather"`` one all-gather of every slot, overlapped with the local
                   chunk only, then one cp_ring_attention_gathered launch
                   over all other slots.
    trace:   optional list; the "slots" pipeline appends ("wait", c) when it
             makes the compute stream wait for slot c and ("attend", c) when
             it issues slot c's attention (own chunk included).
    Returns (out [B, s_q, H, D] fp32, lse [B, H, s_q] fp32) for the local
    queries against all ranks' keys.
    """
    ops = binding if ops is None else ops
    if pipeline not in ("slots", "gather"):
        raise ValueError(f"unknown pipeline {pipeline!r}")
    rank = dist.get_rank(group)
    meta = exchange_shard_meta(q, k, cpu_group if cpu_group is not None else group)
    lengths = [m[0] for m in meta]
    R = len(lengths)
    L = max(lengths)
    B, s, H, D = k.shape
    # Ring Anything: pad K/V to the longest shard.  The padding rows are left
    # as they are: no call below ever attends them, whatever they hold.
    recv = torch.empty((R, 2, B, L, H, D), dtype=k.dtype, device=k.device)
    if pipeline == "gather":
        send = torch.empty((2, B, L, H, D), dtype=k.dtype, device=k.device)
        send[0, :, :s].copy_(k)
        send[1, :, :s].copy_(v)
        work = dist.all_gather_into_tensor(recv.view(-1), send.view(-1), group=group,
                                           async_op=True)
        # the local chunk needs no exchange: fold it in while K/V travel
        out, lse = ops.attn_partial(q, k, v, scale=scale)
        work.wait()
        ops.ring_attention_gathered(q, recv[:, 0], recv[:, 1], lengths, skip_chunk=rank,
                                    scale=scale, out=out, lse=lse, accumulate=True)
        return out, lse
    # "slots": every rank issues the same broadcasts in the same (rank)
    # order; rank c's slot is its own send buffer
    recv[rank, 0, :, :s].copy_(k)
    recv[rank, 1, :, :s].copy_(v)
    works = [dist.broadcast(recv[c], src=dist.get_global_rank(group, c) if group is not None
                            else c, group=group, async_op=True) for c in range(R)]
    if trace is not None:
        trace.append(("attend", rank))
    out, lse = ops.attn_partial(q, k, v, scale=scale)
    for c in range(R):
        if c == rank:
            continue
        if trace is not None:
            trace.append(("wait", c))
        works[c].wait()          # the compute stream waits for slot c only
        if lengths[c] == 0:
            continue
        if trace is not None:
            trace.append(("attend", c))
        n = lengths[c]
        ops.attn_partial_merge(q, recv[c, 0, :, :n], recv[c, 1, :, :n], out, lse, scale=scale)
    works[rank].wait()           # our own broadcast, before recv can be freed
    return out, lse


def _rank_offsets(sizes: Sequence[int]) -> List[int]:
    off = [0]
    for n in sizes:
        off.append(off[-1] + n)
    return off


class _HeadExchange:
    """One rank's side of the Ulysses all-to-all and its inverse.

    scatter(): this rank's tokens of all H heads -> the whole group
    sequence of this rank's head group, held as U rank buffers
    [B, s_p, h_me, D] in rank order (flat).  gather(): the inverse, for an
    fp32 result in that layout.  Heads split ceil(H/U) per rank; shards may
    differ in length (Ulysses Anything)."""

    def __init__(self, ops, group, meta, B, H, D):
        self.ops, self.group = ops, group
        U, me = dist.get_world_size(group), dist.get_rank(group)
        self.U, self.B, self.H, self.D = U, B, H, D
        self.lens = [m[0] for m in meta]
        self.seq_off = _rank_offsets(self.lens)
        self.head_off = binding.ring_chunk_offsets(H, U)
        heads = [self.head_off[g + 1] - self.head_off[g] for g in range(U)]
        self.h_me = heads[me]
        s = self.lens[me]
        self.s = s
        # pack: the sequence side is one buffer holding all s local tokens,
        # the head side is U buffers of heads[g] heads
        self.one = [0] + [s] * U
        self.send_n = [B * s * heads[g] * D for g in range(U)]
        self.recv_n = [B * self.lens[p] * self.h_me * D for p in range(U)]

    def scatter(self, t):
        packed = torch.empty(self.B * self.s * self.H * self.D, dtype=t.dtype, device=t.device)
        self.ops.ulysses_anything_permute(t.reshape(-1), self.B, self.H, self.D, self.one,
                                          self.head_off, binding.SEQ_TO_HEAD, y=packed)
        r = torch.empty(sum(self.recv_n), dtype=t.dtype, device=t.device)
        dist.all_to_all_single(r, packed, output_split_sizes=self.recv_n,
                               input_split_sizes=self.send_n, group=self.group)
        return r

    def gather(self, o_flat):
        back = torch.empty(self.B * self.s * self.H * self.D, dtype=torch.float32,
                           device=o_flat.device)
        dist.all_to_all_single(back, o_flat, output_split_sizes=self.send_n,
                               input_split_sizes=self.recv_n, group=self.group)
        out = torch.empty((self.B, self.s, self.H, self.D), dtype=torch.float32,
                          device=o_flat.device)
        self.ops.ulysses_anything_permute(back, self.B, self.H, self.D, self.one, self.head_off,
                                          binding.HEAD_TO_SEQ, y=out.view(-1))
        return out


def ulysses_attention_all_to_all(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group=None,
                                 cpu_group=None, scale: Optional[float] = None, ops=None,
                                 want_lse: bool = False):
    """Ulysses attention over the ranks of ``group``.

    q, k, v: this rank's tokens of all H heads, [B, s_r, H, D].  With equal
    shards and H % U == 0 this is the guide's Ulysses; otherwise Ulysses
    Anything: the shards may differ in length and the heads split as
    ceil(H/U) per rank, the last ranks holding fewer (possibly none).
    Returns this rank's output tokens [B, s_r, H, D] in fp32 (and, with
    want_lse, the LSE of this rank's head group over the whole sequence,
    [B, h_r, S]).
    """
    ops = binding if ops is None else ops
    U = dist.get_world_size(group)
    meta = exchange_shard_meta(q, k, cpu_group if cpu_group is not None else group)
    if any(m[0] != m[1] for m in meta):
        raise ShardMismatch(f"Ulysses needs q and k/v of one length on every rank: {meta}")
    B, s, H, D = q.shape
    x = _HeadExchange(ops, group, meta, B, H, D)
    recvs = [x.scatter(t) for t in (q, k, v)]
    Hm = x.h_me
    if all(n == x.lens[0] for n in x.lens) and H % U == 0:
        # equal shards: the shard layout [U, B, s, Hm, D], attended in place
        shards = [r.view(U, B, s, Hm, D) for r in recvs]
        out_sh = torch.empty((U, B, s, Hm, D), dtype=torch.float32, device=q.device)
        lse = (torch.empty((B, Hm, U * s), dtype=torch.float32, device=q.device)
               if want_lse else None)
        ops.usp_attention(*shards, U, 1, scale=scale, out=out_sh, lse=lse, want_lse=want_lse)
        o_flat = out_sh.view(-1)
    else:
        o_flat = torch.empty(sum(x.recv_n), dtype=torch.float32, device=q.device)
        lse = (torch.empty((B, Hm, x.seq_off[-1]), dtype=torch.float32, device=q.device)
               if want_lse else None)
        ops.ulysses_anything_attention(*recvs, B, Hm, D, x.seq_off, [0] + [Hm] * U, scale=scale,
                                       out=o_flat, lse=lse, want_lse=want_lse)
    out = x.gather(o_flat)
    return (out, lse) if want_lse else out


def usp_attention_2d(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, ring_group,
                     ulysses_group, ring_cpu_group=None, ulysses_cpu_group=None,
                     scale: Optional[float] = None, ops=None):
    """The unified composition on a 2-D mesh of R x U ranks (ring outer,
    Ulysses inner: rank g = r * U + u holds sequence shard g).

    1. Ulysses all-to-all inside the Ulysses group: this rank then holds the
       whole group sequence block for its head group;
    2. the ring over the ring group: padded all-gather of those blocks,
       local block first, the rest merged in (ring_attention_allgather);
    3. the inverse all-to-all.
    q, k, v: this rank's shard [B, s_g, H, D].  Returns this rank's output
    tokens [B, s_g, H, D] in fp32.
    """
    ops = binding if ops is None else ops
    U = dist.get_world_size(ulysses_group)
    meta = exchange_shard_meta(q, k, ulysses_cpu_group if ulysses_cpu_group is not None
                               else ulysses_group)
    if any(m[0] != m[1] for m in meta):
        raise ShardMismatch(f"the unified layout needs q and k/v of one length: {meta}")
    B, s, H, D = q.shape
    x = _HeadExchange(ops, ulysses_group, meta, B, H, D)
    Hm = x.h_me
    # the Ulysses group's block as one [B, S_u, Hm, D] sequence: the rank
    # buffers are concatenated along the sequence (free when B == 1)
    S_u = x.seq_off[-1]
    blk_heads = [0] + [Hm] * U

    def as_block(r):
        if B == 1:
            return r.view(1, S_u, Hm, D)
        b = torch.empty(B * S_u * Hm * D, dtype=r.dtype, device=r.device)
        ops.ulysses_anything_permute(r, B, Hm, D, x.seq_off, blk_heads, binding.SEQ_TO_HEAD, y=b)
        return b.view(B, S_u, Hm, D)

    qb, kb, vb = (as_block(x.scatter(t)) for t in (q, k, v))
    out_b, _ = ring_attention_allgather(qb, kb, vb, group=ring_group, cpu_group=ring_cpu_group,
                                        scale=scale, ops=ops)
    if B == 1:
        o_flat = out_b.reshape(-1)
    else:
        o_flat = torch.empty(B * S_u * Hm * D, dtype=torch.float32, device=q.device)
        ops.ulysses_anything_permute(out_b.reshape(-1), B, Hm, D, x.seq_off, blk_heads,
                                     binding.HEAD_TO_SEQ, y=o_flat)
    return x.gather(o_flat)
