"""Benchmark of the context-parallel attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}] [--extra]

One step = one fused ring-attention pass (cp_ring_attention) over the
FLUX-shaped joint attention workload: B=1, H=24, S=4608 (4096 image + 512
text tokens), D=128, bf16 q/k/v, ring_degree 4 (four K/V chunks of 1152),
fp32 output and LSE.  The headline value is 4*B*H*S^2*D / time in TFLOP/s.
In the same run the two bandwidth-bound kernels of the path are timed on
their own: the fp32 LSE merge (FLUX shape) and the Ulysses permutation in
both directions (B=2, S=8192, H=24, D=128, degree 4), reported in GB/s.

Timing: CUDA events on the launching stream around every step, the 126 MB
L2 flushed (a 256 MiB buffer is overwritten) between steps outside the
events; W untimed warm-up steps; K timed steps bracketed by a barrier and a
device synchronise; max over ranks.  N>1 runs one independent replica of
the workload per GPU (weak scaling, no collective on the data path).
``--impl reference`` times the CPU fp64 oracle on the host cores instead.

``--mode sharded`` (under torchrun) runs the method itself across the ranks
instead of replicas: the workload's sequence is split over the N ranks
(Ring Anything ceil split) and every step is one call of the multi-rank
module -- ``--method ring`` (K/V exchanged slot by slot while the chunk in
hand is attended), ``ulysses`` (all-to-all, attention per head group,
inverse all-to-all) or ``usp`` (2 x N/2 mesh).  The line then reports the
whole sequence's FLOPs over the slowest rank's step time ("scaling":
"strong") and the bytes each rank sends and receives per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("ring-attention TFLOP/s (4·B·H·S²·D) and % of B200 BF16 peak; "
          "merge/permute GB/s")
WORKLOAD = "flux_joint_ring4"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_ring_tc__flux_joint_ring4.txt")
TC_SOURCES = ("attn_tc.cu", "common.cuh")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _tc_source_sha():
    h = hashlib.sha256()
    for f in TC_SOURCES:
        h.update(open(os.path.join(ROOT, "context_attention_dits_cp_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def _profiled_traffic():
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, or None when there is none or the kernel changed since."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None
    vals = {}
    for line in open(PROFILE_SUMMARY):
        if ":" in line and not line.startswith((" ", "#", "|")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha") != _tc_source_sha():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
             0x100: "display_clock_setting"}

    def __init__(self, device_index: int, interval_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval_s = interval_s
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.NAMES.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.interval_s)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- helpers
def _dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        if world == 1 and n_gpus > 1:
            raise SystemExit("--gpus N>1 needs torchrun with N processes")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    else:
        torch.cuda.set_device(0)
    return rank, world, local, pg


def _barrier(pg, dev):
    """Device synchronise, then a barrier over all ranks, then synchronise."""
    if dev.type == "cuda":
        torch.cuda.synchronize(dev)
    if pg is not None:
        pg.barrier()
    if dev.type == "cuda":
        torch.cuda.synchronize(dev)


def _max_over_ranks(pg, x: float, dev) -> float:
    """The largest of every rank's `x` (the slowest rank sets the job time)."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own replica of the step, and
    the job's step time is the slowest rank's."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def _time_loop(fn, steps, warmup, flush, stream):
    """Per-step CUDA-event times (ms) of fn(), L2 flushed between steps."""
    for _ in range(warmup):
        flush()
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:
        flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


# ---------------------------------------------------------------- CUDA arm
def workload_config(w):
    """The benchmark line's `config`, shared by both arms."""
    from context_attention_dits_cp_b200 import workloads as wl
    lens = wl.ring_chunk_lengths(w.S, w.ring_degree)
    return {"workload": WORKLOAD, "B": w.B, "H": w.H, "S": w.S, "D": w.D,
            "ring_degree": w.ring_degree, "chunks": [int(c) for c in lens],
            "inputs": "N(0,1) q/k/v, key tokens scaled by U[0.5,2]",
            "out": "fp32 out + fp32 lse",
            "l2": "flushed between steps by writing a 256 MiB buffer",
            "per_gpu": "independent replica per GPU"}


def run_cuda(args):
    import context_attention_dits_cp_b200 as cp
    from context_attention_dits_cp_b200 import workloads as wl

    rank, world, local, pg = _dist_init(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    w = wl.workload(WORKLOAD)
    # each rank an independent replica (own seed): weak scaling
    q, k, v = wl.make_qkv(w.B, w.H, w.S, w.D, w.torch_dtype, w.seed + 1000 * rank, w.structure)
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
    dq, dk, dv = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty((w.B, w.S, w.H, w.D), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
    flush_buf = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.fill_(1)
    # The same flush followed by a read of the buffer: L2 is left cold and
    # clean, so a streaming kernel does not also pay for writing back the
    # flush buffer's dirty lines.  Reported beside the plain-flush figures of
    # the bandwidth-bound kernels.
    flush_clean = lambda: (flush_buf.fill_(1), flush_buf.sum(dtype=torch.int32))
    step = lambda: cp.ring_attention(dq, dk, dv, offs, out=out, lse=lse)
    flops = w.flops
    if args.profile_run in ("merge", "permute", "walk"):
        if args.profile_run == "walk":
            # the literal per-chunk ring step: chunk 0 alone, chunks 1.. merged in
            kcs = [(dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]]) for c in range(len(offs) - 1)]
            acc = torch.empty_like(out)
            lacc = torch.empty_like(lse)

            def fn():
                cp.attn_partial(dq, *kcs[0], out=acc, lse=lacc)
                for kc, vc in kcs[1:]:
                    cp.attn_partial_merge(dq, kc, vc, acc, lacc)
        elif args.profile_run == "merge":
            acc = torch.zeros_like(out)
            lacc = torch.full_like(lse, -float("inf"))
            oi = torch.randn(out.shape, device=dev)
            li = torch.randn(lse.shape, device=dev)
            fn = lambda: cp.lse_merge(acc, lacc, oi, li)
        else:
            u = wl.workload("ulysses4_unified2x2")
            x = torch.randn(4, u.B, u.S // 4, u.H, u.D, device=dev).to(torch.bfloat16)
            y = torch.empty(4, u.B, u.S, u.H // 4, u.D, device=dev, dtype=torch.bfloat16)
            fn = lambda: cp.ulysses_permute(x, 4, 0, y=y)
        t = _time_loop(fn, args.steps, args.warmup, flush, stream)
        print(json.dumps({"profile_run": args.profile_run, "ms": float(np.mean(t))}))
        return

    # ---- timed region: K steps of the whole hot path
    for _ in range(args.warmup):
        flush()
        step()
    # clocks: one sampler inside the timed region, one over everything
    # measured below as well (e2e and component loops), so that the median
    # rests on enough samples even when the timed region is a few ms
    sampler = ClockSampler(dev.index)
    run_sampler = ClockSampler(dev.index)
    run_sampler.__enter__()
    _barrier(pg, dev)
    with sampler:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            flush()
            a.record(stream)
            step()
            b.record(stream)
        _barrier(pg, dev)
    times = [a.elapsed_time(b) for a, b in evs]
    if args.profile_run:
        run_sampler.__exit__(None, None, None)
        if rank == 0:
            print(json.dumps({"profile_run": True, "ms_per_step": float(np.mean(times))}))
        if pg is not None:
            pg.destroy_process_group()
        return
    total_ms = _max_over_ranks(pg, float(sum(times)), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, flops, ms_per_step)
    kernel_ms = float(np.mean(times))          # one launch per step
    gpu_launches = args.steps                  # one cp_ring_attention kernel per step

    # ---- end to end through the C-ABI with host buffers: every step copies
    # its q/k/v from pinned host memory and reads its output and lse back.
    # Steps are pipelined over two device buffer sets and three streams, so
    # step i+1's upload, step i's attention and step i-1's download overlap
    # (PCIe moves both directions at once).
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    sets = [(dq, dk, dv, out, lse)] + [tuple(torch.empty_like(t) for t in (dq, dk, dv, out, lse))]
    s_up, s_comp, s_down = (torch.cuda.Stream(dev) for _ in range(3))

    def e2e_run(n):
        ev_in_free = [torch.cuda.Event() for _ in range(2)]    # attention done with set
        ev_out_free = [torch.cuda.Event() for _ in range(2)]   # download done with set
        for e in ev_in_free + ev_out_free:
            e.record(torch.cuda.current_stream(dev))
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_up)
        s_comp.wait_event(t0)
        s_down.wait_event(t0)
        for i in range(n):
            a, bq, bk, bv, bo, bl = i % 2, *sets[i % 2]
            s_up.wait_event(ev_in_free[a])
            with torch.cuda.stream(s_up):
                bq.copy_(hq, non_blocking=True)
                bk.copy_(hk, non_blocking=True)
                bv.copy_(hv, non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_up)
            s_comp.wait_event(up)
            s_comp.wait_event(ev_out_free[a])
            with torch.cuda.stream(s_comp):
                cp.ring_attention(bq, bk, bv, offs, out=bo, lse=bl)
            ev_in_free[a] = torch.cuda.Event()
            ev_in_free[a].record(s_comp)
            s_down.wait_event(ev_in_free[a])
            with torch.cuda.stream(s_down):
                hout.copy_(bo, non_blocking=True)
                hlse.copy_(bl, non_blocking=True)
            ev_out_free[a] = torch.cuda.Event()
            ev_out_free[a].record(s_down)
        s_down.wait_stream(s_up)
        s_down.wait_stream(s_comp)
        t1.record(s_down)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1) / n

    e2e_steps = max(3, min(args.steps, 30))
    e2e_run(3)                                    # warm-up
    _barrier(pg, dev)
    e2e_ms = _max_over_ranks(pg, e2e_run(e2e_steps), dev)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = out.numel() * 4 + lse.numel() * 4
    del sets

    peaks, peak_src = _peaks()
    tc_peak = float(peaks["bf16_tflops"])
    hbm_peak = float(peaks["hbm_gbs"])
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    traffic = _profiled_traffic()

    # ---- bandwidth-bound kernels, timed on their own
    components = {}
    n_merge = 30 if args.steps >= 30 else max(3, args.steps)
    acc = torch.zeros_like(out)
    lacc = torch.full_like(lse, -float("inf"))
    oi = torch.randn(out.shape, device=dev)
    li = torch.randn(lse.shape, device=dev)
    t_m = _time_loop(lambda: cp.lse_merge(acc, lacc, oi, li), n_merge, 3, flush, stream)
    t_mc = _time_loop(lambda: cp.lse_merge(acc, lacc, oi, li), n_merge, 3, flush_clean, stream)
    merge_bytes = out.numel() * 12 + lse.numel() * 12
    mg = merge_bytes / (np.mean(t_m) * 1e-3) / 1e9
    mgc = merge_bytes / (np.mean(t_mc) * 1e-3) / 1e9
    components["lse_merge"] = {"shape": [w.B, w.S, w.H, w.D], "bytes": merge_bytes,
                               "ms": float(np.mean(t_m)), "GB/s": mg,
                               "frac_of_hbm": mg / hbm_peak,
                               "GB/s_clean_l2": mgc, "frac_of_hbm_clean_l2": mgc / hbm_peak}
    u = wl.workload("ulysses4_unified2x2")
    x = torch.randn(4, u.B, u.S // 4, u.H, u.D, device=dev).to(torch.bfloat16)
    y = torch.empty(4, u.B, u.S, u.H // 4, u.D, device=dev, dtype=torch.bfloat16)
    x2 = torch.empty_like(x)
    pbytes = 2 * x.numel() * 2
    for name, fn in (("ulysses_permute_fwd", lambda: cp.ulysses_permute(x, 4, 0, y=y)),
                     ("ulysses_permute_inv", lambda: cp.ulysses_permute(y, 4, 1, y=x2))):
        t_p = _time_loop(fn, n_merge, 3, flush, stream)
        t_pc = _time_loop(fn, n_merge, 3, flush_clean, stream)
        gbs = pbytes / (np.mean(t_p) * 1e-3) / 1e9
        gbc = pbytes / (np.mean(t_pc) * 1e-3) / 1e9
        components[name] = {"shape": list(x.shape), "bytes": pbytes, "ms": float(np.mean(t_p)),
                            "GB/s": gbs, "frac_of_hbm": gbs / hbm_peak,
                            "GB/s_clean_l2": gbc, "frac_of_hbm_clean_l2": gbc / hbm_peak}
    del x, y, x2, oi, li, acc, lacc
    # the literal ring walk on the FLUX workload: one launch per arriving K/V
    # chunk, the first writing (out, lse), the others merging into them
    kcs = [(dk[:, offs[c]:offs[c + 1]], dv[:, offs[c]:offs[c + 1]])
           for c in range(w.ring_degree)]

    def literal_ring():
        cp.attn_partial(dq, *kcs[0], out=out, lse=lse)
        for kc, vc in kcs[1:]:
            cp.attn_partial_merge(dq, kc, vc, out, lse)

    t_r = _time_loop(literal_ring, n_merge, 3, flush, stream)
    tf = flops / (np.mean(t_r) * 1e-3) / 1e12
    components["ring_per_chunk_partial_merge"] = {
        "launches": w.ring_degree, "ms": float(np.mean(t_r)), "TFLOP/s": tf,
        "frac_of_bf16_peak": tf / tc_peak,
        "vs_single_launch": float(kernel_ms / np.mean(t_r))}
    # Ring Anything over ranks, as rank 0 sees it after the padded all-gather:
    # FLUX keys in 4 uneven shards (1172, 1172, 1172, 1092) padded to 1172;
    # own chunk first from local memory, then the other three slots
    g_len = [1172, 1172, 1172, 1092]
    g_pad = max(g_len)
    kg = torch.zeros((4, w.B, g_pad, w.H, w.D), dtype=dk.dtype, device=dev)
    vg = torch.zeros_like(kg)
    o = 0
    for c, n in enumerate(g_len):
        kg[c, :, :n] = dk[:, o:o + n]
        vg[c, :, :n] = dv[:, o:o + n]
        o += n

    def gathered_ring():
        cp.attn_partial(dq, kg[0, :, :g_len[0]], vg[0, :, :g_len[0]], out=out, lse=lse)
        cp.ring_attention_gathered(dq, kg, vg, g_len, skip_chunk=0, out=out, lse=lse,
                                   accumulate=True)

    t_g = _time_loop(gathered_ring, n_merge, 3, flush, stream)
    tf = flops / (np.mean(t_g) * 1e-3) / 1e12
    components["ring_gathered_uneven_own_chunk_first"] = {
        "lengths": g_len, "launches": 2, "ms": float(np.mean(t_g)), "TFLOP/s": tf,
        "frac_of_bf16_peak": tf / tc_peak}
    del kg, vg
    # unified R=2 x U=2 grid (B=2, S=8192, H=24, D=128) from sequence shards
    uq, uk, uv = wl.make_workload_inputs(u)
    ush = [wl.sequence_shards(t, 4).to(dev) for t in (uq, uk, uv)]
    del uq, uk, uv
    uout = torch.empty(ush[0].shape, dtype=torch.float32, device=dev)
    uws = torch.empty(max(1, cp.usp_workspace_bytes(u.B, u.S, u.H, u.D, torch.bfloat16,
                                                    torch.float32, 2, 2)),
                      dtype=torch.uint8, device=dev)
    t_u = _time_loop(lambda: cp.usp_attention(*ush, 2, 2, out=uout, workspace=uws,
                                              want_lse=False), n_merge, 3, flush, stream)
    tf = u.flops / (np.mean(t_u) * 1e-3) / 1e12
    components["usp_attention_R2_U2"] = {"shape": list(ush[0].shape), "flops": u.flops,
                                         "ms": float(np.mean(t_u)), "TFLOP/s": tf,
                                         "frac_of_bf16_peak": tf / tc_peak}
    del ush, uout, uws
    # Ulysses Anything on FLUX at 1008x1008: 3969 + 512 = 4481 tokens, U = 4
    # (1121, 1121, 1121, 1118 tokens per rank; 6 heads each)
    A_S, A_U = 4481, 4
    aq, ak, av = wl.make_qkv(1, 24, A_S, 128, torch.bfloat16, 1101, "kscale")
    so = cp.ring_chunk_offsets(A_S, A_U)
    ho = cp.ring_chunk_offsets(24, A_U)
    flat = lambda t: torch.cat([t[:, so[p]:so[p + 1]].reshape(-1) for p in range(A_U)]).to(dev)
    aq, ak, av = flat(aq), flat(ak), flat(av)
    aout = torch.empty(aq.shape, dtype=torch.float32, device=dev)
    aws = torch.empty(cp.binding.lib().cp_ulysses_anything_workspace_bytes(
        1, A_S, 24, 128, cp.binding.CP_BF16, cp.binding.CP_F32), dtype=torch.uint8, device=dev)
    t_a = _time_loop(lambda: cp.ulysses_anything_attention(aq, ak, av, 1, 24, 128, so, ho,
                                                           out=aout, workspace=aws,
                                                           want_lse=False),
                     n_merge, 3, flush, stream)
    aflops = 4.0 * 24 * A_S * A_S * 128
    tf = aflops / (np.mean(t_a) * 1e-3) / 1e12
    components["ulysses_anything_1008px_U4"] = {"S": A_S, "flops": aflops,
                                                "ms": float(np.mean(t_a)), "TFLOP/s": tf,
                                                "frac_of_bf16_peak": tf / tc_peak}
    del aq, ak, av, aout, aws
    if args.extra:
        components.update(_extra_workloads(cp, wl, dev, stream, flush, tc_peak))

    run_sampler.__exit__(None, None, None)
    clocks = sampler.summary()
    whole = run_sampler.summary()
    clocks["timed_region_samples"] = clocks.pop("samples", 0)
    clocks["timed_region_sm_mhz"] = clocks["sm_mhz"]
    if whole.get("sm_mhz") is not None:
        # the median over the whole measured run (timed region, e2e and
        # component loops), the figure the cycle count below uses
        clocks["sm_mhz"] = whole["sm_mhz"]
        clocks["samples"] = whole.get("samples", 0)
        clocks["reasons"] = sorted((set(clocks["reasons"]) - {"unavailable"}) |
                                   set(whole["reasons"]))
        clocks["sm_kcycles_per_step"] = ms_per_step * whole["sm_mhz"]
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _cpu_baseline(q, k, v, w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w),
            "pct_of_bf16_peak": 100.0 * value / (world * tc_peak),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": achieved / tc_peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "kernel": "attn_ring_tc_kernel<128,4>",
                         "algorithmic": "4*D flops per (query, key, head): 2.609e11 per launch"},
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms,
                    "how": "pinned host q/k/v -> device, cp_ring_attention, out+lse -> "
                           "pinned host, every step; steps pipelined on 3 streams"},
            "gpu_launches": gpu_launches,
            "clocks": clocks,
            "components": components,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def _extra_workloads(cp, wl, dev, stream, flush, tc_peak):
    res = {}
    for name in ("hires_dit_ring8", "video_ring_anything8"):
        w = wl.workload(name)
        q, k, v = (t.to(dev) for t in wl.make_workload_inputs(w))
        offs = wl.chunk_offsets(wl.ring_chunk_lengths(w.S, w.ring_degree))
        out = torch.empty((w.B, w.S, w.H, w.D), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, w.H, w.S), dtype=torch.float32, device=dev)
        t = _time_loop(lambda: cp.ring_attention(q, k, v, offs, out=out, lse=lse), 5, 2,
                       flush, stream)
        tf = w.flops / (np.mean(t) * 1e-3) / 1e12
        res[name] = {"ms": float(np.mean(t)), "TFLOP/s": tf, "frac_of_bf16_peak": tf / tc_peak}
        del q, k, v, out, lse
    # head dim 64: the FLUX token count with twice the heads (same flops)
    q, k, v = (t.to(dev) for t in wl.make_qkv(1, 48, 4608, 64, torch.bfloat16, 1201, "kscale"))
    offs = wl.chunk_offsets(wl.ring_chunk_lengths(4608, 4))
    out = torch.empty((1, 4608, 48, 64), dtype=torch.float32, device=dev)
    lse = torch.empty((1, 48, 4608), dtype=torch.float32, device=dev)
    t = _time_loop(lambda: cp.ring_attention(q, k, v, offs, out=out, lse=lse), 20, 3, flush, stream)
    f64 = 4.0 * 48 * 4608 * 4608 * 64
    tf = f64 / (np.mean(t) * 1e-3) / 1e12
    res["ring_d64_h48_s4608_r4"] = {"ms": float(np.mean(t)), "TFLOP/s": tf,
                                    "frac_of_bf16_peak": tf / tc_peak}
    del q, k, v, out, lse
    u = wl.workload("ulysses4_unified2x2")
    q, k, v = wl.make_workload_inputs(u)
    for R, U in ((1, 4), (2, 2)):
        sh = [wl.sequence_shards(t, R * U).to(dev) for t in (q, k, v)]
        out = torch.empty(sh[0].shape, dtype=torch.float32, device=dev)
        ws = torch.empty(cp.usp_workspace_bytes(u.B, u.S, u.H, u.D, torch.bfloat16,
                                                torch.float32, R, U), dtype=torch.uint8,
                         device=dev)
        t = _time_loop(lambda: cp.usp_attention(*sh, R, U, out=out, workspace=ws,
                                                want_lse=False), 5, 2, flush, stream)
        tf = u.flops / (np.mean(t) * 1e-3) / 1e12
        res[f"usp_R{R}_U{U}"] = {"ms": float(np.mean(t)), "TFLOP/s": tf,
                                 "frac_of_bf16_peak": tf / tc_peak}
    return res


# ---------------------------------------------------------------- sharded mode
def sharded_plan(w, world: int, rank: int, method: str) -> dict:
    """This rank's share of a sharded step: its token range and the bytes it
    sends and receives per step over the exchange (counted from the tensors
    the multi-rank module moves)."""
    from context_attention_dits_cp_b200 import workloads as wl
    lens = wl.ring_chunk_lengths(w.S, world)
    off = wl.chunk_offsets(lens)
    elt = 4 if w.dtype == "f32" else 2
    s_me = lens[rank]
    plan = {"tokens": (off[rank], off[rank + 1]), "shard_lengths": lens}
    if method == "ring":
        L = max(lens)
        slot = 2 * w.B * L * w.H * w.D * elt            # padded [K; V] of one rank
        plan.update(send=slot, recv=(world - 1) * slot)
    elif method == "ulysses":
        hoff = wl.chunk_offsets(wl.ring_chunk_lengths(w.H, world))
        h_me = hoff[rank + 1] - hoff[rank]
        tok = w.B * w.D
        # q, k, v scatter: own tokens of the other groups' heads go out, the
        # other ranks' tokens of this group's heads come in; the fp32 output
        # takes the reverse path
        plan.update(send=3 * tok * s_me * (w.H - h_me) * elt + tok * (w.S - s_me) * h_me * 4,
                    recv=3 * tok * (w.S - s_me) * h_me * elt + tok * s_me * (w.H - h_me) * 4)
    elif method == "usp":
        R, U = 2, world // 2
        r_me, u_me = divmod(rank, U)
        grp = [lens[r_me * U + u] for u in range(U)]       # this Ulysses group's shards
        hoff = wl.chunk_offsets(wl.ring_chunk_lengths(w.H, U))
        h_me = hoff[u_me + 1] - hoff[u_me]
        tok = w.B * w.D
        S_u = sum(grp)
        blocks = [sum(lens[r * U:(r + 1) * U]) for r in range(R)]
        slot = 2 * w.B * max(blocks) * h_me * w.D * elt
        plan.update(send=3 * tok * s_me * (w.H - h_me) * elt + tok * (S_u - s_me) * h_me * 4
                    + slot,
                    recv=3 * tok * (S_u - s_me) * h_me * elt + tok * s_me * (w.H - h_me) * 4
                    + (R - 1) * slot)
    else:
        raise ValueError(method)
    return plan


def run_sharded(args, ops=None, device=None):
    """One rank of ``--mode sharded``: every step is one call of the
    multi-rank module on this rank's shard of the whole sequence."""
    import torch.distributed as dist
    from context_attention_dits_cp_b200 import dist as cpd
    from context_attention_dits_cp_b200 import workloads as wl

    if device is None:
        rank, world, local, pg = _dist_init(args.gpus)
        dev = torch.device("cuda", local if world > 1 else 0)
        if pg is None:                        # one rank: a group of one
            import datetime
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29517")
            dist.init_process_group("nccl", rank=0, world_size=1,
                                    timeout=datetime.timedelta(seconds=120), device_id=dev)
            pg = dist
    else:                                     # host-logic tests: gloo ranks on the CPU
        dev, pg = device, dist
        rank, world = dist.get_rank(), dist.get_world_size()
    cpu_group = dist.new_group(backend="gloo") if dev.type == "cuda" else None
    w = wl.workload(args.workload)
    method = args.method
    if method == "usp" and world % 2:
        raise SystemExit("--method usp needs an even number of ranks (2 x N/2 mesh)")
    plan = sharded_plan(w, world, rank, method)
    q, k, v = wl.make_workload_inputs(w)
    t0, t1 = plan["tokens"]
    q, k, v = (t[:, t0:t1].contiguous().to(dev) for t in (q, k, v))
    groups = None
    if method == "usp":
        R, U = 2, world // 2
        uly = [dist.new_group([r * U + u for u in range(U)]) for r in range(R)]
        ring = [dist.new_group([r * U + u for r in range(R)]) for u in range(U)]
        r_me, u_me = divmod(rank, U)
        groups = (ring[u_me], uly[r_me])
        if dev.type == "cuda":
            ulyc = [dist.new_group([r * U + u for u in range(U)], backend="gloo")
                    for r in range(R)]
            ringc = [dist.new_group([r * U + u for r in range(R)], backend="gloo")
                     for u in range(U)]
            groups += (ringc[u_me], ulyc[r_me])
        else:
            groups += (None, None)

    def step():
        if method == "ring":
            return cpd.ring_attention_allgather(q, k, v, cpu_group=cpu_group, ops=ops)
        if method == "ulysses":
            return cpd.ulysses_attention_all_to_all(q, k, v, cpu_group=cpu_group, ops=ops)
        return cpd.usp_attention_2d(q, k, v, groups[0], groups[1], ring_cpu_group=groups[2],
                                    ulysses_cpu_group=groups[3], ops=ops)

    for _ in range(args.warmup):
        step()
    _barrier(pg, dev)
    if dev.type == "cuda":
        stream = torch.cuda.current_stream(dev)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        _barrier(pg, dev)
        local_ms = a.elapsed_time(b)
    else:
        tt = time.perf_counter()
        for _ in range(args.steps):
            step()
        _barrier(pg, dev)
        local_ms = 1e3 * (time.perf_counter() - tt)
    total_ms = _max_over_ranks(pg, float(local_ms), dev)
    ms_per_step = total_ms / args.steps
    value = w.flops / (ms_per_step * 1e-3) / 1e12        # whole sequence, all ranks
    mine = torch.tensor([float(plan["send"]), float(plan["recv"])], dtype=torch.float64)
    table = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(table, mine, group=cpu_group)      # host integers over gloo
    line = None
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "mode": "sharded",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "S": w.S, "D": w.D,
                       "method": method, "shard_lengths": plan["shard_lengths"],
                       "parallelism": {"ring": f"ring{world}", "ulysses": f"ulysses{world}",
                                       "usp": f"ring2 x ulysses{world // 2}"}[method]},
            "exchange_bytes_per_rank": [{"send": int(t[0]), "recv": int(t[1])} for t in table],
        }
        print(json.dumps(line), flush=True)
    if dev.type == "cuda":
        dist.destroy_process_group()
    return line


# ---------------------------------------------------------------- CPU oracle
def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _cpu_baseline(q, k, v, w, heads=None):
    """The oracle, as it stands, on the host cores (whole workload unless
    `heads` limits it to the first few heads)."""
    import oracle
    f = lambda t: t.float().numpy().astype(np.float64)
    hs = w.H if heads is None else heads
    qn, kn, vn = f(q[:, :, :hs]), f(k[:, :, :hs]), f(v[:, :, :hs])
    # whole passes over the workload until about 10 s of CPU work (at least one)
    runs = 0
    t0 = time.perf_counter()
    while True:
        oracle.attention(qn, kn, vn)
        runs += 1
        dt = time.perf_counter() - t0
        if dt >= 10.0 or runs >= 50:
            break
    flops = 4.0 * w.B * hs * w.S * w.S * w.D * runs
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": _cpu_threads(),
            "kind": "oracle", "seconds": dt, "runs": runs,
            "sample": f"{WORKLOAD}: all {w.S} query rows of {hs} of {w.H} heads, fp64 one-shot, "
                      f"{runs} passes"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    from context_attention_dits_cp_b200 import workloads as wl
    w = wl.workload(WORKLOAD)
    q, k, v = wl.make_workload_inputs(w)
    f = lambda t: t.float().numpy().astype(np.float64)
    qn, kn, vn = f(q), f(k), f(v)
    # size one step so that warm-up + timed steps stay within ~2 minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = 64
    t0 = time.perf_counter()
    oracle.attention(qn[:, :rows], kn, vn)
    per_row = (time.perf_counter() - t0) / rows
    rows = int(max(16, min(w.S, budget / max(per_row, 1e-9))))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        oracle.attention(qn, kn, vn, rows=rng.choice(w.S, rows, replace=False))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention(qn, kn, vn, rows=rng.choice(w.S, rows, replace=False))
    dt = time.perf_counter() - t0
    flops = 4.0 * w.B * w.H * rows * w.S * w.D
    value = args.steps * flops / dt / 1e12
    cores = _cpu_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} random query rows x all {w.H} heads per step "
                                   f"against all {w.S} keys, fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("cuda", "reference"), default="cuda")
    ap.add_argument("--mode", choices=("replicas", "sharded"), default="replicas",
                    help="replicas: one independent copy of the workload per GPU (default); "
                         "sharded: the sequence split over the ranks, exchanged per step")
    ap.add_argument("--method", choices=("ring", "ulysses", "usp"), default="ring",
                    help="sharded mode: which exchange")
    ap.add_argument("--workload", default=WORKLOAD, help="sharded mode: workload name")
    ap.add_argument("--extra", action="store_true", help="also time the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-run", nargs="?", const="ring", default=None,
                    choices=("ring", "merge", "permute", "walk"),
                    help="only warm-up + timed launches of one kernel (for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "sharded":
        run_sharded(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
