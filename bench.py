"""Benchmark of the PSA forward pass (pyramid -> mask -> attention) on B200.

One step = one whole forward pass over one batch of the workload (default: the
Wan2.1-1.3B-shaped video DiT self-attention, B=1, H=12, N=32760, d=128, bf16,
128/64 blocks, thresholds frozen for 91% skipped dense FLOPs).  Inputs are the
seeded synthetic smooth-field-plus-noise tensors of ``workloads``.

Prints ONE JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
batch (independent problems, no data-path collective: weak scaling); the
timing is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "PSA fwd ms/call & dense-equiv TFLOP/s at Wan-1.3B shape; % bf16 tensor peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wan2.1_1.3b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-heads", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward-pass measurement")
    ap.add_argument("--sim-threshold", type=float, default=-1.0,
                    help="cosine-similarity constraint on the pyramid levels (-1: off, the "
                         "method's default)")
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling aid: run only this many query heads (KV heads scaled to match)")
    ap.add_argument("--profile-kernels", action="store_true",
                    help="after the timed region, run the steps again under the torch profiler "
                         "(CUPTI) and add per-kernel microseconds to the line")
    ap.add_argument("--min-timed-seconds", type=float, default=0.5,
                    help="repeat the timed loop of --steps steps until the timed region lasts "
                         "at least this long, so that the clock sampler sees it")
    ap.add_argument("--cpu-baseline-all", action="store_true",
                    help="time the oracle on every workload (one head, extrapolated to the "
                         "whole workload) and the tiny workload on one thread; one JSON line each")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="batch: every rank runs its own batch (weak scaling, the default); "
                         "heads: the ranks split the heads of one problem (strong scaling)")
    return ap.parse_args()


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one
# attention launch, from an ncu capture of that launch, keyed by the workload,
# its query heads and a hash of the attention kernel's sources.  A kernel that
# has changed since the counters were taken has no entry, and the roofline's
# traffic is then null.
ATTN_SOURCES = ("attn_tc.cu", "sm100_ptx.cuh", "psa_internal.cuh", "tile_walk.cuh")
ATTN_TRAFFIC = {("wan2.1_1.3b", 12, "2cd6a4b28733912d"): 476.693248e6 + 91.385600e6}
# the same for one launch of the attention-gradient kernel
BWD_SOURCES = ("attn_bwd_tc.cu", "sm100_ptx.cuh", "psa_internal.cuh", "tile_walk.cuh",
               "bwd_internal.cuh")
BWD_TRAFFIC = {("wan2.1_1.3b", 12, "de7109ecc7e51404"): 1945.523200e6 + 1369.462528e6}


def attn_source_hash(sources=ATTN_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "level_sparse_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["bf16_tflops"], d["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


# --------------------------------------------------------- multi-rank plumbing
#
# Every (batch, head) problem of the forward pass is independent, so N ranks
# each run their own batch of the workload's shape with no data-path
# collective (weak scaling).  The only collectives are measurement: a barrier
# around the timed region and a max over ranks of the timed milliseconds.

def rank_batch0(rank: int, B: int) -> int:
    """Global index of the first batch element that `rank` runs: rank r runs
    elements [r*B, (r+1)*B) of a global batch of world*B."""
    return rank * B


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of `x` over all ranks (x itself when world == 1)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Throughput of the whole job: the work all ranks did over the slowest
    rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


def mask_bytes(w: W.Workload) -> float:
    """Algorithmic HBM bytes of the mask stage: Q read once, the fp32 level-3
    keys read once per KV head, the int8 level map written once."""
    es = 2 if w.dtype == "bf16" else 4
    return float(w.B * w.Hq * w.N * w.d * es + w.B * w.Hkv * (-(-w.N // 8)) * w.d * 4
                 + w.B * w.Hq * w.Nq * w.Nk)


def pyramid_bytes(w: W.Workload) -> float:
    """Algorithmic HBM bytes of the pyramid stage: K and V read once, levels
    1..3 of both written once (1/2 + 1/4 + 1/8 of the input), the fp32
    level-3 keys written once."""
    es = 2 if w.dtype == "bf16" else 4
    return float(2 * w.B * w.Hkv * w.N * w.d * es * (1 + 0.875)
                 + w.B * w.Hkv * (-(-w.N // 8)) * w.d * 4)


# ------------------------------------------------------------- CPU oracle leg

def cpu_sample(w: W.Workload, n_heads: int, sim_threshold: float = -1.0):
    """Time the oracle (as it stands) on `n_heads` whole heads of the workload.
    Returns (dense-equivalent TFLOP/s, seconds, cores, sample description,
    the oracle's per-head results)."""
    import oracle as O
    cores = len(os.sched_getaffinity(0))
    grp = w.Hq // w.Hkv
    heads = list(range(n_heads))
    inp = W.make_inputs(w, heads_q=heads, heads_kv=sorted({h // grp for h in heads}))
    tau = W.thresholds(w)
    t0 = time.perf_counter()
    results = []
    for h in heads:
        results.append(O.psa_head(inp.as_f64("q", 0, h), inp.as_f64("k", 0, h // grp),
                                  inp.as_f64("v", 0, h // grp), w.q_blk, w.kv_blk, tau, w.causal,
                                  w.forced_prefix_tokens,
                                  sim_threshold=None if sim_threshold <= -1 else sim_threshold))
    dt = time.perf_counter() - t0
    dense = w.dense_flops() / (w.B * w.Hq) * n_heads
    return (dense / dt / 1e12, dt, cores,
            f"{n_heads} of {w.B * w.Hq} heads of {w.name}, whole forward (pyramid, mask, attention), "
            f"NumPy float64, BLAS threads = {cores}", results)


def sampled_parity(w: W.Workload, results, level_map, out) -> dict:
    """GPU against the oracle on the sampled heads (batch 0): level-map entries
    that differ, split by the parity criterion of the tests into those excused
    as near-threshold (the oracle's cumulative mass within 1e-5 of a separating
    threshold) or near-tie (a block of the GPU's level within 1e-4 relative
    mass) and unexplained ones; and the output error over the query blocks
    whose map rows agree (so both sides attend to the same keys)."""
    from tests.gpu_common import map_mismatch_report
    mism, n_map, err_max, num, den = 0, 0, 0.0, 0.0, 0.0
    une = thr = tie = 0
    tau = W.thresholds(w)
    for h, r in enumerate(results):
        gm = level_map[0, h].cpu().numpy()
        om = r.mask.level_map
        mism += int((gm != om).sum())
        n_map += om.size
        u, t1, t2 = map_mismatch_report(gm, r.mask, tau, w.assign)
        une, thr, tie = une + u, thr + t1, tie + t2
        same = np.all(gm == om, axis=1)
        rows = np.concatenate([np.arange(a * w.q_blk, min((a + 1) * w.q_blk, w.N))
                               for a in np.nonzero(same)[0]] or [np.zeros(0, dtype=np.int64)])
        g = out[0, h].float().cpu().numpy().astype(np.float64)[rows]
        ref = r.O[rows]
        d = np.abs(g - ref)
        err_max = max(err_max, float(d.max()) if d.size else 0.0)
        num += float(d.sum())
        den += float(np.abs(ref).sum())
    return {"heads": len(results), "map_entries_differing": mism, "map_entries": n_map,
            "near_threshold": thr, "near_tie": tie, "unexplained": une,
            "max_abs": err_max, "mean_rel": num / den if den else 0.0,
            "note": "output compared on query blocks whose GPU and oracle map rows agree"}


def run_cpu_baseline_all():
    """The oracle as it stands on every workload: one head each (the tiny
    workload whole), extrapolated to the whole workload by its head count, with
    BLAS threads = the cores; and the tiny workload again on one thread.  One
    JSON line per timing."""
    cores = len(os.sched_getaffinity(0))
    for w in W.WORKLOADS:
        n = w.B * w.Hq if w.name == "tiny_f32" else 1
        val, dt, cores, sample, _ = cpu_sample(w, n)
        print(json.dumps({"cpu_baseline": w.name, "value": val, "unit": UNIT, "cores": cores,
                          "seconds_sample": round(dt, 3),
                          "seconds_whole_workload": round(dt * w.B * w.Hq / n, 2),
                          "extrapolated": n < w.B * w.Hq, "sample": sample}), flush=True)
    from threadpoolctl import threadpool_limits
    w = W.BY_NAME["tiny_f32"]
    with threadpool_limits(limits=1):
        val, dt, _, sample, _ = cpu_sample(w, w.B * w.Hq)
    print(json.dumps({"cpu_baseline": w.name, "value": val, "unit": UNIT, "cores": 1,
                      "seconds_sample": round(dt, 3), "seconds_whole_workload": round(dt, 3),
                      "extrapolated": False,
                      "sample": sample.replace(f"BLAS threads = {cores}", "BLAS threads = 1")}),
          flush=True)


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = W.BY_NAME[args.workload]
    times, val = [], None
    for _ in range(args.warmup):
        cpu_sample(w, 1)
    for _ in range(args.steps):
        val, dt, cores, sample, _ = cpu_sample(w, 1)
        times.append(dt)
    tot = sum(times)
    dense_head = w.dense_flops() / (w.B * w.Hq)
    value = dense_head * len(times) / tot / 1e12
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "sample": "one head per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------- clock sampler

class ClockSampler:
    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _loop(self):
        nv = self.nv
        names = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                 "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4, "sync_boost": 0x10}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._loop, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------- our leg

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import level_sparse_attention_b200 as P

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = W.BY_NAME[args.workload]
    tau = W.thresholds(w)
    if args.heads:
        grp = w.Hq // w.Hkv
        w = W.with_overrides(w, Hq=args.heads, Hkv=max(1, args.heads // grp))
    w_job = w                                 # the whole job's problem
    if args.shard == "heads":
        # strong scaling: this rank's heads of one problem (its own slice of
        # the generator's heads; the shards need no exchange)
        q0, q1, kv0, kv1 = P.head_shard(w.Hq, w.Hkv, rank, world)
        full = W.make_inputs(w, heads_q=list(range(q0, q1)), heads_kv=list(range(kv0, kv1)))
        w = W.with_overrides(w, Hq=q1 - q0, Hkv=kv1 - kv0)
        inp = W.Inputs(w, np.ascontiguousarray(full.q[:, q0:q1]),
                       np.ascontiguousarray(full.k[:, kv0:kv1]), np.ascontiguousarray(full.v[:, kv0:kv1]))
    else:
        inp = W.make_inputs(w, batch0=rank_batch0(rank, w.B))
    p = P.make_params(w.B, w.Hq, w.Hkv, w.N, w.d, w.q_blk, w.kv_blk, tau, w.causal,
                      w.forced_prefix_tokens, 0.0,
                      torch.bfloat16 if w.dtype == "bf16" else torch.float32,
                      sim_threshold=args.sim_threshold)

    def host(x):
        t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16" \
            else torch.from_numpy(x)
        return t.pin_memory()

    hq, hk, hv = host(inp.q), host(inp.k), host(inp.v)
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    ws = P.new_workspace(p, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    lm = torch.empty(P.map_shape(p), dtype=torch.int8, device=dev)

    def step():
        P.build_pyramid(p, k, v, ws)
        P.score_and_mask(p, q, ws, lm)
        P.attention_fwd(p, q, k, v, ws, out, lse)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    P.check_device(p, ws)

    # executed (algorithmic) attention FLOPs of this map: 4*d*sum(valid q rows * kept keys)
    counts = P.workspace_view(ws, P.workspace_layout(p)["counts"], (w.B, w.Hq, w.Nq, 4),
                              torch.int32).cpu().numpy().astype(np.int64)
    keys_per_row = counts[..., 0] * 64 + counts[..., 1] * 32 + counts[..., 2] * 16 + counts[..., 3] * 8
    qrows = np.array([min(w.q_blk, w.N - a * w.q_blk) for a in range(w.Nq)], dtype=np.int64)
    executed = float(4 * w.d * (keys_per_row * qrows[None, None, :]).sum())
    # (tail KV blocks and the causal diagonal make this an upper bound of a few
    #  keys per row; the oracle's executed_flops is exact)
    dense = w.dense_flops()
    padded_keys = float(np.ceil(keys_per_row / 128.0).sum() * 128)

    # The timed loop of K steps is repeated until the timed region lasts at
    # least --min-timed-seconds (every rank takes the same number of repeats:
    # the estimate is the max over ranks), so that the clock sampler sees it.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        flush.zero_()
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    est_ms = max_over_ranks(e0.elapsed_time(e1) / 3, world, dev)
    reps = max(1, math.ceil(args.min_timed_seconds * 1e3 / (args.steps * est_ms)))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps * reps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps * reps):
            flush.zero_()                       # L2 flush outside the timed events
            e = ev[i]
            e[0].record(stream)
            P.build_pyramid(p, k, v, ws)
            e[1].record(stream)
            P.score_and_mask(p, q, ws, lm)
            e[2].record(stream)
            P.attention_fwd(p, q, k, v, ws, out, lse)
            e[3].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    pyr_ms = [e[0].elapsed_time(e[1]) for e in ev]
    mask_ms = [e[1].elapsed_time(e[2]) for e in ev]
    attn_ms = [e[2].elapsed_time(e[3]) for e in ev]
    ms = max_over_ranks(sum(step_ms), world, dev) / (args.steps * reps)
    # weak: every rank's batch has the workload's dense FLOPs; strong: the
    # ranks' shares add up to one problem's
    value = (whole_job_tflops(dense, world, ms) if args.shard == "batch"
             else w_job.dense_flops() / (ms * 1e-3) / 1e12)

    # end to end through the public API with host buffers: psa_forward_host
    # copies Q, K, V from pinned host memory and O back, per head group on two
    # copy streams, pipelined behind the kernels; every step inside the timed
    # region (the compute stream completes after the last copy back)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_steps = max(3, min(args.steps, 20))
    P.forward_host(p, hq, hk, hv, hout, q, k, v, out, ws, h2d, d2h, stream=stream)   # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        P.forward_host(p, hq, hk, hv, hout, q, k, v, out, ws, h2d, d2h, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    job_dense = dense * world if args.shard == "batch" else w_job.dense_flops()
    P.check_device(p, ws)

    # the backward pass (dQ, dK, dV with this map held fixed), timed the same
    # way: L2 flushed between steps, CUDA events on the launch stream.  Its
    # executed FLOPs are 5 tile GEMMs (S, dP, dQ, dK, dV) against the
    # forward's 2, over the same packed tiles.
    bwd = None
    if not args.no_backward:
        gen = torch.Generator(device=dev).manual_seed(1234)
        dout = torch.randn(out.shape, generator=gen, device=dev, dtype=torch.float32).to(out.dtype)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = P.new_backward_workspace(p, dev)

        def bstep():
            P.backward(p, q, k, v, out, lse, dout, ws, bws, dq, dk, dv)

        step()                                   # the forward this backward belongs to
        for _ in range(max(3, args.warmup)):
            bstep()
        torch.cuda.synchronize()
        P.check_device(p, ws)
        b_steps = max(3, min(args.steps, 20))
        bev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(b_steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(b_steps):
            flush.zero_()
            bev[i][0].record(stream)
            bstep()
            bev[i][1].record(stream)
        torch.cuda.synchronize()
        P.check_device(p, ws)
        b_ms = max_over_ranks(sum(b[0].elapsed_time(b[1]) for b in bev) / b_steps, world, dev)
        b_exec = 2.5 * executed
        bwd = {"ms_per_call": b_ms, "steps": b_steps, "call": "psa_backward",
               "stages": "pyramid rebuild, D = dO . O, attention gradient, unpool",
               "executed_flops": b_exec,
               "executed_tflops": b_exec * (world if args.shard == "batch" else 1) / (b_ms * 1e-3) / 1e12,
               "dense_equiv_tflops": 2.5 * (job_dense / (b_ms * 1e-3) / 1e12),
               "traffic": BWD_TRAFFIC.get((w.name, w.Hq, attn_source_hash(BWD_SOURCES))),
               "gpu_launches_per_call": 4}
    kernels_us = None
    if args.profile_kernels:
        # per-kernel device times over extra steps (not the timed ones)
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for _ in range(args.steps):
                flush.zero_()
                step()
                if bwd is not None:
                    flush.zero_()
                    bstep()
            torch.cuda.synchronize()
        agg = {}
        for e in prof.events():
            if e.device_type == torch.autograd.DeviceType.CUDA and "psa::" in e.name:
                name = e.name.replace("psa::(anonymous namespace)::", "").replace("void ", "")
                name = name.split("(")[0]
                agg.setdefault(name, []).append(e.device_time_total)
        kernels_us = {k: round(statistics.median(v), 2) for k, v in sorted(agg.items())}

    bf16_peak, hbm_peak, peak_kind = peaks()
    attn_avg = sum(attn_ms) / len(attn_ms)
    achieved = executed / (attn_avg * 1e-3) / 1e12
    es = 2 if w.dtype == "bf16" else 4
    pyr_avg = sum(pyr_ms) / len(pyr_ms)
    mask_avg = sum(mask_ms) / len(mask_ms)
    pyr_gbs = pyramid_bytes(w) / (pyr_avg * 1e-3) / 1e9
    mask_gbs = mask_bytes(w) / (mask_avg * 1e-3) / 1e9
    if bwd is not None:
        bwd["frac_of_peak"] = bwd["executed_tflops"] / (world if args.shard == "batch" else 1) / bf16_peak
        bwd["peak_kind"] = f"{peak_kind} bf16 burst"
    if rank != 0:
        return
    cpu, parity = None, None
    if not args.no_cpu_baseline and world == 1:
        val, dt, cores, sample, results = cpu_sample(w, args.cpu_sample_heads, args.sim_threshold)
        cpu = {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(dt, 2)}
        parity = sampled_parity(w, results, lm, out)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak" if args.shard == "batch" else "strong",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded smooth 3-D field + noise)",
        "config": {"workload": w.name, "global_batch": w.B * world if args.shard == "batch" else w.B,
                   "shard": args.shard, "B": w.B, "Hq": w_job.Hq, "Hkv": w_job.Hkv, "N": w.N, "d": w.d,
                   "q_blk": w.q_blk, "kv_blk": w.kv_blk, "tau": [round(t, 6) for t in tau],
                   "causal": w.causal, "skipped_dense_fraction": 1.0 - executed / dense,
                   "sim_threshold": args.sim_threshold,
                   "l2": "flushed between steps (256 MiB write, outside the timed events)",
                   "timed_repeats": reps,
                   "timing": f"{args.steps} timed steps, repeated {reps} times back to back "
                             f"(>= {args.min_timed_seconds} s of timed region for the clock "
                             f"samples); ms_per_step is the mean over all of them",
                   "parallelism": (f"independent batch per GPU x{world}" if args.shard == "batch"
                                   else f"heads of one problem split over {world} GPUs")},
        "ms_per_call": ms, "pct_bf16_peak_dense_equiv": 100.0 * value / world / bf16_peak,
        "executed_tflops": executed * (world if args.shard == "batch" else 1) / (ms * 1e-3) / 1e12,
        "kernel_ms": {"pyramid": pyr_avg, "mask": mask_avg, "attention": attn_avg},
        "hbm": {"peak_gbs": hbm_peak, "peak_kind": f"{peak_kind} copy",
                "pyramid": {"bytes": pyramid_bytes(w), "gbs": pyr_gbs, "frac": pyr_gbs / hbm_peak},
                "mask": {"bytes": mask_bytes(w), "gbs": mask_gbs, "frac": mask_gbs / hbm_peak}},
        "roofline": {"kernel": "attn_tc_kernel", "bound": "tensor", "achieved": achieved,
                     "peak": bf16_peak, "peak_kind": f"{peak_kind} bf16 burst", "unit": "TFLOP/s",
                     "frac": achieved / bf16_peak,
                     "traffic": ATTN_TRAFFIC.get((w.name, w.Hq, attn_source_hash())),
                     "executed_flops_per_launch": executed,
                     "padding_fraction": 1.0 - (keys_per_row.sum() / max(padded_keys, 1.0))},
        "backward": bwd,
        "cpu_baseline": cpu,
        "parity": parity,
        "e2e": {"value": job_dense / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "ms_per_step": e2e_ms, "call": "psa_forward_host",
                "head_groups": P.host_groups(p),
                "h2d_bytes_per_step": int((q.numel() + k.numel() + v.numel()) * es),
                "d2h_bytes_per_step": int(out.numel() * es)},
        "gpu_launches": 5 * args.steps * reps,
        "kernels_us": kernels_us,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.cpu_baseline_all:
        return run_cpu_baseline_all() if rank == 0 else None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
