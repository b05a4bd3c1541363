"""Benchmark of one video-DiT attention layer: Top-p block routing + block-sparse attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dit] [--impl ours|reference]

A step is one pass of the whole hot path over one synthetic layer already resident in HBM:
fvattn_route (pool -> fp64 scores/softmax/Top-p -> CSR, loads, tile order) followed by
fvattn_sparse_attn. The layer is B=1, H=40, S=32760 (21 frames x 1560 tokens), d=128, bf16,
block 64, p=0.9 with the diagonal forced; inputs (1 GB of Q, K, V) are larger than L2.

`value` is the effective TFLOPS of the step: attention FLOPs of the selected blocks only
(4*d per selected query/key token pair) divided by the step time.

With N > 1 GPUs (torchrun, one rank per GPU) the one layer is split over the ranks by head: each
rank holds H/N heads over the whole sequence (the layout sequence parallelism reaches after its
all-to-all), routes them, and runtime head migration between ranks (rlb.balanced_attention:
all-gather of per-head loads, the plan, point-to-point moves of Q, K, V and O) evens out the
ranks' loads before and during the attention. --ulysses starts instead from sequence-sharded
inputs (every rank has all heads of its S/N-token slice) and adds the sequence-to-head and
head-to-sequence all-to-alls (ulysses_attention). Strong scaling: the layer is fixed, the time is
the max over ranks. --sharded runs this path on one GPU too; --replicas gives every rank its own
independent layer instead (weak scaling).

--impl reference times the CPU oracle (fp64 NumPy) on a bounded sample of the same layer (the same
input draw as the GPU arm, copied to the host).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn effective TFLOPS & ms per layer at S=32760,H=40,p=0.9; % bf16 peak"
UNIT = "TFLOPS"
NOMINAL_BF16_TFLOPS = 2250.0    # B200 datasheet dense bf16 (context: the roofline uses the measured peak)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK}, "measured"
    return dict(FALLBACK), "fallback"


def env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def workload_desc(w, mode: str = "topp", topk_frames: int = 4, sasa_coef: float = 0.0, sasa_trigger: int = 1,
                  frame_exact: bool = False) -> str:
    sel = (f"p={w.p},diag forced" if mode == "topp" else
           f"frame top-k={topk_frames} + frames +-1 + frame 0 + diag" + (", token-exact" if frame_exact else ""))
    if sasa_coef > 0:
        sel += f",tile slack augmentation coef={sasa_coef} trigger={sasa_trigger}"
    return (f"{w.name}: B={w.B},H={w.H},S={w.S} ({w.frames} frames x {w.frame_len} tokens),d={w.d},{w.dtype},"
            f"block=64,{sel}")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark(self, which: str):
        """Host time of the start / end of the timed region: only samples between the two count."""
        setattr(self, "t_" + which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        import datetime
        t0, t1 = getattr(self, "t_start", None), getattr(self, "t_end", None)
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        for _, c, m, rs in (inside or rows):          # a region shorter than the interval: every sample
            sm.append(c)
            mx.append(m)
            for n, v in zip(names, rs):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ FLOP / byte accounting

def selected_flops_from_csr(csr, S: int, d: int):
    """4*d*sum over selected (query block i, key block j) of valid-token counts n_i*n_j."""
    import torch
    nb = csr.nb
    n = torch.full((nb,), 64, dtype=torch.int64, device=csr.row_ptr.device)
    n[-1] = S - 64 * (nb - 1)
    rp = csr.row_ptr.long()
    nnz = int(csr.nnz.item())
    counts = rp[1:] - rp[:-1]
    rows = torch.repeat_interleave(torch.arange(counts.numel(), device=rp.device), counts)
    qi = rows % nb
    kj = csr.col_idx[:nnz].long()
    pairs = int((n[qi] * n[kj]).sum().item())
    padded = int(counts.sum().item()) * 64 * 64
    kv_tokens = int(n[kj].sum().item())
    return 4 * d * pairs, nnz, 4 * d * padded, kv_tokens


def selected_flops_exact(csr, S: int, d: int) -> int:
    """4*d * the (query token, key token) pairs that token-exact frame mode attends: per CSR
    entry, the allowed (query frame side, key frame side) quarters of the block pair, counted
    over valid tokens only (the codes of fvattn_csr.col_code)."""
    import torch
    nb = csr.nb
    rp = csr.row_ptr.long()
    nnz = int(csr.nnz.item())
    counts = rp[1:] - rp[:-1]
    rows = torch.repeat_interleave(torch.arange(counts.numel(), device=rp.device), counts)
    i = rows % nb
    j = csr.col_idx[:nnz].long()
    code = csr.col_code[:nnz].long()
    nq = torch.clamp(S - 64 * i, max=64)
    nk = torch.clamp(S - 64 * j, max=64)
    qrow = torch.minimum((code >> 16) & 255, nq)
    kcol = torch.minimum((code >> 8) & 255, nk)
    rq = (qrow, nq - qrow)
    ck = (kcol, nk - kcol)
    pairs = sum(((code >> (2 * a + b)) & 1) * rq[a] * ck[b] for a in range(2) for b in range(2))
    return 4 * d * int(pairs.sum().item())


def tile_mma_flops(csr, d: int) -> int:
    """FLOPs the attention kernel's MMAs issue: every key block of a 128-row tile's union is one
    128 x 64 step of S = Q K^T and O += P V, whichever of the tile's two rows selected it."""
    return 4 * d * 128 * 64 * int(csr.tile_cost.long().sum().item())


def router_bytes(BH: int, S: int, d: int, esize: int, nb: int, nnz: int) -> int:
    nt = BH * ((nb + 1) // 2)
    return 2 * BH * S * d * esize + 4 * (BH * nb + 1) + 4 * nnz + 8 * BH + 8 * nt + 8


def traffic_from_profile(kernel_src: str):
    """dram bytes per launch of the attention kernel from the committed ncu summary, if it was
    taken on the current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "attn_tc_dit_layer.traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    if d.get("source_sha256_16") != h:
        return None
    return d.get("dram_bytes_per_launch")


def reduce_over_ranks(ms: float, flops: float, device):
    """Max of the device-timed milliseconds and sum of the work over all ranks (the job's
    time is its slowest rank's; its work is every rank's). Identity on one process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), float(flops)
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    f = torch.tensor([float(flops)], device=device, dtype=torch.float64)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_layer(w, q_cpu, k_cpu):
    """The oracle's routing of the whole layer (its masks and selected FLOPs), the scale of every
    sample below. Not timed by the reference arm; timed in full by the GPU arm's cpu_baseline."""
    import oracle
    BH = w.B * w.H
    Q = q_cpu.reshape(BH, w.S, w.d)
    K = k_cpu.reshape(BH, w.S, w.d)
    t0 = time.perf_counter()
    r = oracle.route(Q, K, oracle.RouteCfg(p=w.p, force_diag=True))
    t_route = time.perf_counter() - t0
    return r, oracle.selected_flops(r["mask"], w.S, 64, w.d), t_route


def oracle_sample(w, q_cpu, k_cpu, v_cpu, r, layer_flops, n_items: int, route_heads: int, seed: int,
                  t_route_all=None):
    """Time the oracle (as it stands) on a bounded sample of the layer and scale it to the layer:
    the router on `route_heads` heads (time x heads of the layer; or the measured whole-layer
    router time t_route_all) plus exact attention of `n_items` seeded query blocks (time x the
    layer's selected FLOPs / the sample's). Returns (estimated layer seconds, description)."""
    import numpy as np
    import oracle
    BH = w.B * w.H
    Q = q_cpu.reshape(BH, w.S, w.d)
    K = k_cpu.reshape(BH, w.S, w.d)
    V = v_cpu.reshape(BH, w.S, w.d)
    rng = np.random.default_rng(seed)
    if t_route_all is None:
        heads = rng.choice(BH, size=route_heads, replace=False)
        t0 = time.perf_counter()
        oracle.route(Q[heads], K[heads], oracle.RouteCfg(p=w.p, force_diag=True))
        t_route = (time.perf_counter() - t0) * BH / route_heads
        rdesc = f"router on {route_heads}/{BH} heads scaled by heads"
    else:
        t_route = t_route_all
        rdesc = f"router on all {BH} heads"
    # query blocks drawn in proportion to their selected FLOPs, so that the sample's time per FLOP
    # is that of the layer
    nrow = np.array([min(w.S, (i + 1) * 64) - i * 64 for i in range(w.nb)])
    wts = (r["mask"] * nrow[None, None, :]).sum(axis=2) * nrow[None, :]
    n_items = min(n_items, int((wts > 0).sum()))
    flat = rng.choice(wts.size, size=n_items, replace=False, p=(wts / wts.sum()).reshape(-1))
    items = [(int(f // w.nb), int(f % w.nb)) for f in flat]
    t0 = time.perf_counter()
    oracle.attention_rows(Q, K, V, r["mask"], 1.0 / math.sqrt(w.d), items)
    t_attn = time.perf_counter() - t0
    f_items = sum(4 * w.d * int(nrow[i]) * int(nrow[r["mask"][b, i]].sum()) for b, i in items)
    t_layer = t_route + t_attn * (layer_flops / max(f_items, 1))
    desc = (f"fp64 NumPy oracle: {rdesc} ({t_route:.1f} s for the layer) + exact attention of {n_items} query "
            f"blocks drawn by selected-FLOP weight ({t_attn:.2f} s), scaled by the layer's selected FLOPs")
    return t_layer, desc


def layer_inputs_host(w):
    """The layer's Q, K, V as the GPU arm draws them (on the GPU when there is one), on the host."""
    import torch
    from workloads import make_inputs
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = make_inputs(w, device=dev)
    return x["q"].cpu(), x["k"].cpu(), x["v"].cpu(), dev


def run_reference(args, w):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    q, k, v, drawn_on = layer_inputs_host(w)
    r, layer_flops, _ = oracle_layer(w, q, k)
    threads = oracle_threads()
    times, wall = [], []
    desc = None
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        t_layer, desc = oracle_sample(w, q, k, v, r, layer_flops, n_items=4, route_heads=1, seed=s)
        if s >= args.warmup:
            times.append(t_layer)
            wall.append(time.perf_counter() - t0)
    t = statistics.median(times)
    value = layer_flops / t / 1e12
    desc += f"; inputs drawn on the {drawn_on} as the GPU arm's; median over {args.steps} samples"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w), "l2": "n/a (CPU)"},
            # ms_per_step is the layer time the sample extrapolates to; the samples themselves took:
            "measured_sample_ms_per_step": statistics.mean(wall) * 1e3,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def emulate_ranks(fv, q, k, v, cfg, csr, out, stream, R: int, target: float, budget: int, reps: int = 5):
    """Runtime load balancing over R ranks, emulated on this GPU: the layer's H heads are split
    into R contiguous groups (the heads each rank holds under sequence parallelism), the
    migration plan is made from the routed layer's per-head loads, and the attention of each
    rank's head set is timed on this GPU (CUDA events), before and after the plan. The step of
    an R-GPU job waits for its slowest rank: the critical path is the maximum over ranks."""
    import numpy as np
    import torch
    from block_sparse_top_fvattn_b200 import rlb
    B, H, S, d = q.shape
    if B != 1 or H % R:
        return {"skipped": f"H={H} is not a multiple of {R} ranks"}
    Hl = H // R
    fv.route(q, k, cfg, csr=csr)
    torch.cuda.synchronize()
    loads = csr.head_load.cpu().numpy().reshape(R, Hl)
    plan = rlb.make_plan(loads, target, budget)
    full_order = csr.tile_order.clone()
    n_all = int(csr.status[3].item())
    owner = np.repeat(np.arange(R), Hl)
    after = owner.copy()
    for s_, h, dst in plan.moves:
        after[s_ * Hl + h] = dst

    def rank_ms(owners, r):
        act = torch.tensor((owners == r).astype(np.uint8), device=q.device)
        times = []
        for it in range(reps + 1):
            csr.tile_order.copy_(full_order)
            csr.status[3].fill_(n_all)
            fv.select_heads(csr, act)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fv.sparse_attn(q, k, v, csr, out=out)
            b.record(stream)
            torch.cuda.synchronize()
            if it:
                times.append(a.elapsed_time(b))
        return float(np.median(times))

    t_before = [rank_ms(owner, r) for r in range(R)]
    t_after = [rank_ms(after, r) for r in range(R)]
    csr.tile_order.copy_(full_order)
    csr.status[3].fill_(n_all)
    esize = q.element_size()
    return {
        "ranks": R, "heads_per_rank": Hl, "target_imbalance": target, "max_moves_per_rank": budget,
        "moves": len(plan.moves), "load_imbalance_before": plan.imbalance_before,
        "load_imbalance_after": plan.imbalance_after,
        "rank_attn_ms_before": t_before, "rank_attn_ms_after": t_after,
        "critical_path_ms_before": max(t_before), "critical_path_ms_after": max(t_after),
        "time_imbalance_before": max(t_before) / (sum(t_before) / R),
        "time_imbalance_after": max(t_after) / (sum(t_after) / R),
        "migrated_bytes": len(plan.moves) * 4 * S * d * esize,
        "note": "per-rank attention of each rank's head set timed on one B200; migration traffic (Q, K, V out, O "
                "back) not included in the times",
    }


def run_sharded(args, w):
    """The layer split over the ranks (see the module docstring): Ulysses sequence parallelism
    with runtime head migration. Strong scaling; the time of a step is the slowest rank's."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_top_fvattn_b200 as fv
    from block_sparse_top_fvattn_b200 import rlb, ulysses
    from workloads import make_inputs

    rank, world, local = env_rank()
    torch.cuda.set_device(local)                 # before the process group: NCCL binds this device
    dev = torch.device("cuda", local)
    if "MASTER_ADDR" in os.environ:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:                                        # one process without torchrun (--sharded)
        dist.init_process_group("nccl", init_method=f"file://{tempfile.mktemp(prefix='fvattn_pg_')}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120), device_id=dev)
    R = dist.get_world_size()
    fv.load()
    pk, pk_src = peaks()
    B, H, S, d = w.B, w.H, w.S, w.d
    if B != 1 or H % R or S % R:
        raise SystemExit(f"the sharded layer needs B = 1 and H, S divisible by {R} ranks")
    x = make_inputs(w, device=dev)              # the one layer, drawn identically on every rank
    Sl = S // R
    ql, kl, vl = (x[n][:, :, rank * Sl:(rank + 1) * Sl].contiguous() for n in ("q", "k", "v"))
    cfg = fv.RouteConfig(p=w.p, force_diag=True)
    kernels = rlb.Kernels(cfg)
    # the layer's selected FLOPs (the routing does not depend on how the layer is split)
    csr_full = fv.route(x["q"], x["k"], cfg)
    flops, nnz, _, _ = selected_flops_from_csr(csr_full, S, d)
    density = nnz / (B * H * csr_full.nb * csr_full.nb)
    # this rank's heads over the whole sequence, for the attention kernel's own roofline figure
    Hl = H // R
    qh, kh, vh = (x[n][:, rank * Hl:(rank + 1) * Hl].contiguous() for n in ("q", "k", "v"))
    del x, csr_full
    torch.cuda.empty_cache()

    if args.ulysses:
        def step(balance):
            return ulysses.ulysses_attention(ql, kl, vl, cfg, balance=balance, target=args.rlb_target,
                                             max_moves_per_rank=args.rlb_budget, kernels=kernels, overlap_pool=True)
    else:
        ql, kl, vl = qh, kh, vh                  # this rank's heads over the whole sequence
        out_h = torch.empty_like(qh)

        def step(balance):
            if balance:
                return rlb.balanced_attention(ql, kl, vl, cfg, target=args.rlb_target,
                                              max_moves_per_rank=args.rlb_budget, kernels=kernels)
            kernels.attend(ql, kl, vl, kernels.route(ql, kl), None, out_h)
            return out_h, None

    def timed(n, balance):
        dist.barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        plan = None
        for _ in range(n):
            _, plan = step(balance)
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / n
        per_rank = [torch.zeros(1, dtype=torch.float64, device=dev) for _ in range(R)]
        dist.all_gather(per_rank, torch.tensor([ms], dtype=torch.float64, device=dev))
        dist.barrier()
        return [float(t.item()) for t in per_rank], plan

    for _ in range(max(args.warmup, 3)):
        step(True)
    torch.cuda.synchronize()
    n_cmp = min(args.steps, 20)
    unbalanced, _ = timed(n_cmp, False)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    sampler.mark("start")
    balanced, plan = timed(args.steps, True)
    sampler.mark("end")
    clocks = sampler.stop()
    ms_step = max(balanced)
    value = flops / (ms_step * 1e-3) / 1e12

    # end to end: this rank's slice of Q, K, V from pinned host memory in, its slice of O out
    hq, hk, hv = (t.cpu().pin_memory() for t in (ql, kl, vl))
    ho = torch.empty(ql.shape, dtype=ql.dtype, pin_memory=True)
    n_e2e = max(3, min(6, args.steps))
    dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n_e2e):
        ql.copy_(hq, non_blocking=True)
        kl.copy_(hk, non_blocking=True)
        vl.copy_(hv, non_blocking=True)
        o, _ = step(True)
        ho.copy_(o, non_blocking=True)
    b.record()
    torch.cuda.synchronize()
    e_ms = torch.tensor([a.elapsed_time(b) / n_e2e], dtype=torch.float64, device=dev)
    dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
    e_ms = float(e_ms.item())

    # the attention kernel alone on this rank's own heads (outside the timed region)
    csr_l = fv.route(qh, kh, cfg)
    out_l = torch.empty_like(qh)
    f_local, _, _, _ = selected_flops_from_csr(csr_l, S, d)
    ts = []
    for i in range(8):
        ea = torch.cuda.Event(enable_timing=True)
        eb = torch.cuda.Event(enable_timing=True)
        ea.record()
        fv.sparse_attn(qh, kh, vh, csr_l, out=out_l)
        eb.record()
        torch.cuda.synchronize()
        if i >= 3:
            ts.append(ea.elapsed_time(eb))
    attn_local_tflops = f_local / (statistics.median(ts) * 1e-3) / 1e12
    if fv.read_status(csr_l) != 0:
        raise RuntimeError("device status after the attention of the local heads")
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return 0
    esize = ql.element_size()
    loads = plan.loads if plan is not None else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": R, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w),
                   "parallelism": (f"sequence parallel x{R} (Ulysses all-to-all over NCCL) + runtime head migration"
                                   if args.ulysses else f"heads split over {R} ranks + runtime head migration (NCCL)"),
                   "l2": "inputs larger than L2"},
        "density": density, "selected_flops_per_layer": flops,
        "rlb": {"heads_per_rank": Hl, "rank_head_loads": loads.tolist() if loads is not None else None,
                "moves": len(plan.moves) if plan is not None else 0,
                "load_imbalance_before": plan.imbalance_before if plan is not None else None,
                "load_imbalance_after": plan.imbalance_after if plan is not None else None,
                "rank_ms_unbalanced": unbalanced, "rank_ms_balanced": balanced,
                "time_imbalance_unbalanced": max(unbalanced) / (sum(unbalanced) / R),
                "time_imbalance_balanced": max(balanced) / (sum(balanced) / R),
                "migrated_bytes_per_step": (len(plan.moves) if plan is not None else 0) * 4 * S * d * esize},
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (rank 0's heads, timed alone)",
                     "achieved": attn_local_tflops, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": attn_local_tflops / pk["bf16_tflops"], "traffic": None,
                     "peak_kind": f"bf16 burst ({pk_src})"},
        "e2e": {"value": flops / (e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
                "h2d_bytes_per_step": 3 * ql.numel() * esize * R, "d2h_bytes_per_step": ql.numel() * esize * R,
                "pipeline": "per rank: its part of Q, K, V in, the layer, its part of O out (no overlap)"},
        "cpu_baseline": None,
        # rank 0's launches of this library's kernels in the timed region: the router (pooling per
        # arriving slice + 4 kernels, or 5), the attention, and with head migration fvattn_select_heads
        # on a sender and the router + attention of the received heads on a receiver
        "gpu_launches": args.steps * (((R + 4) if (args.ulysses and Sl % 64 == 0) else 5) + 1 +
                                      (1 if plan is not None and any(m[0] == 0 for m in plan.moves) else 0) +
                                      (6 if plan is not None and any(m[2] == 0 for m in plan.moves) else 0)),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_sparse_top_fvattn_b200 as fv
    from workloads import make_inputs

    rank, world, local = env_rank()
    if args.sharded or (world > 1 and not args.replicas):
        return run_sharded(args, w)
    torch.cuda.set_device(local)                 # before the process group: NCCL binds this device
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120), device_id=dev)
    fv.load()
    pk, pk_src = peaks()

    # every rank draws its own layer (weak scaling): seed offset by rank
    x = make_inputs(w, device=dev, seed=w.seed + 1000 * rank)
    q, k, v = x["q"], x["k"], x["v"]
    B, H, S, d = q.shape
    BH = B * H
    if args.mode == "frame_topk":
        cfg = fv.RouteConfig(mode="frame_topk", topk_frames=args.topk_frames, frame_len=w.frame_len, frame_window=1,
                             force_first_frame=True, force_diag=True, frame_exact=args.frame_exact)
    else:
        cfg = fv.RouteConfig(p=w.p, force_diag=True, sasa_coef=args.sasa_coef, sasa_trigger=args.sasa_trigger)
    csr = fv.alloc_csr(B, H, S, dev, codes=cfg.frame_exact)
    ws = torch.empty(fv.workspace_bytes(q, cfg), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()

    # --plain-order: ascending tile ids instead of the router's longest-first order (to measure
    # what the order buys; a diagnostic, not the product path)
    plain = torch.arange(csr.tile_order.numel(), dtype=torch.int32, device=dev) if args.plain_order else None

    def route_now():
        fv.route(q, k, cfg, csr=csr, workspace=ws)
        if plain is not None:
            csr.tile_order.copy_(plain)

    def step():
        route_now()
        fv.sparse_attn(q, k, v, csr, out=out)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if fv.read_status(csr) != 0:
        raise RuntimeError(f"device status {fv.read_status(csr)}")
    flops, nnz, flops_padded, kv_tokens = selected_flops_from_csr(csr, S, d)
    if cfg.frame_exact:
        flops = selected_flops_exact(csr, S, d)
    density = nnz / (BH * csr.nb * csr.nb)
    mma_flops = tile_mma_flops(csr, d)

    # timed region: K steps; per-kernel events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler.mark("start")
    t_start.record(stream)
    routed_steps = 0
    for s in range(args.steps):
        ev[s][0].record(stream)
        if s % args.refresh_every == 0:              # routing reuse: refresh every N steps
            route_now()
            routed_steps += 1
        ev[s][1].record(stream)
        fv.sparse_attn(q, k, v, csr, out=out)
        ev[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    sampler.mark("end")
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    route_ms = [ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps) if s % args.refresh_every == 0]
    attn_ms = [ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)]
    total_ms, flops_all = reduce_over_ranks(total_ms, flops, dev)
    ms_step = total_ms / args.steps
    value = flops_all * args.steps / (total_ms * 1e-3) / 1e12
    attn_avg = statistics.mean(attn_ms)
    route_avg = statistics.mean(route_ms)
    attn_tflops = flops / (attn_avg * 1e-3) / 1e12
    rbytes = router_bytes(BH, S, d, q.element_size(), csr.nb, nnz)
    router_gbs = rbytes / (route_avg * 1e-3) / 1e9
    traffic = traffic_from_profile(os.path.join(ROOT, "block_sparse_top_fvattn_b200", "csrc", "attn_tc.cu"))

    # The same step captured once in a CUDA graph (route + attention, static buffers) and replayed
    # K times: what a caller that replays graphs sees, without per-call launch work on the host.
    graph = None
    if not args.no_graph and args.refresh_every == 1 and plain is None and world == 1:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step()
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(args.steps):
                g.replay()
            g1.record(stream)
            torch.cuda.synchronize()
            if fv.read_status(csr) != 0:
                raise RuntimeError(f"device status {fv.read_status(csr)}")
            gms = g0.elapsed_time(g1)
            graph = {"ms_per_step": gms / args.steps, "value": flops * args.steps / (gms * 1e-3) / 1e12,
                     "unit": UNIT, "steps": args.steps,
                     "note": "route + attention captured once in a CUDA graph, replayed; timed after the main region"}
            del g
        except Exception as exc:                   # reported, not fatal: the headline is the plain launches
            graph = {"error": f"{type(exc).__name__}: {exc}"}

    # SM busy-time imbalance of the persistent attention grid (outside the timed region): one
    # stamped launch on the router's longest-first order, one on ascending tile ids.
    sm_busy = None
    if q.dtype == torch.bfloat16 and not args.no_sm_busy:
        fv.route(q, k, cfg, csr=csr, workspace=ws)
        _, st_lpt = fv.sparse_attn_stamped(q, k, v, csr, out=out)
        csr.tile_order.copy_(torch.arange(csr.tile_order.numel(), dtype=torch.int32, device=dev))
        _, st_asc = fv.sparse_attn_stamped(q, k, v, csr, out=out)
        torch.cuda.synchronize()
        if fv.read_status(csr) != 0:
            raise RuntimeError(f"device status {fv.read_status(csr)}")
        a, b = fv.sm_busy_imbalance(st_lpt), fv.sm_busy_imbalance(st_asc)
        sm_busy = {"longest_first": round(a["imbalance"], 4), "ascending": round(b["imbalance"], 4),
                   "sms": a["sms"], "max_busy_ms": [round(a["max_ns"] / 1e6, 4), round(b["max_ns"] / 1e6, 4)],
                   "definition": "per SM: last CTA end - first CTA start (globaltimer); max / mean over SMs"}

    # End to end through the public API with host buffers (pinned): every step copies its Q, K, V
    # in and its O out inside the timed region. As a serving loop would, the transfers of
    # neighbouring steps overlap the compute: the inputs of step s+1 go up and the output of step
    # s-1 comes down while step s routes and attends (two device buffer sets, three streams).
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        dq = [torch.empty_like(q) for _ in range(2)]
        dk = [torch.empty_like(k) for _ in range(2)]
        dv = [torch.empty_like(v) for _ in range(2)]
        do = [torch.empty_like(out) for _ in range(2)]
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        n_e2e = max(3, min(6, args.steps))

        def e2e_steps(n, t0=None):
            for st in range(n):
                bb = st % 2
                if st >= 2:
                    s_in.wait_event(ev_cmp[bb])                  # step st-2 has finished reading buffer bb
                with torch.cuda.stream(s_in):
                    if st == 0 and t0 is not None:
                        t0.record(s_in)
                    dq[bb].copy_(hq, non_blocking=True)
                    dk[bb].copy_(hk, non_blocking=True)
                    dv[bb].copy_(hv, non_blocking=True)
                    ev_in[bb].record(s_in)
                s_cmp.wait_event(ev_in[bb])
                if st >= 2:
                    s_cmp.wait_event(ev_out[bb])                 # output buffer bb has been read back
                with torch.cuda.stream(s_cmp):
                    fv.route(dq[bb], dk[bb], cfg, csr=csr, workspace=ws)
                    fv.sparse_attn(dq[bb], dk[bb], dv[bb], csr, out=do[bb])
                    ev_cmp[bb].record(s_cmp)
                s_out.wait_event(ev_cmp[bb])
                with torch.cuda.stream(s_out):
                    ho[bb].copy_(do[bb], non_blocking=True)
                    ev_out[bb].record(s_out)

        e2e_steps(2)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        e2e_steps(n_e2e, t0=a)
        b.record(s_out)                                      # after the last step's read-back
        torch.cuda.synchronize()
        if fv.read_status(csr) != 0:
            raise RuntimeError("device status after the end-to-end steps")
        e_ms = a.elapsed_time(b) / n_e2e
        if world > 1:
            tt = torch.tensor([e_ms], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            e_ms = float(tt.item())
        e2e = {"value": flops_all / (e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
               "pipeline": "H2D of step s+1 and D2H of step s-1 overlap step s (2 buffer sets, 3 streams)",
               "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
               "d2h_bytes_per_step": out.numel() * out.element_size()}

    rlb_em = None
    if args.emulate_ranks > 1 and world == 1:
        rlb_em = emulate_ranks(fv, q, k, v, cfg, csr, out, stream, args.emulate_ranks, args.rlb_target,
                               args.rlb_budget)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
        r, layer_flops_oracle, t_route_all = oracle_layer(w, qh, kh)
        t_layer, desc = oracle_sample(w, qh, kh, vh, r, layer_flops_oracle, n_items=48, route_heads=BH, seed=0,
                                      t_route_all=t_route_all)
        cpu = {"value": layer_flops_oracle / t_layer / 1e12, "unit": UNIT, "cores": oracle_threads(),
               "kind": "oracle", "sample": desc + "; the GPU arm's input draw"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    # The denominator follows the clocks seen during the timed region: the burst GEMM figure when
    # the SMs held their maximum clock, the sustained (power-capped) one when the power cap was
    # active or the clock sat below 95 % of its maximum.
    capped = "sw_power_cap" in (clocks.get("reasons") or []) or (
        clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
    bf16_peak = pk["bf16_tflops_sustained"] if capped else pk["bf16_tflops"]
    peak_kind = ("bf16 sustained, power-capped clocks" if capped else "bf16 burst, maximum clocks") + f" ({pk_src})"
    # The attention time scaled to the maximum SM clock by the median clock sampled under load
    # (the kernel is compute bound, so its time scales with the clock): the burst fraction
    # that does not depend on where the clock sat during the timed region.
    clock_ratio = (clocks["sm_mhz"] / clocks["sm_max_mhz"]) if clocks.get("sm_mhz") and clocks.get("sm_max_mhz") else None
    attn_at_max = attn_avg * clock_ratio if clock_ratio else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w, args.mode, args.topk_frames, args.sasa_coef, args.sasa_trigger,
                                             args.frame_exact),
                   "l2": f"inputs larger than L2 (Q,K,V = {3 * q.numel() * q.element_size() / 1e9:.2f} GB per layer)",
                   "parallelism": f"independent layer per GPU x{world}",
                   **({"routing_refresh_every": args.refresh_every} if args.refresh_every > 1 else {}),
                   "tile_order": "ascending tile id" if args.plain_order else "longest first"},
        "route_ms": route_avg, "attn_ms": attn_avg, "attn_tflops": attn_tflops,
        "pct_bf16_peak": 100.0 * value / pk["bf16_tflops"],
        "pct_bf16_peak_attn": 100.0 * attn_tflops / pk["bf16_tflops"],
        "density": density, "selected_flops_per_layer": flops, "padded_tile_flops_per_layer": flops_padded,
        "tile_mma_flops_per_layer": mma_flops, "tile_utilisation": flops / mma_flops if mma_flops else None,
        "sm_busy_imbalance": sm_busy,
        "selected_kv_tokens_per_s": kv_tokens / (attn_avg * 1e-3),
        "query_tokens_per_s": BH * S / (ms_step * 1e-3),
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": attn_tflops, "peak": bf16_peak,
                     "unit": "TFLOP/s", "frac": attn_tflops / bf16_peak, "traffic": traffic,
                     "peak_kind": peak_kind,
                     "frac_of_burst": attn_tflops / pk["bf16_tflops"],
                     "frac_of_sustained": attn_tflops / pk["bf16_tflops_sustained"],
                     # the MMA work the 128-row tiles execute (both query blocks of a tile over
                     # the union of their key blocks), for context; `achieved` counts selected
                     # pairs only
                     "executed_tflops": mma_flops / (attn_avg * 1e-3) / 1e12,
                     "frac_executed": mma_flops / (attn_avg * 1e-3) / 1e12 / bf16_peak,
                     "frac_of_datasheet": attn_tflops / NOMINAL_BF16_TFLOPS,
                     "attn_ms_at_max_clock": attn_at_max,
                     "frac_of_burst_at_max_clock": (flops / (attn_at_max * 1e-3) / 1e12 / pk["bf16_tflops"])
                     if attn_at_max else None},
        "roofline_router": {"bound": "hbm", "achieved": router_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                            "frac": router_gbs / pk["hbm_gbs"], "algorithmic_bytes": rbytes,
                            "peak_kind": f"hbm copy ({pk_src})"},
        "e2e": e2e, "cpu_baseline": cpu,
        **({"graph_replay": graph} if graph is not None else {}),
        **({"rlb_emulated": rlb_em} if rlb_em is not None else {}),
        "gpu_launches": 5 * routed_steps + args.steps,   # router: 5 kernels, attention: 1
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="dit")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sm-busy", action="store_true", help="skip the stamped launches of the SM busy-time imbalance")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing of the step")
    ap.add_argument("--heads", type=int, default=0, help="override H (smaller profiling case)")
    ap.add_argument("--p", type=float, default=0.0, help="override the Top-p threshold")
    ap.add_argument("--mode", default="topp", choices=["topp", "frame_topk"])
    ap.add_argument("--topk-frames", type=int, default=4)
    ap.add_argument("--frame-exact", action="store_true", help="token-exact frame mode (with --mode frame_topk)")
    ap.add_argument("--sasa-coef", type=float, default=0.0, help="tile slack augmentation coefficient (0: off)")
    ap.add_argument("--sasa-trigger", type=int, default=1)
    ap.add_argument("--refresh-every", type=int, default=1,
                    help="recompute the routing every N steps and reuse it in between (1: every step)")
    ap.add_argument("--plain-order", action="store_true",
                    help="diagnostic: attention takes tiles in ascending id order instead of longest first")
    ap.add_argument("--emulate-ranks", type=int, default=0,
                    help="emulate runtime load balancing over this many ranks on one GPU (0: off)")
    ap.add_argument("--rlb-target", type=float, default=1.05)
    ap.add_argument("--rlb-budget", type=int, default=1, help="heads a rank may send")
    ap.add_argument("--sharded", action="store_true",
                    help="the sequence-parallel layer with head migration also on one process")
    ap.add_argument("--ulysses", action="store_true",
                    help="the sharded layer from sequence-sharded inputs, with the Ulysses all-to-alls")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1: an independent layer per rank (weak scaling) instead of the sharded layer")
    args = ap.parse_args()
    if args.refresh_every < 1:
        ap.error("--refresh-every must be >= 1")
    from workloads import get_workload
    w = get_workload(args.workload)
    if args.heads:
        w = w.replace(H=args.heads)
    if args.p:
        w = w.replace(p=args.p)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
