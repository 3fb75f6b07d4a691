"""Benchmark of the GSA layer (sparse global attention over N views) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload pages]
    python bench.py --impl reference ...      # the float64 CPU oracle, timed

A step is one whole GSA layer (pooling, compressed attention, S_guide top-K,
top-K merge, selected attention with the gate) over the workload's tokens, with
Q/K/V resident in HBM.  The metric is tokens per second of the layer (and ms
per layer); the dense global attention it replaces is timed in the same run.
Multi-GPU runs (torchrun, one rank per GPU) split one scene's heads over the
ranks (every head attends independently, so the layer has no exchange step):
strong scaling, the scene's tokens over the slowest rank's time.  With
``--parallel replicas`` every rank runs its own scene of the same size instead
(weak scaling, all ranks' tokens over the slowest rank's time).

Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import WORKLOADS, generate  # noqa: E402

METRIC = "global-attn layer ms & tokens/s at N views; % of bf16 tensor peak / HBM BW"
UNIT = "tokens/s"
SM_COUNT = 148
FFMA_PER_SM_PER_CLK = 128


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"],
                    bf16_tflops_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


# ---------------------------------------------------------------------------
# algorithmic work per step (counts only what the method computes)


def stage_work(z, H, D, K_eff) -> dict:
    """Per-stage algorithmic work of one layer: (bound, amount, unit)."""
    T, Tc, NB, NS, NK = z.T, z.Tc, z.NB, z.NS, z.NK
    return {
        # read Q, K, V once; write qc32, kc32 (fp32), vc, qc, kc (bf16) and the
        # head-major copies of the always-kept tokens' K, V (read again when they
        # are not the specials)
        "pool": ("hbm", 3 * T * H * D * 2 + Tc * H * D * (4 + 4 + 2 + 2 + 2) + 2 * NK * H * D * 2
                 + (2 * NK * H * D * 2 if NK != NS else 0), "bytes"),
        # QK^T and PV over the Tc x Tc pooled sequence
        "compressed_attn": ("tensor", 4 * Tc * Tc * H * D, "flop"),
        # K > 64: the second, ranking-only pass of the fused kernel: QK^T in tf32
        "block_scores": ("tensor", 2 * Tc * Tc * H * D, "flop"),
        # the ordering of the selection branch's pairs (each row's best block
        # read twice, the order written once), and for K > 64 the union of the
        # two selections (two lists read, one written)
        "topk_merge": ("hbm", H * Tc * 12 + (H * Tc * K_eff * 12 if K_eff > 64 else 0), "bytes"),
        # QK^T and PV of every token over the NK always-kept tokens
        "kept_attn": ("tensor", 4 * T * NK * H * D, "flop"),
        # the selected blocks' K and V gathered per (entry, head): K_eff blocks
        # of (on average) Hp*Wp/Bf valid tokens x 128 bytes, K and V; the bench
        # replaces this with the exact count of the run's own selection
        "selected_gate": ("gather", H * Tc * K_eff * (z.T - NS) // max(z.NB, 1) * D * 2 * 2, "bytes"),
    }


def selected_bytes(sel, z, shape) -> int:
    """K and V bytes of the valid tokens of every selected block, summed over
    all (head, entry) selections: what the selection branch must gather."""
    Bh = -(-shape.hp // shape.pool)
    Bw = -(-shape.wp // shape.pool)
    rows = torch.clamp(shape.hp - torch.arange(Bh) * shape.pool, max=shape.pool)
    cols = torch.clamp(shape.wp - torch.arange(Bw) * shape.pool, max=shape.pool)
    per_block = (rows[:, None] * cols[None, :]).reshape(-1).to(sel.device)  # valid tokens by position
    valid = sel >= 0
    tokens = torch.where(valid, per_block[torch.where(valid, sel, 0) % (Bh * Bw)], 0)
    return int(tokens.sum().item()) * shape.head_dim * 2 * 2


def dense_flops(z, H, D) -> int:
    return 4 * z.T * z.T * H * D


def frame_flops(z, H, D) -> int:
    # every token against the L tokens of its own frame: QK^T and PV
    return 4 * z.T * z.L * H * D


# ---------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            p = torch.cuda.get_device_properties(device)
            self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (cpu_baseline and --impl reference)


def sample_entries(geo, n_entries: int, seed: int) -> np.ndarray:
    """All fine tokens of ``n_entries`` seeded compressed entries (query blocks)."""
    rng = np.random.default_rng([seed, 5])
    ents = np.sort(rng.choice(geo.Tc, size=min(n_entries, geo.Tc), replace=False))
    return np.concatenate([geo.tokens_of_entry(int(a)) for a in ents])


def oracle_sample(x, n_entries: int, seed: int, pooled=None):
    """Time the oracle: one pooling pass (unless given), then the rest of the
    layer for every token of ``n_entries`` sampled query blocks.  Returns
    (pool_s, rest_s, res, rows, pooled); the full layer takes about
    pool_s + rest_s * Tc / n_entries."""
    from oracle import gsa_oracle as O
    geo = O.geometry_of(x.workload)
    t0 = time.perf_counter()
    if pooled is None:
        pooled = (O.pool(geo, x.q), O.pool(geo, x.k), O.pool(geo, x.v))
    t1 = time.perf_counter()
    rows = sample_entries(geo, n_entries, seed)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, pooled=pooled)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, res, rows, pooled


def cpu_threads() -> int:
    return torch.get_num_threads()


def run_reference(args) -> None:
    """The float64 CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    torch.set_num_threads(os.cpu_count() or 1)
    wl = chosen_workload(args)
    x = generate(wl)
    from oracle import gsa_oracle as O
    geo = O.geometry_of(wl)
    t0 = time.perf_counter()
    pooled = (O.pool(geo, x.q), O.pool(geo, x.k), O.pool(geo, x.v))
    t_pool = time.perf_counter() - t0
    n_ent = args.ref_entries
    times = []
    for i in range(args.warmup + args.steps):
        _, t_rest, _, _, _ = oracle_sample(x, n_ent, seed=100 + i, pooled=pooled)
        if i >= args.warmup:
            times.append(t_rest)
    t_rest = statistics.mean(times)
    layer_s = t_pool + t_rest * geo.Tc / n_ent
    value = geo.T / layer_s
    sample = (f"float64 oracle: one pooling pass over all {geo.T} tokens ({t_pool:.1f} s) plus, per step, "
              f"all tokens of {n_ent} seeded query blocks through compressed attention, top-K, selected "
              f"attention and the gate ({t_rest:.2f} s mean); full-layer time extrapolated as "
              f"pool + sample * Tc / {n_ent} = {layer_s:.0f} s")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, l2_note(wl, world, args.parallel), parallelism_of(wl, world, args.parallel)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def chosen_workload(args):
    wl = WORKLOADS[args.workload]
    if args.top_k is not None:
        wl = wl.with_(top_k=args.top_k)
    if args.keep:
        wl = wl.with_(keep=args.keep)
    return wl


def inputs_exceed_l2(in_bytes: int) -> bool:
    """Q/K/V of one rank large enough (4x the 126 MB L2) that no flush is needed."""
    return in_bytes > 4 * 126 * 2**20


def l2_note(wl, world: int = 1, parallel: str = "replicas") -> str:
    """How the timed region keeps one rank's inputs out of L2."""
    heads = wl.n_heads
    if world > 1 and parallel == "heads":
        heads = -(-wl.n_heads // world)  # the largest head slice
    in_bytes = 3 * wl.n_tokens * heads * wl.head_dim * 2
    if inputs_exceed_l2(in_bytes):
        return f"inputs larger than L2 ({in_bytes / 1e9:.1f} GB of Q/K/V)"
    return "L2 flushed between steps (256 MB write, outside the per-kernel events)"


def parallelism_of(wl, world: int, parallel: str) -> str:
    if world > 1 and parallel == "heads":
        return f"heads (one scene; {wl.n_heads} heads split over {world} ranks, no exchange in the layer)"
    return "replicas (independent scene per rank)"


def workload_config(wl, l2_note=None, parallelism="replicas (independent scene per rank)") -> dict:
    kept = ("frame 0 + every camera token always kept" if wl.keep == 1 else "every special token always kept")
    c = {"workload": f"{wl.name}: N={wl.n_frames} frames x ({wl.n_special} special + {wl.hp}x{wl.wp} patches) "
                     f"= {wl.n_tokens} tokens, {wl.n_heads} heads x {wl.head_dim}, pool {wl.pool}x{wl.pool}, "
                     f"top-K {wl.top_k}, {kept}, {wl.kind} generator seed {wl.seed}",
         "n_frames": wl.n_frames, "tokens": wl.n_tokens, "heads": wl.n_heads, "head_dim": wl.head_dim,
         "pool": wl.pool, "top_k": wl.top_k, "keep": "reference" if wl.keep == 1 else "specials",
         "parallelism": parallelism}
    if l2_note:
        c["l2"] = l2_note
    return c


# ---------------------------------------------------------------------------


def source_hash(path: str) -> str:
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def recorded_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        rec = json.load(open(path)).get(f"{kernel_file}@{workload}")
        src = os.path.join(ROOT, "sparse_global_attention_view_b200", "csrc", kernel_file)
        if rec and rec.get("source_sha") == source_hash(src):
            return rec["bytes_per_launch"]
    except Exception:
        pass
    return None


def rank_workload(wl, rank: int, parallel: str = "replicas"):
    """Replicas: rank r > 0 runs an independent scene of the same size (seed +
    1000 r).  Heads: every rank holds the same scene and takes its own heads."""
    if parallel == "heads":
        return wl
    return wl if rank == 0 else wl.with_(seed=wl.seed + 1000 * rank)


def head_slice(world: int, rank: int, n_heads: int) -> tuple[int, int]:
    """Contiguous heads [h0, h1) of rank r when the heads are split over the
    ranks as evenly as possible (every head attends independently, so the layer
    needs no exchange between ranks -- as after a column-parallel QKV
    projection)."""
    if world > n_heads:
        raise ValueError(f"{world} ranks for {n_heads} heads")
    base, extra = divmod(n_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def reduce_max(value: float, dist, device) -> float:
    """Max of ``value`` over all ranks (identity without a process group)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, tokens_per_rank: int, step_ms_max: float, parallel: str = "replicas") -> float:
    """Whole-job tokens/s over the slowest rank's step time: every rank's own
    scene (replicas), or the one scene all ranks share by heads."""
    tokens = tokens_per_rank if parallel == "heads" else world * tokens_per_rank
    return tokens / (step_ms_max / 1e3)


STAGE_SOURCE = {"pool": "pool.cu", "compressed_attn": "attn_cmp_tc.cu", "block_scores": "topk.cu",
                "topk_merge": "topk.cu", "kept_attn": "attn_tc.cu", "selected_gate": "selected_tc.cu"}


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["gsa", "reference"], default="gsa")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="pages")
    ap.add_argument("--top-k", type=int, default=None, help="override the workload's top-K (e.g. 128)")
    ap.add_argument("--keep", type=int, choices=[0, 1], default=0,
                    help="always-kept set: 0 every special token, 1 frame 0 + camera tokens")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense global attention baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle sample")
    ap.add_argument("--dense-steps", type=int, default=1)
    ap.add_argument("--no-frame", action="store_true", help="skip the frame attention leg")
    ap.add_argument("--frame-steps", type=int, default=5)
    ap.add_argument("--sga-windows", default="4,8",
                    help="AVGGT SGA legs: comma-separated window sizes s (s x s windows); empty for none")
    ap.add_argument("--sga-steps", type=int, default=2)
    ap.add_argument("--cpu-entries", type=int, default=48, help="query blocks in the cpu_baseline sample")
    ap.add_argument("--ref-entries", type=int, default=16, help="query blocks per reference-arm step")
    ap.add_argument("--parallel", choices=["replicas", "heads"], default="heads",
                    help="N > 1: one scene split by heads (strong scaling, the default) or independent "
                         "scenes per rank (weak scaling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "gsa":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
        return

    import sparse_global_attention_view_b200 as G

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dist, torch.device("cuda", local))

    mode = args.parallel if world > 1 else "replicas"
    wl = rank_workload(chosen_workload(args), rank, args.parallel)
    wl_scene = wl
    x = generate(wl)
    parallelism = parallelism_of(wl, world, mode)
    if mode == "heads":
        h0, h1 = head_slice(world, rank, wl.n_heads)
        x.q, x.k, x.v = (t[:, h0:h1].contiguous() for t in (x.q, x.k, x.v))
        x.w = x.w[h0:h1].contiguous()
        wl = wl.with_(n_heads=h1 - h0)
    shape = G.Shape.of(wl)
    z = G.derive(shape)
    H, D = shape.n_heads, shape.head_dim
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    q, k, v, w = (t.to(dev) for t in (x.q, x.k, x.v, x.w))
    out = torch.empty_like(q)
    layer = G.GsaLayer(shape, dev)
    big = inputs_exceed_l2(3 * q.numel() * 2)
    flush = None if big else torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    n_ev = len(G.FORWARD_STEPS) + 1

    def new_events(n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n)]
        for row in evs:
            for e in row:
                e.record(stream)  # create the handles
        return evs

    warm = new_events(1)[0]
    for _ in range(args.warmup):
        G.forward_timed(shape, q, k, v, w, out, layer.ws, warm, stream)
        if flush is not None:
            flush.fill_(1)
    torch.cuda.synchronize()
    G.check_device_error(layer.ws)

    evs = new_events(args.steps)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    launches = 0
    start.record(stream)
    for i in range(args.steps):
        launches += G.forward_timed(shape, q, k, v, w, out, layer.ws, evs[i], stream)
        if flush is not None:
            flush.fill_(1)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    G.check_device_error(layer.ws)

    per_step = [[evs[i][s].elapsed_time(evs[i][s + 1]) for s in range(n_ev - 1)] for i in range(args.steps)]
    stage_ms = {name: statistics.mean(r[s] for r in per_step) for s, name in enumerate(G.FORWARD_STEPS)}
    step_ms_local = (start.elapsed_time(stop) / args.steps) if flush is None else \
        statistics.mean(sum(r) for r in per_step)
    step_ms = max_over_ranks(step_ms_local)
    value = job_value(world, z.T, step_ms, mode)

    # ---- per-stage roofline from the same timed steps ----
    P = peaks()
    work = stage_work(z, H, D, min(shape.top_k, z.NB))
    gathered = selected_bytes(G.workspace_view(layer.ws, shape, "sel"), z, shape)
    alu_peak = SM_COUNT * FFMA_PER_SM_PER_CLK * 2 * P["sm_max_mhz"] * 1e6 / 1e12  # TFLOP/s fp32 FMA
    # the fused compressed stage does QK^T in tf32 (half the bf16 rate) and PV in
    # bf16, equal flops each: its tensor peak is 2/3 of the bf16 peak
    fused_cmp = True
    stages = {}
    for name in G.FORWARD_STEPS:
        bound, amount, unit = work[name]
        ms = stage_ms[name]
        if ms <= 0:
            continue
        if name == "selected_gate":
            amount = gathered
        if bound in ("hbm", "gather"):
            ach, peak, u = amount / (ms / 1e3) / 1e9, P["hbm_gbs"], "GB/s"
        elif bound == "tensor":
            ach, peak, u = amount / (ms / 1e3) / 1e12, P["bf16_tflops"], "TFLOP/s"
            if name == "compressed_attn" and fused_cmp:
                peak = P["bf16_tflops"] * 2.0 / 3.0
            if name == "block_scores":  # tf32 only: half the bf16 rate
                peak = P["bf16_tflops"] / 2.0
        else:
            ach, peak, u = amount / (ms / 1e3) / 1e12, alu_peak, "TFLOP/s"
        if ms < 0.005:
            continue  # fused into the previous step
        stages[name] = {"ms": round(ms, 4), "share": round(ms / sum(stage_ms.values()), 4), "bound": bound,
                        "achieved": round(ach, 2), "peak": round(peak, 1), "unit": u,
                        "frac": round(ach / peak, 4)}
        dram = recorded_traffic(STAGE_SOURCE[name], wl.name)
        if dram:
            # DRAM bytes of one launch (committed ncu counters of this source)
            # against the measured HBM copy bandwidth
            stages[name]["dram_bytes"] = dram
            stages[name]["dram_frac"] = round(dram / (ms / 1e3) / 1e9 / P["hbm_gbs"], 4)
        if name == "selected_gate":
            stages[name]["note"] = ("achieved = K/V bytes of the valid tokens of the selected blocks "
                                    f"({amount / 1e9:.1f} GB, counted from this run's selection) per second, "
                                    "moved L2 -> SM; peak = measured HBM copy bandwidth")
    dom = max(stages, key=lambda n: stages[n]["ms"])
    ds = stages[dom]
    traffic = recorded_traffic(STAGE_SOURCE[dom], wl.name)
    roofline = {"kernel": dom, "bound": ds["bound"], "achieved": ds["achieved"], "peak": ds["peak"],
                "unit": ds["unit"], "frac": ds["frac"], "traffic": traffic,
                "peak_source": (f"{P['source']} (MEASURED_PEAKS.json)" if ds["bound"] != "alu" else
                                f"fp32 FFMA: {SM_COUNT} SMs x {FFMA_PER_SM_PER_CLK} FMA/clk x 2 x "
                                f"{P['sm_max_mhz']:.0f} MHz")}

    # ---- end to end: pinned host buffers, copies inside the timed region ----
    # Every step copies its inputs from pinned host memory and its output back.
    # Two device buffer sets and two copy streams let step i+1's host-to-device
    # copy and step i-1's device-to-host copy run while step i computes (the
    # link is full duplex); the timed region spans the first copy in to the
    # last copy out.
    hq, hk, hv, hw = (t.pin_memory() for t in (x.q, x.k, x.v, x.w))
    houts = [torch.empty_like(x.q).pin_memory() for _ in range(2)]
    sets = [(q, k, v, w, out)] + [tuple(torch.empty_like(t) for t in (q, k, v, w, out))]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e_steps = max(2, args.steps)

    def e2e_run(n_steps):
        computed = [None, None]  # compute of the step that last used set b
        drained = [None, None]   # device-to-host copy of the step that last used set b
        last = None
        for i in range(n_steps):
            b = i % 2
            qb, kb, vb, wb, ob = sets[b]
            with torch.cuda.stream(s_in):
                if computed[b] is not None:
                    s_in.wait_event(computed[b])
                for dst, src in ((qb, hq), (kb, hk), (vb, hv), (wb, hw)):
                    dst.copy_(src, non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(s_in)
            stream.wait_event(loaded)
            if drained[b] is not None:
                stream.wait_event(drained[b])
            G.forward(shape, qb, kb, vb, wb, ob, layer.ws, stream)
            computed[b] = torch.cuda.Event()
            computed[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                houts[b].copy_(ob, non_blocking=True)
                drained[b] = torch.cuda.Event()
                drained[b].record(s_out)
            last = drained[b]
        for ev_ in drained:
            if ev_ is not None:
                stream.wait_event(ev_)
        return last

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    e2e_run(e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps)
    assert torch.equal(houts[(e_steps - 1) % 2], out.cpu()), "end-to-end output differs from the device run"
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hw))
    d2h = houts[0].numel() * houts[0].element_size()
    e2e = {"value": job_value(world, z.T, e2e_ms, mode), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3), "steps": e_steps,
           "path": ("pinned host Q/K/V/w -> device, gsa_forward, device -> pinned host out, every step; "
                    "two device buffer sets on separate copy streams so copies overlap the previous "
                    "and next steps' compute")}
    del sets[1:]

    # ---- the dense global attention baseline on the same inputs ----
    dense = None
    if not args.no_dense:
        dout = torch.empty_like(q)
        G.dense_global_attn(shape, q, k, v, dout, layer.ws, stream)
        torch.cuda.synchronize()
        barrier()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(args.dense_steps):
            G.dense_global_attn(shape, q, k, v, dout, layer.ws, stream)
        d1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(d0.elapsed_time(d1) / args.dense_steps)
        tf = dense_flops(z, H, D) / (dms / 1e3) / 1e12
        dense = {"ms_per_layer": round(dms, 3), "tokens_per_s": job_value(world, z.T, dms, mode),
                 "tflops": round(tf, 1), "frac_bf16_peak": round(tf / P["bf16_tflops"], 4),
                 "gsa_speedup": round(dms / step_ms, 2), "kernel": "tcgen05/TMEM + TMA flash attention",
                 "steps": args.dense_steps}
        del dout

    # ---- frame attention (attention within each frame) on the same inputs ----
    frame = None
    if not args.no_frame:
        fout = torch.empty_like(q)
        for _ in range(2):
            G.frame_attn(shape, q, k, v, fout, layer.ws, stream)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.frame_steps):
            G.frame_attn(shape, q, k, v, fout, layer.ws, stream)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        G.check_device_error(layer.ws)
        fms = max_over_ranks(f0.elapsed_time(f1) / args.frame_steps)
        tf = frame_flops(z, H, D) / (fms / 1e3) / 1e12
        frame = {"ms_per_layer": round(fms, 3), "tokens_per_s": job_value(world, z.T, fms, mode),
                 "tflops": round(tf, 1), "frac_bf16_peak": round(tf / P["bf16_tflops"], 4),
                 "kernel": "tcgen05/TMEM + TMA flash attention, one key segment per frame",
                 "steps": args.frame_steps}
        del fout

    # ---- AVGGT subsampled global attention on the same inputs ----
    sga = None
    windows = [int(w_) for w_ in args.sga_windows.split(",") if w_.strip()]
    if windows:
        sga = {}
        for sub in windows:
            ws_sga = G.new_sga_workspace(shape, sub, sub)
            sout = torch.empty_like(q)
            G.sga_attn(shape, sub, sub, q, k, v, sout, ws_sga, stream)
            torch.cuda.synchronize()
            barrier()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(args.sga_steps):
                G.sga_attn(shape, sub, sub, q, k, v, sout, ws_sga, stream)
            s1.record(stream)
            torch.cuda.synchronize()
            barrier()
            G.check_device_error(ws_sga)
            sms = max_over_ranks(s0.elapsed_time(s1) / args.sga_steps)
            nk = z.NS + wl.n_frames * (-(-wl.hp // sub)) * (-(-wl.wp // sub))
            tf = 4 * z.T * (nk + 2) * H * D / (sms / 1e3) / 1e12
            sga[f"{sub}x{sub}"] = {"ms_per_layer": round(sms, 3), "tokens_per_s": job_value(world, z.T, sms, mode),
                                   "kept_keys": nk, "tflops": round(tf, 1),
                                   "frac_bf16_peak": round(tf / P["bf16_tflops"], 4), "steps": args.sga_steps}
            del ws_sga, sout
        sga["kernels"] = ("gather of the kept keys, per-frame sums of the dropped ones, their means, "
                          "tcgen05/TMEM attention over the kept keys, log-sum-exp merge of the own key "
                          "and the mean pair")

    # ---- the CPU oracle on a bounded sample, and parity of the sampled rows ----
    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        torch.set_num_threads(os.cpu_count() or 1)
        sel_gpu = G.workspace_view(layer.ws, shape, "sel").permute(1, 0, 2).contiguous().cpu().numpy()
        out_host = out.cpu()
        t_pool, t_rest, res0, rows, pooled = oracle_sample(x, args.cpu_entries, seed=7)
        layer_s = t_pool + t_rest * z.Tc / args.cpu_entries
        cpu = {"value": z.T / layer_s, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": (f"one float64 pooling pass over all {z.T} tokens ({t_pool:.1f} s) + all tokens of "
                          f"{args.cpu_entries} seeded query blocks through the rest of the layer "
                          f"({t_rest:.1f} s); full-layer time extrapolated as pool + sample * Tc / "
                          f"{args.cpu_entries} = {layer_s:.0f} s")}
        from oracle import gsa_oracle as O
        geo = O.geometry_of(wl)
        res = O.gsa_layer(geo, x.q, x.k, x.v, x.w, rows=rows, sel_override=sel_gpu, pooled=pooled)
        a = out_host[torch.as_tensor(rows)].double().numpy()
        b = res["out"]
        d = np.abs(a - b)
        wide = res["gap"] >= 1e-3
        parity = {"rows": int(len(rows)), "max_abs": float(d.max()), "mean_abs": float(d.mean()),
                  "rel_l2": float(np.linalg.norm(a - b) / np.linalg.norm(b)),
                  "sel_valid_frac": float(res["sel_valid"].mean()),
                  "sel_exact_where_gap_ge_1e-3": float(res["sel_exact"][wide].mean()) if wide.any() else None,
                  "sel_exact_frac": float(res["sel_exact"].mean())}

    l2 = l2_note(wl_scene, world, mode)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "strong" if mode == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded scene model, random projections)",
        "config": workload_config(wl_scene, l2, parallelism), "roofline": roofline, "stages": stages, "cpu_baseline": cpu,
        "e2e": e2e, "gpu_launches": launches, "clocks": clk, "dense_baseline": dense, "frame_attention": frame, "sga": sga,
        "parity": parity,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
