"""Benchmark of the expert-parallel dispatch path on B200.

One step = one pass of the whole path over every layer of one synthetic batch:
  per layer: route (ep_route_stats -> ep_plan -> ep_layout -> ep_align_sort, as
  one cooperative launch) -> ep_dispatch -> ep_combine -> ep_replica_grad_reduce
(the expert GEMM between dispatch and combine is outside the path; combine
reads the dispatched rows).  Metric: routed (token, k) pairs per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (default, --config 4): the fine-grained layer sequence,
R=64 simulated EP ranks x S=8192 tokens, E=384 experts, top-K=8, H=7168 bf16,
block_m=128, router bias b_e ~ N(0,1) redrawn for each of 8 consecutive
layers; a step runs all 8 layers (4,194,304 pairs each), chained as in one
forward pass: layer l+1 dispatches the rows layer l combined (two row buffers
and a 60 GB dispatch buffer shared by the layers).  It is the largest
workload that fits one GPU.  After it, the same run times the other four
workloads (--others) with the same method and reports each under `workloads`.

`value`: device-resident inputs; the step is captured once as a CUDA graph and
replayed K times, with CUDA events around each replay on the launching stream,
L2 flushed (a 512 MB write) between replays outside the events, max over ranks.
The per-op breakdown and the roofline come from an eager pass of the same K
steps with CUDA events between the ops.  `e2e`: the same steps through the
public API (layer.run_host_batches) from pinned host buffers: every batch's
routing and gate weights for every layer and its hidden rows copied in, the
last layer's combined rows copied out, all inside one timed region, batch b+1's
inbound copies running while batch b's layers run and its outbound copies
drain (in token slices over two copy streams; the copies are torch's, around
the C-ABI kernels); `e2e.one_batch_at_a_time`: each batch alone
(layer.run_host_chain), timed step by step.  `e2e_rows_per_layer`: every layer's
hidden rows in and combined rows out (layer.run_host_layers).  Under torchrun
each rank runs its own independent layers (weak scaling, no data-path
collective); --rank-local times the rank-local form instead.

`cpu_baseline` and --impl reference time the CPU oracle (the plain
single-threaded definition of the same path) on one host core, on a bounded
sample of the same workload: the route over a whole layer, dispatch + combine
over a contiguous token slice, the replica gradient reduction over a column
slice; the value is the layer's pairs over the sum of the phases' per-unit
costs times the layer's units.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed (token,k) pairs/s for plan+dispatch+combine; achieved HBM GB/s vs peak"
UNIT = "pairs/s"
OPS = ["route", "dispatch", "combine", "grad_reduce"]
ROUTE_PARTS = ["route_stats", "plan", "layout", "align_sort"]
HEADLINE = 4
L2_NOTE = "flushed between steps (512 MB write, outside the step events)"
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (the measured copy bandwidth is the roofline's peak)


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=HEADLINE,
                    help="headline workload (1-5); 4, the fine-grained 8-layer sequence, is the largest")
    ap.add_argument("--others", default="1,2,3,5",
                    help="comma list of further workloads timed after the headline ('' for none)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens-per-rank", type=int, default=None,
                    help="override S (a smaller case of the same shape, e.g. for a profiler capture)")
    ap.add_argument("--layers", type=int, default=None, help="override the number of layers per step")
    ap.add_argument("--hidden", type=int, default=None,
                    help="override H (e.g. a full-size route with small rows, for a profiler capture of the route)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=12, help="token slices of the host-fed pipeline, one batch at a time")
    ap.add_argument("--e2e-batch-chunks", type=int, default=4,
                    help="token slices per batch with batches in flight (measured on B200: moderate EP8 3.03 ms per "
                         "batch with 2 slices, 3.05 with 4, 3.19 with 12; the fine-grained workload 200-201 ms for "
                         "4 to 24)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the backward of dispatch and combine")
    ap.add_argument("--no-quota", action="store_true", help="skip timing the quota-driven planner")
    ap.add_argument("--no-side", action="store_true",
                    help="skip every side measurement (backward, quota, plan+dispatch+combine, fused route+dispatch, "
                         "rank-local, prefetch slots)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager per-op pass only (default: the headline value comes from replaying the "
                         "step as one captured CUDA graph; the per-op breakdown from the eager pass)")
    ap.add_argument("--route", choices=["fused", "separate"], default="fused",
                    help="route phase as one cooperative launch (ep_route_fused) or the four separate calls")
    ap.add_argument("--rank-local", action="store_true",
                    help="time the rank-local form instead: the workload's R ranks spread over the N processes "
                         "(R/N per GPU), peer buffers mapped by CUDA IPC, counts all-gathered, rows written into "
                         "and read from the other processes' buffers")
    return ap.parse_args(argv)


def workload_shape(cfg, tokens_per_rank=None, layers=None, hidden=None):
    """The workload's shape dict, with the optional smaller-case overrides."""
    import workload as W
    c = dict(W.CONFIGS[cfg])
    if tokens_per_rank:
        c["S"] = int(tokens_per_rank)
    if layers:
        c["layers"] = int(layers)
    if hidden:
        c["H"] = int(hidden)
    c = W.shape(c)
    c["cfg"] = cfg
    return c


def workload_desc(c):
    g = f", replica grads {c['grad_n']} {c['grad_dtype']} per expert" if c["grad_n"] else ""
    lay = f", {c['layers']} layers per step" if c["layers"] > 1 else ""
    return (f"{c['name']}: R={c['R']} simulated EP ranks x S={c['S']} tokens, E={c['E']} experts, top-K={c['K']}, "
            f"H={c['H']} bf16, block_m={c['block_m']}, router bias {c['bias']}{g}{lay}")


def config_obj(c):
    """The workload as the JSON line's `config`: identical for both arms."""
    return {"workload": workload_desc(c), "layers": c["layers"], "R": c["R"], "S": c["S"], "E": c["E"], "K": c["K"],
            "H": c["H"], "tokens_per_layer": c["T"], "pairs_per_layer": c["P"], "pairs_per_step": c["P"] * c["layers"],
            "block_m": c["block_m"], "step": "per layer: route(" + "+".join(ROUTE_PARTS) + ")+dispatch+combine"
            + ("+grad_reduce" if c["grad_n"] else "")
            + ("; layer l+1 dispatches the rows layer l combined" if c["layers"] > 1 else "")}


def algorithmic_bytes(c, n_rep, n_chunks):
    """Bytes each op must move (read + write) for one layer."""
    T, P, E, H = c["T"], c["P"], c["E"], c["H"]
    bm = c["block_m"]
    n = c["grad_n"] or 0
    gb = 4 if c["grad_dtype"] == "f32" else 2
    parts = {
        "route_stats": 4 * P + 4 * E,
        "plan": 4 * E,
        "layout": 4 * P + 8 * P,                      # read ids, write pos + src
        "align_sort": 4 * P + 4 * P + 4 * (P + E * (bm - 1)),  # read ids twice, write padded ids
    }
    return {
        "route": sum(parts.values()),
        "dispatch": 2 * T * H + 2 * P * H + 4 * P,    # x once, every buffer row once, pos
        "combine": 2 * P * H + 8 * P + 2 * T * H,     # every buffer row, w + pos, out once
        "grad_reduce": n_chunks * 8 * n + n_rep * gb * n,
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return parse_clock_lines(self.lines)


def parse_clock_lines(lines):
    """Median SM clock, max clock and the throttle reasons seen, from
    nvidia-smi csv lines (noheader, nounits) of ClockSampler.FIELDS."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            mx = float(parts[1])
        except ValueError:
            continue
        for nm, v in zip(names, parts[4:8]):
            if v.lower() == "active":
                reasons.add(nm)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------ multi-rank host logic

def rank_seed(base, rank):
    """Every rank runs its own independent layer (weak scaling): its own seed."""
    return base + 1000 * rank


def max_over_ranks(value_ms, world, device):
    """Max of a per-rank device time over all ranks (the job's time)."""
    import torch
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_ok(ok, world, device):
    """True on every rank when every rank's `ok` is true (one max over ranks),
    so that all ranks take an optional pass together or none does."""
    return max_over_ranks(0.0 if ok else 1.0, world, device) == 0.0


def job_throughput(world, pairs_per_step, steps, job_ms):
    """Whole-job pairs/s: all ranks' pairs over the slowest rank's time."""
    return world * pairs_per_step * steps / (job_ms / 1e3)


def side_steps(steps, step_ms_est, budget_ms=2500.0):
    """Replays for a side measurement: all K steps while they take under
    `budget_ms`, else as many as fit (at least 3)."""
    if step_ms_est <= 0:
        return steps
    return int(max(3, min(steps, budget_ms // step_ms_est)))


# --------------------------------------------------------------- our arm

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def traffic_record(kernel, c):
    """ncu DRAM bytes per launch of `kernel` on workload `c`, if a committed
    capture covers that kernel at its current source on a case of the same
    shape: the capture's bytes scaled by (pairs per launch here) / (pairs per
    launch in the capture).  None when there is none or the source changed."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    recs = json.load(open(p))
    rec = recs.get(f"{kernel}@{c['name']}")
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != rec["source_sha"]:
        return None
    scale = c["P"] / rec["pairs_per_launch"]
    return {"dram_bytes_per_launch": int(round(rec["dram_bytes_per_launch"] * scale)),
            "capture": rec["capture"], "scaled_by": round(scale, 6)}


def run_workload(args, cfg, rank, world, local_rank, full=True):
    """Time one workload on this rank's GPU.  full=False: the step, its
    per-op breakdown, the roofline and the end-to-end pass only."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    import workload as W
    from token_dispatch_histogram_b200.layer import chain_buffers, run_host_batches, run_host_chain, run_host_layers

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    over = cfg == args.config
    c = workload_shape(cfg, args.tokens_per_rank if over else None, args.layers if over else None,
                       args.hidden if over else None)
    seed = rank_seed(args.seed, rank)
    R, S, E, K, H, T, P = c["R"], c["S"], c["E"], c["K"], c["H"], c["T"], c["P"]
    nl = c["layers"]
    gdt = torch.float32 if c["grad_dtype"] in ("f32", None) else torch.bfloat16
    layers = []
    for i in range(nl):  # consecutive layers share the large buffers
        layers.append(tdh.EpLayer(R, S, K, E, H, c["block_m"], device=dev, grad_n=c["grad_n"] or 0, grad_dtype=gdt,
                                  share=layers[0] if layers else None))
    # as in one forward pass, layer l+1 reads the rows layer l combined (two row buffers, nothing copied)
    chain_buffers(layers)
    layer = layers[0]

    # inputs: host-generated routing (per layer); hidden rows and gradients
    # from the device copy of the same counter-based generator
    routes = [W.routing(c, seed, i) for i in range(nl)]
    for ly, (tk, ww) in zip(layers, routes):
        ly.topk_ids.copy_(torch.from_numpy(tk))
        ly.w.copy_(torch.from_numpy(ww))
    W.fill_device(layer.x, seed, W.STREAM_X)
    if layer.grad_n:
        W.fill_device(layer.g_home, seed, W.STREAM_GHOME)
        W.fill_device(layer.g_rep, seed, W.STREAM_GREP)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 512 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def check(what):
        for ly in layers:
            st = ly.status(stream)
            if st:
                raise RuntimeError(f"device status {st:#x} {what}")

    fused = args.route == "fused"

    def step(rec=None, st=stream):
        # st=None: the binding uses torch's current stream (the capture stream
        # while a CUDA graph is being recorded)
        for ly in layers:
            if rec:
                rec("route")
            ly.route(st, fused=fused)
            if rec:
                rec("dispatch")
            tdh.ep_dispatch(ly.x, K, ly.pos, ly.buf, ly.dev_status, st)
            if rec:
                rec("combine")
            tdh.ep_combine(ly.buf, ly.w, ly.pos, ly.out, ly.dev_status, st)
            if ly.grad_n:
                if rec:
                    rec("grad_reduce")
                ly.grad_reduce(False, st)
        if rec:
            rec(None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check("after warm-up")
    n_rep = [int(ly.plan_view("n_rep", 1).item()) for ly in layers]
    n_chunks = [int(ly.plan_view("n_chunks", 1).item()) for ly in layers]
    max_vio = [float(ly.max_vio.item()) for ly in layers]
    top_share = [round(float(ly.loads.max().item()) / P, 5) for ly in layers]  # hottest expert's share of the pairs
    max_rep_rank = [int(ly.plan_view("rank_nrep", R).max().item()) for ly in layers]

    # ---- device-resident timed region: per-op CUDA events on the launching stream
    marks = []  # per step: list of (op, event)

    def recorder(lst):
        def rec(op):
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            lst.append((op, e))
        return rec

    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = tdh.ep_launch_count()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)  # outside the step's events
        lst = []
        step(recorder(lst))
        marks.append(lst)
    torch.cuda.synchronize()
    barrier()
    launches = tdh.ep_launch_count() - launches0
    clk = clocks.stop()
    per_op = {op: 0.0 for op in OPS}
    launches_per_op = {op: 0 for op in OPS}
    step_ms = []
    for lst in marks:
        for (op, e0), (_, e1) in zip(lst[:-1], lst[1:]):
            per_op[op] += e0.elapsed_time(e1)
            launches_per_op[op] += 1
        step_ms.append(lst[0][1].elapsed_time(lst[-1][1]))
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    check("in the timed region")
    est_ms = total_ms / args.steps  # one step, for sizing the side measurements
    nside = side_steps(args.steps, est_ms)

    # ---- the same step replayed as one captured CUDA graph: the headline timing
    graph = None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            torch.cuda.synchronize()
            c0 = tdh.ep_launch_count()
            with torch.cuda.graph(g):
                step(st=None)
            per_replay = tdh.ep_launch_count() - c0
            g.replay()
            torch.cuda.synchronize()
            gs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
            ge = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
            clocks_g = ClockSampler(local_rank)
            barrier()
            torch.cuda.synchronize()
            clocks_g.start()
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                gs[i].record(stream)
                g.replay()
                ge[i].record(stream)
            torch.cuda.synchronize()
            barrier()
            clk_g = clocks_g.stop()
            per_step = sorted(a.elapsed_time(b) for a, b in zip(gs, ge))
            g_ms = max_over_ranks(sum(per_step), world, dev)
            graph = {"ms": g_ms, "launches": int(per_replay * args.steps), "clocks": clk_g,
                     "step_ms_median": per_step[len(per_step) // 2], "step_ms_min": per_step[0]}
            del g
            check("in the graph replays")
        except RuntimeError as exc:  # capture unsupported here: keep the eager timing
            if "device status" in str(exc):
                raise
            graph = None
            print(f"graph capture unavailable: {exc}", file=sys.stderr)

    def replay_ms(fn, flush_between, n=None):
        """Mean ms of fn captured as one CUDA graph and replayed n (default:
        the side-measurement count) times (L2 flushed before each replay when
        asked), max over ranks."""
        n = n or nside
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            if flush_between:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        del g
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / n

    side = full and not args.no_side and not args.no_graph

    # ---- backward of combine and of dispatch (timed apart from the step)
    backward = None
    bwd_bytes = 2 * P * H + 2 * T * H + 4 * T * K  # dy, dx, dw
    if not args.no_graph and not args.no_backward and bwd_bytes + (2 << 30) <= torch.cuda.mem_get_info(dev)[0]:
        dy = torch.empty_like(layer.buf)
        dx = torch.empty_like(layer.x)
        dw = torch.empty((T, K), dtype=torch.float32, device=dev)
        ops_b = {
            "combine_backward": (lambda: tdh.ep_combine_backward(layer.out, layer.w, layer.buf, layer.pos, dy, dw,
                                                                 layer.dev_status, stream),
                                 2 * T * H + 2 * 2 * P * H + 12 * P + 4 * P),
            "dispatch_backward": (lambda: tdh.ep_dispatch_backward(layer.buf, layer.pos, T, K, dx, layer.dev_status,
                                                                   stream),
                                  2 * P * H + 4 * P + 2 * T * H),
        }
        backward = {}
        for name, (fn, nbytes) in ops_b.items():
            for _ in range(3):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                ev[i][0].record(stream)
                fn()
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / args.steps
            gbs = nbytes / (ms / 1e3) / 1e9
            backward[name] = {"ms": round(ms, 5), "GB_s": round(gbs, 1), "frac": round(gbs / peaks()[0], 4),
                              "algorithmic_bytes": nbytes}
        st = layer.status(stream)
        if st:
            raise RuntimeError(f"device status {st:#x} in the backward timing")
        del dy, dx, dw

    # ---- the quota-driven planner (a per-rank replica budget B) in place of
    # the exact-S*K plan: the same step (route, dispatch, combine, replica
    # gradients) and the route alone, each as one captured graph, replayed
    quota = {}
    if side and not args.no_quota:
        q_lay = tdh.ep_quota_plan_layout(E, R)
        q_plans = [torch.zeros(q_lay["words"], dtype=torch.int32, device=dev) for _ in layers]
        q_loads = torch.zeros(E, dtype=torch.int32, device=dev)
        q_pos = torch.zeros(P, dtype=torch.int32, device=dev)
        q_src = torch.zeros(P, dtype=torch.int32, device=dev)
        q_ws = torch.zeros(tdh.ep_quota_workspace_size(T, K, E, R), dtype=torch.uint8, device=dev)

        def q_route(B, li, ly):
            tdh.ep_quota_route(ly.topk_ids, E, R, S, B, q_loads, q_plans[li], q_pos, q_src, q_ws, ly.dev_status)

        def q_step(B):
            for li, ly in enumerate(layers):
                q_route(B, li, ly)
                tdh.ep_dispatch(ly.x, K, q_pos, ly.buf, ly.dev_status)
                tdh.ep_combine(ly.buf, ly.w, q_pos, ly.out, ly.dev_status)
                if ly.grad_n:
                    tdh.ep_quota_replica_grad_reduce(ly.g_home, ly.g_rep, E, R, q_plans[li], False, ly.dev_status)

        def q_routes(B):
            for li, ly in enumerate(layers):
                q_route(B, li, ly)

        try:
            for B in sorted({1, 3, E // R}):
                for _ in range(2):
                    q_step(B)
                torch.cuda.synchronize()
                step_ms_q = replay_ms(lambda: q_step(B), True)
                route_ms_q = replay_ms(lambda: q_routes(B), True, args.steps)
                taus, nreps, locs = [], [], []
                for li in range(nl):
                    pl = q_plans[li]
                    taus.append(round(int(pl[q_lay["tau"]].item()) * R / P, 4))
                    nreps.append(int(pl[q_lay["n_rep"]].item()))
                    locs.append(round(int(pl[q_lay["n_local"]].item()) / P, 4))
                one = nl == 1
                quota[f"B={B}"] = {
                    "ms_per_step": round(step_ms_q, 5),
                    "value": job_throughput(world, nl * P, 1, step_ms_q), "unit": UNIT,
                    "route_us": round(route_ms_q * 1e3 / nl, 2),
                    "max_rank_load_over_SK": taus[0] if one else taus,
                    "n_rep": nreps[0] if one else nreps,
                    "local_pair_fraction": locs[0] if one else locs}
            check("in the quota-planner timing")
        except RuntimeError as exc:
            if "device status" in str(exc):
                raise
            print(f"graph capture unavailable: {exc}", file=sys.stderr)
        del q_plans, q_pos, q_src, q_ws

    # ---- the metric exactly as named (plan + dispatch + combine): the route
    # without the align-sort walk, dispatch and combine, as one graph; and the
    # align-sort and the replica gradient reduction alone.  `value` above is
    # the whole step (all of them), so it is the lower of the two numbers.
    as_named = None
    route_alone = None
    if not args.no_graph:
        def pdc():
            for ly in layers:
                tdh.ep_route_fused(ly.topk_ids, E, R, S, ly.loads, ly.max_vio, ly.plan, ly.pos, ly.src, ly.ws,
                                   ly.pair_slot, 0, None, None, None, ly.dev_status)
                tdh.ep_dispatch(ly.x, K, ly.pos, ly.buf, ly.dev_status)
                tdh.ep_combine(ly.buf, ly.w, ly.pos, ly.out, ly.dev_status)

        def routes_only():
            for ly in layers:
                ly.route(fused=fused)

        def align_only():
            for ly in layers:
                tdh.ep_align_sort(ly.topk_ids, E, ly.block_m, ly.sorted_token_ids, ly.expert_ids,
                                  ly.num_tokens_post_pad, ly.ws, ly.dev_status)

        def grads_only():
            for ly in layers:
                if ly.grad_n:
                    ly.grad_reduce(False)

        # the route phase alone (a few MB of latency-bound passes), per layer,
        # as one graph, L2 flushed: the eager breakdown's route includes the
        # launch gaps between the eager kernels
        route_alone = round(replay_ms(routes_only, True, args.steps) * 1e3 / nl, 2)
        if side:
            pdc_ms = replay_ms(pdc, True)
            as_named = {"value": job_throughput(world, nl * P, 1, pdc_ms), "unit": UNIT,
                        "ms_per_step": round(pdc_ms, 5),
                        "what": "route without align-sort + dispatch + combine, one graph, L2 flushed",
                        "align_sort_us": round(replay_ms(align_only, True, args.steps) * 1e3 / nl, 2)}
            if any(ly.grad_n for ly in layers):
                as_named["grad_reduce_us"] = round(replay_ms(grads_only, True) * 1e3 / nl, 2)
        check("in the route and plan+dispatch+combine timing")

    # ---- fused layout + dispatch: the route (with align-sort) and dispatch in
    # one cooperative launch, against ep_route_fused followed by ep_dispatch
    route_dispatch = None
    if side:
        def rd_separate():
            for ly in layers:
                ly.route()
                tdh.ep_dispatch(ly.x, K, ly.pos, ly.buf, ly.dev_status)

        def rd_fused():
            for ly in layers:
                ly.route_dispatch()

        sep_ms = replay_ms(rd_separate, True)
        fus_ms = replay_ms(rd_fused, True)
        route_dispatch = {"fused_ms": round(fus_ms, 5), "separate_ms": round(sep_ms, 5),
                          "what": "route (stats, plan, layout, align-sort) + dispatch per step: "
                                  "ep_route_dispatch_fused (one launch per layer) against ep_route_fused then "
                                  "ep_dispatch; one graph each, L2 flushed"}
        check("in the fused route + dispatch timing")

    # ---- the rank-local form emulated on this GPU: R rank buffers reached
    # through the peer table, each rank's dispatch and combine launched in
    # turn (one graph), against the one-buffer dispatch + combine above
    rank_local = None
    if side and nl == 1 and 2 * P * H <= (4 << 30):
        from token_dispatch_histogram_b200.ranks import EpRank
        rks = [EpRank(r, R, S, K, E, H, device=dev) for r in range(R)]
        for r, rk in enumerate(rks):
            rk.topk_local.copy_(layer.topk_ids[r * S:(r + 1) * S])
            rk.w_local.copy_(layer.w[r * S:(r + 1) * S])
            rk.x_local.copy_(layer.x[r * S:(r + 1) * S])
            rk.count()
        counts = torch.stack([rk.counts_row for rk in rks])  # the all-gather, emulated
        peers = tdh.peer_table([rk.buf for rk in rks])
        for rk in rks:
            rk.counts.copy_(counts)
            rk.plan_and_layout()
            rk.set_peers(peers)

        side_streams = [torch.cuda.Stream(dev) for _ in rks]

        def rank_rows():  # the ranks run side by side, as on R GPUs; combine after every dispatch
            cur = torch.cuda.current_stream(dev)
            for phase in ("dispatch", "combine"):
                for rk, s2 in zip(rks, side_streams):
                    s2.wait_stream(cur)
                    with torch.cuda.stream(s2):
                        getattr(rk, phase)(s2)
                for s2 in side_streams:
                    cur.wait_stream(s2)

        def one_buffer_rows():
            for ly in layers:
                tdh.ep_dispatch(ly.x, K, ly.pos, ly.buf, ly.dev_status)
                tdh.ep_combine(ly.buf, ly.w, ly.pos, ly.out, ly.dev_status)

        rl_ms = replay_ms(rank_rows, True)
        ob_ms = replay_ms(one_buffer_rows, True)
        same = all(torch.equal(rk.out_local, layer.out[r * S:(r + 1) * S]) for r, rk in enumerate(rks))
        st = max(rk.status(stream) for rk in rks)
        if st or not same:
            raise RuntimeError(f"rank-local rows differ from the one-buffer rows (status {st:#x})")
        rank_local = {"dispatch_combine_ms": round(rl_ms, 5), "one_buffer_ms": round(ob_ms, 5),
                      "launches": 2 * R,
                      "what": "R ranks' dispatch_peer, then their combine_peer, each rank on its own stream, one graph, "
                              "L2 flushed"}
        del rks, peers, side_streams

    # ---- prefetch slots under a per-rank budget B (one small launch, timed
    # apart as device time: 20 launches in one captured graph, replayed):
    # replicas whose weights are read from the home rank, and the rank loads if
    # slotless replicas' pairs stayed home instead (B = 0: the unplanned loads)
    prefetch = {}
    if side:
        SK = S * K
        cap = layer.plan_layout["cap"]
        pf_slot = torch.empty(cap, dtype=torch.int32, device=dev)
        pf_rem = torch.empty(R, dtype=torch.int32, device=dev)
        pf_load = torch.empty(R, dtype=torch.int64, device=dev)
        for B in sorted({0, 3, 4, E // R}):
            rem, worst = [], []
            for ly in layers:
                tdh.ep_prefetch_slots(ly.plan, E, R, SK, B, pf_slot, pf_rem, pf_load, stream)
                torch.cuda.synchronize()
                rem.append(int(pf_rem.sum().item()))
                worst.append(round(int(pf_load.max().item()) / SK, 4))
            gp = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gp):
                for _ in range(20):
                    tdh.ep_prefetch_slots(layer.plan, E, R, SK, B, pf_slot, pf_rem, pf_load)
            gp.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                gp.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            us = round(e0.elapsed_time(e1) * 1e3 / (20 * args.steps), 2)
            del gp
            prefetch[f"B={B}"] = {"us_per_launch": us,
                                  "replicas_read_from_home": rem if nl > 1 else rem[0],
                                  "max_rank_load_if_pairs_stay_home_over_SK": worst if nl > 1 else worst[0]}
        del pf_slot, pf_rem, pf_load

    # ---- end to end through the public API, pinned host buffers: the batch's
    # hidden rows and every layer's routing in, the last layer's combined rows
    # out -- batches in flight (run_host_batches) and one batch at a time
    # (run_host_chain); and, for several layers, every layer's rows in and out
    # (run_host_layers)
    e2e = None
    e2e_rows = None
    pinned = None
    if not args.no_e2e:
        # every rank pins its own batch (15 GB on the fine-grained workload); the ranks take the end-to-end pass
        # together or not at all, so that none waits at a barrier for a rank that could not pin its buffers
        try:
            pinned = ([torch.from_numpy(tk).pin_memory() for tk, _ in routes],
                      [torch.from_numpy(ww).pin_memory() for _, ww in routes],
                      torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True),
                      torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True))
        except RuntimeError as exc:
            print(f"pinned host buffers for the end-to-end pass: {str(exc).splitlines()[0][:200]}", file=sys.stderr)
            pinned = None
        if not all_ranks_ok(pinned is not None, world, dev):
            pinned = None
            e2e = {"unavailable": "the pinned host buffers of the end-to-end pass could not be allocated on every rank"}
    if pinned is not None:
        topk_h, w_h, x_h, out_h = pinned
        del pinned
        W.fill_device(layer.x, seed, W.STREAM_X)
        x_h.copy_(layer.x)  # the generator's rows, as a caller's host batch
        route_bytes = sum(t.numel() * 4 for t in topk_h) + sum(t.numel() * 4 for t in w_h)

        def timed_host(host_step, budget_ms):
            host_step()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            host_step()
            torch.cuda.synchronize()
            first_ms = max_over_ranks((time.perf_counter() - t0) * 1e3, world, dev)  # every rank takes the same count
            n = side_steps(args.steps, first_ms, budget_ms)
            for _ in range(max(0, min(2, args.warmup) - 1)):
                host_step()
            torch.cuda.synchronize()
            barrier()
            starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            for i in range(n):
                flush.fill_(i & 0xFF)
                starts[i].record(stream)
                host_step()
                ends[i].record(stream)
            torch.cuda.synchronize()
            barrier()
            check("in the end-to-end pass")
            return max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), world, dev), n

        ms, n = timed_host(lambda: run_host_chain(layers, topk_h, w_h, x_h, out_h, stream, fused=fused,
                                                  chunks=args.e2e_chunks), 30000.0)
        alone = {"value": job_throughput(world, nl * P, n, ms), "unit": UNIT,
                 "h2d_bytes_per_step": route_bytes + x_h.numel() * 2, "d2h_bytes_per_step": out_h.numel() * 2,
                 "ms_per_step": ms / n, "steps": n, "chunks": args.e2e_chunks,
                 "what": "run_host_chain, one batch at a time (each timed alone, L2 flushed before it): every layer's "
                         "routing and weights and the batch's hidden rows in from pinned host memory, the layers in "
                         "sequence (each reads the rows the one before combined), the last layer's combined rows "
                         "out; torch copies around the C-ABI kernels, in token slices on two copy streams "
                         "overlapping the first and the last layer"}
        e2e = alone
        # the host link alone, for the same bytes: the batch's hidden rows in and the combined rows out as whole
        # copies, each direction alone and both at once (the floor any host-fed step on this machine has)
        h2d_s, d2h_s = layer._copy_streams()

        def link_ms(inbound, outbound, reps=3):
            best = None
            for _ in range(reps):
                torch.cuda.synchronize()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                h2d_s.wait_stream(stream)
                d2h_s.wait_stream(stream)
                if inbound:
                    with torch.cuda.stream(h2d_s):
                        layer.x.copy_(x_h, non_blocking=True)
                if outbound:
                    with torch.cuda.stream(d2h_s):
                        out_h.copy_(layer.out, non_blocking=True)
                stream.wait_stream(h2d_s)
                stream.wait_stream(d2h_s)
                b.record(stream)
                torch.cuda.synchronize()
                t = a.elapsed_time(b)
                best = t if best is None else min(best, t)
            return max_over_ranks(best, world, dev)

        host_link = {"rows_in_ms": round(link_ms(True, False), 4), "rows_out_ms": round(link_ms(False, True), 4),
                     "both_ms": round(link_ms(True, True), 4), "bytes_each_way": x_h.numel() * 2,
                     "what": "the batch's hidden rows copied in and the combined rows copied out as one whole copy "
                             "each (pinned host memory), each direction alone and both at once; best of 3"}
        alone["host_link"] = host_link
        # batches in flight: batch b+1's rows come in while batch b's layers run and its rows go out
        # (run_host_batches with stage buffers apart from the chain's row buffers)
        if 2 * x_h.numel() * 2 + (2 << 30) <= torch.cuda.mem_get_info(dev)[0]:
            x_stage = torch.empty_like(layer.x)
            out_stage = torch.empty_like(layer.x)
            nb = side_steps(args.steps, alone["ms_per_step"], 30000.0)

            def batches(k):
                run_host_batches(layers, [(topk_h, w_h, x_h, out_h)] * k, x_stage, out_stage, stream, fused=fused,
                                 chunks=args.e2e_batch_chunks)

            batches(2)
            torch.cuda.synchronize()
            barrier()
            flush.fill_(0)
            b0 = torch.cuda.Event(enable_timing=True)
            b1 = torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            batches(nb)
            b1.record(stream)
            torch.cuda.synchronize()
            barrier()
            check("in the batched end-to-end pass")
            ms_b = max_over_ranks(b0.elapsed_time(b1), world, dev)
            e2e = {"value": job_throughput(world, nl * P, nb, ms_b), "unit": UNIT,
                   "h2d_bytes_per_step": alone["h2d_bytes_per_step"], "d2h_bytes_per_step": alone["d2h_bytes_per_step"],
                   "ms_per_step": ms_b / nb, "steps": nb, "chunks": args.e2e_batch_chunks,
                   "what": f"run_host_batches: {nb} batches (steps) in one timed region, each batch's routing and "
                           "weights for every layer and its hidden rows in from pinned host memory and the last "
                           "layer's combined rows out, every copy inside the region; batch b+1's inbound copies "
                           "run while batch b's layers run and its outbound copies drain (stage buffers apart from "
                           "the chain's row buffers); torch copies around the C-ABI kernels, in token slices on "
                           "two copy streams; L2 flushed once before the region, not between the batches (each "
                           "batch's rows are larger than the L2 on every workload but the tiny one)",
                   "host_link": host_link, "one_batch_at_a_time": alone}
            del x_stage, out_stage
        if nl > 1:
            ms, n = timed_host(lambda: run_host_layers(layers, topk_h, w_h, [x_h] * nl, [out_h] * nl, stream,
                                                       fused=fused, chunks=args.e2e_chunks), 20000.0)
            e2e_rows = {"value": job_throughput(world, nl * P, n, ms), "unit": UNIT,
                        "h2d_bytes_per_step": route_bytes + nl * x_h.numel() * 2,
                        "d2h_bytes_per_step": nl * out_h.numel() * 2, "ms_per_step": ms / n, "steps": n,
                        "what": "run_host_layers: every layer's hidden rows in from and its combined rows out to "
                                "pinned host memory, the next layer's inbound copies overlapping this layer's "
                                "outbound ones"}
        del topk_h, w_h, x_h, out_h

    # ---- roofline of the dominant kernel and the per-op breakdown (bytes summed over layers)
    abs_ = [algorithmic_bytes(c, nr, nc) for nr, nc in zip(n_rep, n_chunks)]
    ab = {op: sum(a[op] for a in abs_) for op in OPS}
    peak, peak_kind = peaks()
    mean_ms = {op: per_op[op] / args.steps for op in OPS}  # per step (all layers)
    dom = max(("dispatch", "combine", "grad_reduce"), key=lambda op: mean_ms[op])
    # the library's combine for problems of 2^28 row elements and more (K <= 8) is its shared-memory ring kernel
    kernel_of = {"dispatch": "k_dispatch", "combine": "k_combine_ring" if T * H >= (1 << 28) and K <= 8 else "k_combine",
                 "grad_reduce": "k_grad_reduce"}
    achieved = ab[dom] / (mean_ms[dom] / 1e3) / 1e9 if mean_ms[dom] else 0.0
    tr = traffic_record(kernel_of[dom], c)
    roofline = {"bound": "hbm", "kernel": kernel_of[dom], "achieved": round(achieved, 1), "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4),
                "algorithmic_bytes_per_launch": ab[dom] // nl,
                "launch_ms": round(mean_ms[dom] / nl, 5),
                "traffic": (tr["dram_bytes_per_launch"] if tr else None),
                "traffic_source": (f"{tr['capture']}, scaled by {tr['scaled_by']} (pairs per launch)" if tr else None)}
    breakdown = {op: {"ms": round(mean_ms[op], 5),
                      "GB_s": round(ab[op] / (mean_ms[op] / 1e3) / 1e9, 1) if mean_ms[op] else None,
                      "launches_per_step": launches_per_op[op] // args.steps}
                 for op in OPS}
    step_bytes = sum(ab.values())
    eager = {"value": job_throughput(world, nl * P, args.steps, total_ms), "ms_per_step": total_ms / args.steps,
             "gpu_launches": int(launches)}
    timed_ms = graph["ms"] if graph else total_ms
    value = job_throughput(world, nl * P, args.steps, timed_ms)
    d_c_ms = mean_ms["dispatch"] + mean_ms["combine"]
    dc_gbs = (ab["dispatch"] + ab["combine"]) / (d_c_ms / 1e3) / 1e9
    one = nl == 1
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": timed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox4x32-10 router logits with a per-workload expert bias, hidden rows ~ normal)",
        "config": config_obj(c),
        "l2": L2_NOTE,
        "roofline": roofline,
        "e2e": e2e,
        "e2e_rows_per_layer": e2e_rows,
        "gpu_launches": graph["launches"] if graph else int(launches),
        "clocks": graph["clocks"] if graph else clk,
        "timing": ("one captured CUDA graph per step, replayed; CUDA events around each replay"
                   if graph else "eager launches; CUDA events around each step"),
        "step_ms_median": round(graph["step_ms_median"], 5) if graph else None,
        "step_ms_min": round(graph["step_ms_min"], 5) if graph else None,
        "eager": eager,
        "breakdown": breakdown,
        "route_us_per_layer": route_alone,
        "step_hbm": {"bytes": step_bytes, "GB_s": round(step_bytes / (timed_ms / args.steps / 1e3) / 1e9, 1),
                     "frac": round(step_bytes / (timed_ms / args.steps / 1e3) / 1e9 / peak, 4)},
        "dispatch_combine": {"ms": round(d_c_ms, 5), "GB_s": round(dc_gbs, 1), "frac": round(dc_gbs / peak, 4),
                             "frac_of_nominal_8TBs": round(dc_gbs / NOMINAL_HBM_GBS, 4),
                             "algorithmic_bytes": ab["dispatch"] + ab["combine"]},
        "routing": {"max_vio": max_vio[0] if one else max_vio, "n_rep": n_rep[0] if one else n_rep,
                    "replicated_experts": n_chunks[0] if one else n_chunks,
                    "top_expert_share": top_share[0] if one else top_share,
                    "max_replicas_per_rank": max_rep_rank[0] if one else max_rep_rank},
        "layers_per_step": nl,
        "route_path": args.route,
        "backward": backward,
    }
    if full:
        res.update({"prefetch_slots": prefetch, "quota_planner": quota,
                    "plan_dispatch_combine": as_named, "route_dispatch": route_dispatch, "rank_local": rank_local})
    del layers, layer, flush
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res, (c, seed, routes)


def run_rank_local(args, rank, world, local_rank):
    """The rank-local form of the headline workload over the job's processes:
    ranks [p*R/N, (p+1)*R/N) on process p's GPU (RankLocalJob).  A step, per
    layer: every local rank's counts, one all-gather of the count rows (NCCL),
    plan and layout per rank, dispatch into the ranks' buffers (peers through
    CUDA IPC mappings), a fence (stream synchronisation + barrier), combine
    from the peers; with gradients a second fence and the replica gradient
    reduction.  The R ranks and the tokens are the workload's whatever N is
    (strong scaling).  Timed with CUDA events around each step, max over
    ranks; the fences make each step's time include the host round trips."""
    import torch
    import torch.distributed as dist
    import workload as W
    from token_dispatch_histogram_b200.ranks import RankLocalJob

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    c = workload_shape(args.config, args.tokens_per_rank, args.layers, args.hidden)
    R, S, E, K, H, T, P = c["R"], c["S"], c["E"], c["K"], c["H"], c["T"], c["P"]
    nl = c["layers"]
    if R % world:
        raise SystemExit(f"--rank-local: R={R} ranks do not divide over {world} processes")
    gdt = torch.float32 if c["grad_dtype"] in ("f32", None) else torch.bfloat16
    group = None
    job = RankLocalJob(R, S, K, E, H, group=group, device=dev, grad_n=c["grad_n"] or 0, grad_dtype=gdt)
    # inputs: the same routing and hidden rows on every process (seed args.seed);
    # each process keeps its own ranks' slices, per layer
    routes = [W.routing(c, args.seed, i) for i in range(nl)]
    per_layer = []
    for tk, ww in routes:
        per_layer.append([(torch.from_numpy(tk[rk.rank * S:(rk.rank + 1) * S]).to(dev),
                           torch.from_numpy(ww[rk.rank * S:(rk.rank + 1) * S]).to(dev)) for rk in job.ranks])
    x_all = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    W.fill_device(x_all, args.seed, W.STREAM_X)
    for rk in job.ranks:
        rk.x_local.copy_(x_all[rk.rank * S:(rk.rank + 1) * S])
        if rk.grad_n:
            W.fill_device(rk.g_home, args.seed, W.STREAM_GHOME, rk.rank * (E // R) * rk.grad_n)
            W.fill_device(rk.g_rep, args.seed + 1 + rk.rank, W.STREAM_GREP)
    del x_all
    job.open_peers()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 512 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for li in range(nl):
            for rk, (tk, ww) in zip(job.ranks, per_layer[li]):
                rk.topk_local, rk.w_local = tk, ww
            job.route(stream)
            job.dispatch(stream)
            job.fence()
            job.combine(stream)
            if c["grad_n"]:
                job.fence()
                job.grad_reduce(False, stream)
            job.fence()

    for _ in range(args.warmup):
        step()
    st = job.status(stream)
    if st:
        raise RuntimeError(f"device status {st:#x} after warm-up")
    import token_dispatch_histogram_b200 as tdh
    clocks = ClockSampler(local_rank)
    job.fence()
    clocks.start()
    launches0 = tdh.ep_launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    job.fence()
    launches = tdh.ep_launch_count() - launches0
    clk = clocks.stop()
    st = job.status(stream)
    if st:
        raise RuntimeError(f"device status {st:#x} in the timed region")
    job_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev)
    value = nl * P * args.steps / (job_ms / 1e3)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": job_ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox4x32-10 router logits with a per-workload expert bias, hidden rows ~ normal)",
        "config": config_obj(c), "l2": L2_NOTE,
        "form": f"rank-local: {R} ranks over {world} processes, {R // world} per GPU, "
                + ("other processes' buffers mapped by CUDA IPC" if world > 1 else "every peer buffer local"),
        "e2e": None, "gpu_launches": int(launches), "clocks": clk,
        "timing": "CUDA events around each eager step (host fences inside), max over ranks",
    }
    job.close()
    del flush
    return res


def workload_summary(res):
    """The keys of a non-headline workload's result kept in the JSON line."""
    keep = ("value", "unit", "ms_per_step", "step_ms_median", "step_ms_min", "steps", "dispatch_combine", "step_hbm",
            "roofline", "breakdown", "route_us_per_layer", "routing", "e2e", "clocks", "gpu_launches",
            "layers_per_step", "backward")
    out = {k: res[k] for k in keep if k in res}
    out["workload"] = res["config"]["workload"]
    return out


# ------------------------------------------------------------- CPU oracle

def sample_tokens(c):
    """Tokens per oracle sample of dispatch + combine (about 2^28 row
    elements, or the whole layer when smaller)."""
    return int(min(c["T"], max(1, (1 << 28) // (c["K"] * c["H"]))))


def sample_cols(c):
    """Gradient columns per oracle sample of the replica gradient reduction."""
    return int(min(c["grad_n"] or 0, 1 << 22))


def oracle_sample(c, seed, topk, w, t0):
    """One bounded sample of one layer through the CPU oracle (single thread):

      route   -- loads + max_vio, plan, layout, align-sort over the whole layer;
      rows    -- dispatch and combine of the tokens [t0, t0 + Ts), into a buffer
                 holding only their rows (in the layout's row order);
      grads   -- the replica gradient reduction over the first Nc columns of
                 the replicated experts' home rows and of the replica rows.

    Returns (t_route, t_rows, t_grad) in seconds and the sample sizes; the
    inputs of the rows and gradients are generated outside the timed parts."""
    import oracle as O
    import workload as W
    E, R, S, K, H, T = c["E"], c["R"], c["S"], c["K"], c["H"], c["T"]
    Ts = sample_tokens(c)
    t0 = int(t0) % max(1, T - Ts + 1)
    a = time.perf_counter()
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    O.align_sort(topk, E, c["block_m"])
    t_route = time.perf_counter() - a
    pos = lo["pos"][t0 * K:(t0 + Ts) * K]
    local = np.empty_like(pos)
    local[np.argsort(pos, kind="stable")] = np.arange(pos.size, dtype=np.int32)
    x = W.hidden(Ts, H, seed, 0, t0)
    ws = np.ascontiguousarray(w[t0:t0 + Ts])
    a = time.perf_counter()
    buf = O.dispatch(x, local, K, Ts * K)
    O.combine(buf, ws, local, K)
    t_rows = time.perf_counter() - a
    t_grad, nc = 0.0, 0
    if c["grad_n"]:
        nc = sample_cols(c)
        experts = sorted(set(pl["rep_expert"].tolist()))
        idx = {e: i for i, e in enumerate(experts)}
        gh = np.stack([W.normal_f32(seed, W.STREAM_GHOME, e * c["grad_n"], nc) for e in experts]) if experts else \
            np.zeros((1, nc), np.float32)
        if c["grad_dtype"] == "f32":
            gr = np.stack([W.normal_f32(seed, W.STREAM_GREP, m * c["grad_n"], nc) for m in range(pl["n_rep"])])
        else:
            gr = np.stack([W.normal_bf16(seed, W.STREAM_GREP, m * c["grad_n"], nc) for m in range(pl["n_rep"])])
        rep_local = np.array([idx[e] for e in pl["rep_expert"]], dtype=np.int32)
        a = time.perf_counter()
        O.grad_reduce(gh, gr, rep_local)
        t_grad = time.perf_counter() - a
    return t_route, t_rows, t_grad, Ts, nc


def layer_seconds(c, t_route, t_rows, t_grad, Ts, nc):
    """The oracle's time for a whole layer from one sample: each phase's
    per-unit cost times the layer's units (pairs for the route, which ran in
    full; tokens for the rows; gradient columns for the reduction)."""
    s = t_route + t_rows * (c["T"] / Ts)
    if nc:
        s += t_grad * (c["grad_n"] / nc)
    return s


def time_oracle(c, seed, routes, samples, budget_s=None):
    """`samples` oracle samples on one host core (layer i mod layers, token
    slices spread over the layer); returns (per-sample seconds actually
    spent, per-sample extrapolated layer seconds)."""
    spent, layer_s = [], []
    prev = os.sched_getaffinity(0) if hasattr(os, "sched_getaffinity") else None
    if prev:
        os.sched_setaffinity(0, {min(prev)})
    try:
        t_begin = time.perf_counter()
        for i in range(samples):
            topk, w = routes[i % len(routes)]
            t0 = (i * 7919 * sample_tokens(c)) % c["T"]
            tr, tw, tg, Ts, nc = oracle_sample(c, seed, topk, w, t0)
            spent.append(tr + tw + tg)
            layer_s.append(layer_seconds(c, tr, tw, tg, Ts, nc))
            if budget_s is not None and time.perf_counter() - t_begin > budget_s:
                break
    finally:
        if prev:
            os.sched_setaffinity(0, prev)
    return spent, layer_s


def sample_desc(c, n):
    Ts, nc = sample_tokens(c), sample_cols(c)
    rows = "every token" if Ts == c["T"] else f"a contiguous slice of {Ts} of its {c['T']} tokens"
    g = (f", and the replica gradient reduction over {'all' if nc == c['grad_n'] else nc} of its {c['grad_n']} "
         f"gradient columns") if c["grad_n"] else ""
    return (f"{n} samples, one layer each (layer i mod {c['layers']}): the route (stats, plan, layout, align-sort) over "
            f"the whole layer ({c['P']} pairs), dispatch + combine over {rows}{g}; value = the layer's pairs over the "
            f"sum of each phase's time per unit times the layer's units. Single thread, {cpu_model()} "
            f"({os.cpu_count()} cores on the host)")


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    import workload as W
    c = workload_shape(args.config, args.tokens_per_rank, args.layers, args.hidden)
    nl = c["layers"]
    routes = [W.routing(c, args.seed, i) for i in range(nl)]
    time_oracle(c, args.seed, routes, args.warmup)
    spent, layer_s = time_oracle(c, args.seed, routes, args.steps)
    value = c["P"] * len(layer_s) / sum(layer_s)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": len(spent),
        "warmup": args.warmup, "ms_per_step": sum(spent) / len(spent) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Philox4x32-10 router logits with a per-workload expert bias, hidden rows ~ normal)",
        "config": config_obj(c),
        "l2": "n/a (CPU)",
        "step_what": "each step is one bounded oracle sample (see cpu_baseline.sample); ms_per_step is the time "
                     "actually spent per sample, extrapolated_layer_ms the oracle's time for a whole layer",
        "extrapolated_layer_ms": sum(layer_s) / len(layer_s) * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample_desc(c, len(spent))},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    if args.rank_local:
        res = run_rank_local(args, rank, world, local_rank)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(res))
        return
    res, (c, seed, routes) = run_workload(args, args.config, rank, world, local_rank, full=True)
    others = [int(s) for s in args.others.split(",") if s.strip()]
    workloads = {}
    for cfg in others:
        if cfg == args.config:
            continue
        r2, _ = run_workload(args, cfg, rank, world, local_rank, full=False)
        workloads[str(cfg)] = workload_summary(r2)
    if workloads:
        res["workloads"] = workloads
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        spent, layer_s = time_oracle(c, seed, routes, max(1, c["layers"]), budget_s=20.0)
        v = c["P"] * len(layer_s) / sum(layer_s)
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": sample_desc(c, len(spent)), "seconds": round(sum(spent), 2)}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
