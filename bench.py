"""Benchmark of the expert-parallel dispatch path on B200.

One step = one pass of the whole path over one layer's synthetic batch:
  ep_route_stats -> ep_plan -> ep_layout -> ep_align_sort -> ep_dispatch
  -> ep_combine -> ep_replica_grad_reduce
(the expert GEMM between dispatch and combine is outside the path; combine
reads the dispatched rows).  Metric: routed (token, k) pairs per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (default): the moderate EP8 layer, R=8 simulated ranks x S=4096
tokens, E=64 experts, top-K=6, H=2048 bf16, block_m=64, replica gradients of
3*2048*1024 fp32 per expert; router logits N(0,1)+b_e with b_e ~ N(0,0.5^2).

`value`: device-resident inputs; the step is captured once as a CUDA graph and
replayed K times, with CUDA events around each replay on the launching stream,
L2 flushed (a 512 MB write) between replays outside the events, max over ranks.
The per-op breakdown and the roofline come from an eager pass of the same K
steps with CUDA events between the ops.  `e2e`: the same steps through the public API (EpLayer.run_host) from
pinned host buffers: routing, gate weights and hidden rows copied in, the
combined rows copied out, inside the timed region (run_host pipelines the
copies in token slices over two copy streams).  Under torchrun each rank
runs its own independent layer (weak scaling, no data-path collective).

--impl reference times the CPU oracle (the plain single-threaded definition of
the same path) on the host, on the same workload and metric.
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload number (1-5); 2 is the headline")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip timing the backward of dispatch and combine")
    ap.add_argument("--no-quota", action="store_true", help="skip timing the quota-driven planner")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager per-op pass only (default: the headline value comes from replaying the "
                         "step as one captured CUDA graph; the per-op breakdown from the eager pass)")
    ap.add_argument("--route", choices=["fused", "separate"], default="fused",
                    help="route phase as one cooperative launch (ep_route_fused) or the four separate calls")
    return ap.parse_args()


def workload_desc(c):
    g = f", replica grads {c['grad_n']} {c['grad_dtype']} per expert" if c["grad_n"] else ""
    lay = f", {c['layers']} layers per step" if c["layers"] > 1 else ""
    return (f"{c['name']}: R={c['R']} simulated EP ranks x S={c['S']} tokens, E={c['E']} experts, top-K={c['K']}, "
            f"H={c['H']} bf16, block_m={c['block_m']}, router bias {c['bias']}{g}{lay}")


def config_obj(c, l2):
    return {"workload": workload_desc(c), "layers": c["layers"], "R": c["R"], "S": c["S"], "E": c["E"], "K": c["K"], "H": c["H"],
            "tokens_per_step": c["T"], "pairs_per_step": c["P"], "block_m": c["block_m"], "l2": l2,
            "step": "route(" + "+".join(ROUTE_PARTS) + ")+dispatch+combine+grad_reduce"}


def algorithmic_bytes(c, n_rep, n_chunks):
    """Bytes each op must move (read + write) for one step."""
    T, P, E, H, K = c["T"], c["P"], c["E"], c["H"], c["K"]
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
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
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


def job_throughput(world, pairs_per_step, steps, job_ms):
    """Whole-job pairs/s: all ranks' pairs over the slowest rank's time."""
    return world * pairs_per_step * steps / (job_ms / 1e3)


# --------------------------------------------------------------- our arm

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def traffic_record(kernel):
    """ncu DRAM bytes per launch for `kernel`, if the committed capture was taken
    on the current source of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != rec["source_sha"]:
        return None
    return rec


def run_ours(args, rank, world, local_rank):
    import torch
    import token_dispatch_histogram_b200 as tdh
    import workload as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    c = W.shape(args.config)
    seed = rank_seed(args.seed, rank)
    R, S, E, K, H, T, P = c["R"], c["S"], c["E"], c["K"], c["H"], c["T"], c["P"]
    nl = c["layers"]
    gdt = torch.float32 if c["grad_dtype"] in ("f32", None) else torch.bfloat16
    layers = []
    for i in range(nl):  # consecutive layers share the large buffers
        layers.append(tdh.EpLayer(R, S, K, E, H, c["block_m"], device=dev, grad_n=c["grad_n"] or 0, grad_dtype=gdt,
                                  share=layers[0] if layers else None))
    layer = layers[0]

    # inputs: host-generated routing (per layer) and hidden rows (pinned when the
    # end-to-end pass runs), device-generated gradients
    routes = [W.routing(args.config, seed, i) for i in range(nl)]
    for ly, (tk, ww) in zip(layers, routes):
        ly.topk_ids.copy_(torch.from_numpy(tk))
        ly.w.copy_(torch.from_numpy(ww))
    host_x = T * H * 2 <= (4 << 30)
    if host_x:
        x_np = W.hidden(T, H, seed)
        layer.x.copy_(torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16))
    else:
        x_np = None
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
    for ly in layers:
        st = ly.status(stream)
        if st:
            raise RuntimeError(f"device status {st:#x} after warm-up")
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
    step_ms = []
    for lst in marks:
        for (op, e0), (_, e1) in zip(lst[:-1], lst[1:]):
            per_op[op] += e0.elapsed_time(e1)
        step_ms.append(lst[0][1].elapsed_time(lst[-1][1]))
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    for ly in layers:
        st = ly.status(stream)
        if st:
            raise RuntimeError(f"device status {st:#x} in the timed region")

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
            for ly in layers:
                st = ly.status(stream)
                if st:
                    raise RuntimeError(f"device status {st:#x} in the graph replays")
        except RuntimeError as exc:  # capture unsupported here: keep the eager timing
            graph = None
            print(f"graph capture unavailable: {exc}", file=sys.stderr)

    # ---- backward of combine and of dispatch (timed apart from the step)
    backward = None
    if not args.no_backward and 2 * P * H <= (20 << 30):
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

    def replay_ms(fn, flush_between):
        """Mean ms of fn captured as one CUDA graph and replayed args.steps
        times (L2 flushed before each replay when asked), max over ranks."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        g.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            if flush_between:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            g.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        del g
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, dev) / args.steps

    # ---- the quota-driven planner (a per-rank replica budget B) in place of
    # the exact-S*K plan: the same step (route, dispatch, combine, replica
    # gradients) and the route alone, each as one captured graph, replayed
    quota = {}
    if not args.no_graph and not args.no_quota:
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
                route_ms_q = replay_ms(lambda: q_routes(B), True)
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
            for ly in layers:
                st = ly.status(stream)
                if st:
                    raise RuntimeError(f"device status {st:#x} in the quota-planner timing")
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
    if not args.no_graph:
        def pdc():
            for ly in layers:
                tdh.ep_route_fused(ly.topk_ids, E, R, S, ly.loads, ly.max_vio, ly.plan, ly.pos, ly.src, ly.ws,
                                   ly.pair_slot, 0, None, None, None, ly.dev_status)
                tdh.ep_dispatch(ly.x, K, ly.pos, ly.buf, ly.dev_status)
                tdh.ep_combine(ly.buf, ly.w, ly.pos, ly.out, ly.dev_status)

        def align_only():
            for ly in layers:
                tdh.ep_align_sort(ly.topk_ids, E, ly.block_m, ly.sorted_token_ids, ly.expert_ids,
                                  ly.num_tokens_post_pad, ly.ws, ly.dev_status)

        def grads_only():
            for ly in layers:
                if ly.grad_n:
                    ly.grad_reduce(False)

        pdc_ms = replay_ms(pdc, True)
        as_named = {"value": job_throughput(world, nl * P, 1, pdc_ms), "unit": UNIT, "ms_per_step": round(pdc_ms, 5),
                    "what": "route without align-sort + dispatch + combine, one graph, L2 flushed",
                    "align_sort_us": round(replay_ms(align_only, True) * 1e3 / nl, 2)}
        if any(ly.grad_n for ly in layers):
            as_named["grad_reduce_us"] = round(replay_ms(grads_only, True) * 1e3 / nl, 2)
        for ly in layers:
            st = ly.status(stream)
            if st:
                raise RuntimeError(f"device status {st:#x} in the plan+dispatch+combine timing")

    # ---- fused layout + dispatch: the route (with align-sort) and dispatch in
    # one cooperative launch, against ep_route_fused followed by ep_dispatch
    route_dispatch = None
    if not args.no_graph:
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
                          "what": "route (stats, plan, layout, align-sort) + dispatch per layer: ep_route_dispatch_fused "
                                  "(one launch) against ep_route_fused then ep_dispatch; one graph each, L2 flushed"}
        for ly in layers:
            st = ly.status(stream)
            if st:
                raise RuntimeError(f"device status {st:#x} in the fused route + dispatch timing")

    # ---- the rank-local form emulated on this GPU: R rank buffers reached
    # through the peer table, each rank's dispatch and combine launched in
    # turn (one graph), against the one-buffer dispatch + combine above
    rank_local = None
    if not args.no_graph and nl == 1 and 2 * P * H <= (4 << 30):
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

        side = [torch.cuda.Stream(dev) for _ in rks]

        def rank_rows():  # the ranks run side by side, as on R GPUs; combine after every dispatch
            cur = torch.cuda.current_stream(dev)
            for phase in ("dispatch", "combine"):
                for rk, s2 in zip(rks, side):
                    s2.wait_stream(cur)
                    with torch.cuda.stream(s2):
                        getattr(rk, phase)(s2)
                for s2 in side:
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
        del rks, peers, side

    # ---- prefetch slots under a per-rank budget B (one small launch, timed
    # apart as device time: 20 launches in one captured graph, replayed):
    # replicas whose weights are read from the home rank, and the rank loads if
    # slotless replicas' pairs stayed home instead (B = 0: the unplanned loads)
    prefetch = {}
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
        us = None
        if not args.no_graph:
            try:
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
            except RuntimeError as exc:
                print(f"graph capture unavailable: {exc}", file=sys.stderr)
        prefetch[f"B={B}"] = {"us_per_launch": us,
                              "replicas_read_from_home": rem if nl > 1 else rem[0],
                              "max_rank_load_if_pairs_stay_home_over_SK": worst if nl > 1 else worst[0]}
    del pf_slot, pf_rem, pf_load

    # ---- end to end through the public API, pinned host buffers
    e2e = None
    if not args.no_e2e and host_x and nl == 1:
        topk_h = torch.from_numpy(routes[0][0]).pin_memory()
        w_h = torch.from_numpy(routes[0][1]).pin_memory()
        x_h = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
        out_h = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
        for _ in range(min(3, args.warmup)):
            layer.run_host(topk_h, w_h, x_h, out_h, stream, fused=fused)
        torch.cuda.synchronize()
        barrier()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            layer.run_host(topk_h, w_h, x_h, out_h, stream, fused=fused)
            ends[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), world, dev)
        bi = topk_h.numel() * 4 + w_h.numel() * 4 + x_h.numel() * 2
        bo = out_h.numel() * 2
        e2e = {"value": job_throughput(world, P, args.steps, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms / args.steps}

    # ---- roofline of the dominant kernel and the per-op breakdown (bytes summed over layers)
    abs_ = [algorithmic_bytes(c, nr, nc) for nr, nc in zip(n_rep, n_chunks)]
    ab = {op: sum(a[op] for a in abs_) for op in OPS}
    peak, peak_kind = peaks()
    calls = args.steps
    mean_ms = {op: per_op[op] / calls for op in OPS}  # per step (all layers)
    dom = max(("dispatch", "combine", "grad_reduce"), key=lambda op: mean_ms[op])
    kernel_of = {"dispatch": "k_dispatch", "combine": "k_combine", "grad_reduce": "k_grad_reduce"}
    achieved = ab[dom] / (mean_ms[dom] / 1e3) / 1e9 if mean_ms[dom] else 0.0
    tr = traffic_record(kernel_of[dom]) if args.config == 2 else None
    roofline = {"bound": "hbm", "kernel": kernel_of[dom], "achieved": round(achieved, 1), "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                "algorithmic_bytes_per_launch": ab[dom] // nl,
                "traffic": (tr["dram_bytes_per_launch"] if tr else None),
                "traffic_source": (tr["capture"] if tr else None)}
    breakdown = {op: {"ms": round(mean_ms[op], 5),
                      "GB_s": round(ab[op] / (mean_ms[op] / 1e3) / 1e9, 1) if mean_ms[op] else None}
                 for op in OPS}
    step_bytes = sum(ab.values())
    eager = {"value": job_throughput(world, nl * P, args.steps, total_ms), "ms_per_step": total_ms / args.steps,
             "gpu_launches": int(launches)}
    timed_ms = graph["ms"] if graph else total_ms
    value = job_throughput(world, nl * P, args.steps, timed_ms)
    d_c_ms = mean_ms["dispatch"] + mean_ms["combine"]
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": timed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Philox4x32-10 router logits with a per-workload expert bias, hidden rows ~ normal)",
        "config": config_obj(c, "flushed between steps (512 MB write, outside the step events)"),
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": graph["launches"] if graph else int(launches),
        "clocks": graph["clocks"] if graph else clk,
        "timing": ("one captured CUDA graph per step, replayed; CUDA events around each replay"
                   if graph else "eager launches; CUDA events around each step"),
        "step_ms_median": round(graph["step_ms_median"], 5) if graph else None,
        "step_ms_min": round(graph["step_ms_min"], 5) if graph else None,
        "eager": eager,
        "breakdown": breakdown,
        "step_hbm": {"bytes": step_bytes, "GB_s": round(step_bytes / (timed_ms / args.steps / 1e3) / 1e9, 1),
                     "frac": round(step_bytes / (timed_ms / args.steps / 1e3) / 1e9 / peak, 4)},
        "dispatch_combine": {"ms": round(d_c_ms, 5),
                             "GB_s": round((ab["dispatch"] + ab["combine"]) / (d_c_ms / 1e3) / 1e9, 1),
                             "frac": round((ab["dispatch"] + ab["combine"]) / (d_c_ms / 1e3) / 1e9 / peak, 4)},
        "routing": {"max_vio": max_vio if nl > 1 else max_vio[0], "n_rep": n_rep if nl > 1 else n_rep[0],
                    "replicated_experts": n_chunks if nl > 1 else n_chunks[0],
                    "top_expert_share": top_share if nl > 1 else top_share[0],
                    "max_replicas_per_rank": max_rep_rank if nl > 1 else max_rep_rank[0]},
        "backward": backward,
        "prefetch_slots": prefetch,
        "quota_planner": quota,
        "plan_dispatch_combine": as_named,
        "route_dispatch": route_dispatch,
        "rank_local": rank_local,
        "layers_per_step": nl,
        "route_path": args.route,
    }
    return res, (routes[0][0], routes[0][1], x_np, c, seed)


# ------------------------------------------------------------- CPU oracle

def oracle_step(c, topk, w, x, gh, gr, rep_expert_local):
    """One pass of the path through the CPU oracle (single thread)."""
    import oracle as O
    loads, mv, _ = O.route_stats(topk, c["E"])
    pl = O.plan(loads, c["R"], c["S"], c["K"], c["E"])
    lo = O.layout(topk, pl, c["R"], c["S"], c["E"])
    O.align_sort(topk, c["E"], c["block_m"])
    buf = O.dispatch(x, lo["pos"], c["K"], c["P"])
    O.combine(buf, w, lo["pos"], c["K"])
    if gh is not None:
        O.grad_reduce(gh, gr, rep_expert_local)
    return pl


def oracle_inputs(c, seed, topk):
    """Gradient rows the oracle's grad-reduce touches: the replicated experts'
    home rows and the replica rows, with the replica->expert map remapped to
    the compact home block (same adds, fewer untouched rows generated)."""
    import oracle as O
    import workload as W
    if not c["grad_n"]:
        return None, None, None
    loads, _, _ = O.route_stats(topk, c["E"])
    pl = O.plan(loads, c["R"], c["S"], c["K"], c["E"])
    experts = sorted(set(pl["rep_expert"].tolist()))
    idx = {e: i for i, e in enumerate(experts)}
    n = c["grad_n"]
    gh = W.grad_rows(seed, W.STREAM_GHOME, n, max(1, len(experts)))
    gr = W.grad_rows(seed, W.STREAM_GREP, n, max(1, pl["n_rep"]), c["grad_dtype"])
    local = np.array([idx[e] for e in pl["rep_expert"]], dtype=np.int32)
    return gh, gr, local


def time_oracle(c, seed, steps, topk=None, w=None, x=None, budget_s=None):
    import workload as W
    if topk is None:
        raise ValueError("routing required")
    if x is None:
        x = W.hidden(c["T"], c["H"], seed)
    gh, gr, local = oracle_inputs(c, seed, topk)
    times = []
    # one host core, as the oracle is single-threaded (restored afterwards)
    prev = os.sched_getaffinity(0) if hasattr(os, "sched_getaffinity") else None
    if prev:
        os.sched_setaffinity(0, {min(prev)})
    try:
        t_begin = time.perf_counter()
        for i in range(steps):
            t0 = time.perf_counter()
            oracle_step(c, topk, w, x, gh, gr, local)
            times.append(time.perf_counter() - t0)
            if budget_s is not None and time.perf_counter() - t_begin > budget_s:
                break
    finally:
        if prev:
            os.sched_setaffinity(0, prev)
    return times


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
    c = W.shape(args.config)
    topk, w = W.routing(args.config, args.seed)
    x = W.hidden(c["T"], c["H"], args.seed)
    time_oracle(c, args.seed, args.warmup, topk, w, x)
    times = time_oracle(c, args.seed, args.steps, topk, w, x)
    total = sum(times)
    value = c["P"] * len(times) / total
    sample = (f"the full step on the full workload, {len(times)} timed steps after {args.warmup} warm-up, "
              f"single thread, {cpu_model()}")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": len(times),
        "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Philox)",
        "config": config_obj(c, "n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res, (topk, w, x, c, seed) = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and x is not None and c["P"] * c["H"] <= (1 << 30):
        times = time_oracle(c, seed, 3, topk, w, x, budget_s=20.0)
        v = c["P"] * len(times) / sum(times)
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": f"{len(times)} full steps of the same workload and seed, single thread, "
                                         f"{cpu_model()} ({os.cpu_count()} cores on the host)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
