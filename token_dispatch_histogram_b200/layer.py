"""EpLayer: one expert-parallel MoE layer's dispatch path on static buffers.

Allocates every buffer once at its static capacity (the S*K-per-rank contract
makes all shapes known in advance: [GR] "Online planning, zero copy και
στατικά σχήματα", twodots.gr MoonEP article) and runs the path as a fixed
sequence of libep.so calls on one stream, with no host synchronisation:

  ep_route_fused (= ep_route_stats -> ep_plan -> ep_layout -> ep_align_sort)
  -> ep_dispatch -> [expert: outside the path] -> ep_combine -> ep_replica_grad_reduce

`step()` is one pass of that sequence over the resident inputs; `run_host()`
is the same pass fed from pinned host buffers (copies in, result out),
pipelined in token slices so the host transfers overlap.
Plumbing only: every computation happens in the library's kernels.
"""
import torch

from . import (align_sort_capacity, ep_align_sort, ep_combine, ep_dispatch, ep_expert_scale, ep_layout,
               ep_plan, ep_plan_layout, ep_replica_grad_reduce, ep_route_dispatch_fused, ep_route_fused, ep_route_stats,
               ep_status_read,
               ep_workspace_size)


def slice_bounds(T, chunks):
    """Token boundaries of the host-fed pipeline's `chunks` slices.  From five
    slices on, the first and last two are smaller (weights 1, 2, 4, ..., 4, 2,
    1), so the first rows reach the kernels sooner and the last rows leave
    sooner; measured on B200 for the moderate EP8 workload: 3.27 ms per step
    against 3.33 ms with equal slices.  Slices may be empty for tiny T."""
    if chunks < 5:
        wts = [1] * chunks
    else:
        wts = [1, 2] + [4] * (chunks - 4) + [2, 1]
    tot = sum(wts)
    b, acc = [0], 0
    for wt in wts:
        acc += wt
        b.append(T * acc // tot)
    return b


class EpLayer:
    def __init__(self, R, S, K, E, H, block_m, device="cuda", grad_n=0, grad_dtype=torch.float32,
                 with_pair_slot=False, share=None):
        """share: another EpLayer of the same shape whose row buffers (x, the
        dispatch buffer, out), workspace and gradients this layer reuses --
        consecutive layers of a model run one after another, so one set of the
        large buffers serves them all."""
        self.R, self.S, self.K, self.E, self.H, self.block_m = R, S, K, E, H, block_m
        self.T = R * S
        self.P = self.T * K
        self.device = torch.device(device)
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_ids = torch.zeros((self.T, K), **i32)
        self.w = torch.zeros((self.T, K), dtype=torch.float32, device=dev)
        self.x = share.x if share is not None else torch.zeros((self.T, H), dtype=torch.bfloat16, device=dev)
        self.loads = torch.zeros(E, **i32)
        self.max_vio = torch.zeros(1, dtype=torch.float64, device=dev)
        self.ws = share.ws if share is not None else torch.zeros(ep_workspace_size(self.T, K, E), dtype=torch.uint8,
                                                                 device=dev)
        self.plan_layout = ep_plan_layout(E, R)
        self.plan = torch.zeros(self.plan_layout["words"], **i32)
        self.pos = torch.zeros(self.P, **i32)
        self.src = torch.zeros(self.P, **i32)
        self.pair_slot = torch.zeros(self.P, **i32) if with_pair_slot else None
        if share is not None:
            self.buf, self.out = share.buf, share.out
        else:
            self.buf = torch.zeros((self.P, H), dtype=torch.bfloat16, device=dev)  # dispatch output / combine input
            self.out = torch.zeros((self.T, H), dtype=torch.bfloat16, device=dev)
        cap, capb = align_sort_capacity(self.P, E, block_m)
        self.sorted_token_ids = torch.zeros(cap, **i32)
        self.expert_ids = torch.zeros(capb, **i32)
        self.num_tokens_post_pad = torch.zeros(1, **i32)
        self.dev_status = torch.zeros(1, **i32)
        self.grad_n = grad_n
        if grad_n and share is not None and share.grad_n == grad_n:
            self.g_home, self.g_rep = share.g_home, share.g_rep
        elif grad_n:
            self.g_home = torch.zeros((E, grad_n), dtype=torch.float32, device=dev)
            self.g_rep = torch.zeros((self.plan_layout["cap"], grad_n), dtype=grad_dtype, device=dev)
        else:
            self.g_home = self.g_rep = None

    # --- the path ---------------------------------------------------------
    def route(self, stream=None, fused=True):
        """a1-a4: loads/max_vio, plan, layout, align-sort (one cooperative
        launch when fused, else the four separate entry points)."""
        if fused:
            ep_route_fused(self.topk_ids, self.E, self.R, self.S, self.loads, self.max_vio, self.plan, self.pos,
                           self.src, self.ws, self.pair_slot, self.block_m, self.sorted_token_ids, self.expert_ids,
                           self.num_tokens_post_pad, self.dev_status, stream)
            return
        ep_route_stats(self.topk_ids, self.E, self.loads, self.max_vio, self.ws, self.dev_status, stream)
        ep_plan(self.loads, self.R, self.S, self.K, self.E, self.plan, self.dev_status, stream)
        ep_layout(self.topk_ids, self.E, self.R, self.S, self.plan, self.ws, self.pos, self.src, self.pair_slot,
                  self.dev_status, stream)
        ep_align_sort(self.topk_ids, self.E, self.block_m, self.sorted_token_ids, self.expert_ids,
                      self.num_tokens_post_pad, self.ws, self.dev_status, stream)

    def route_dispatch(self, stream=None):
        """route() and dispatch() in one cooperative launch: each tile's rows
        are copied as soon as the tile is placed (same outputs)."""
        ep_route_dispatch_fused(self.topk_ids, self.E, self.R, self.S, self.loads, self.max_vio, self.plan, self.pos,
                                self.src, self.ws, self.x, self.buf, self.pair_slot, self.block_m,
                                self.sorted_token_ids, self.expert_ids, self.num_tokens_post_pad, self.dev_status,
                                stream)

    def dispatch(self, stream=None):
        ep_dispatch(self.x, self.K, self.pos, self.buf, self.dev_status, stream)

    def expert_standin(self, scale, stream=None):
        """y = bf16(buf * s_e) in place (stands in for the grouped GEMM)."""
        ep_expert_scale(self.buf, self.src, self.topk_ids, scale, self.buf, self.dev_status, stream)

    def combine(self, stream=None):
        ep_combine(self.buf, self.w, self.pos, self.out, self.dev_status, stream)

    def grad_reduce(self, clear=False, stream=None):
        if self.grad_n:
            ep_replica_grad_reduce(self.g_home, self.g_rep, self.E, self.R, self.plan, clear, self.dev_status, stream)

    def step(self, stream=None, grads=True, fused=True, overlap=False):
        """One pass of the whole path over the resident inputs.  overlap=True
        runs the replica gradient reduction on a second stream beside combine
        (they share no data: the reduction needs only the plan); the caller's
        stream waits for both.  Measured on B200: 415.8 against 421.9 us per
        graph-replayed step on the moderate EP8 workload."""
        self.route(stream, fused)
        self.dispatch(stream)
        if not (overlap and grads and self.grad_n):
            self.combine(stream)
            if grads:
                self.grad_reduce(False, stream)
            return
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        if not hasattr(self, "_side"):
            self._side = torch.cuda.Stream(self.device)
        side = self._side
        side.wait_stream(main)
        self.grad_reduce(False, side)
        self.combine(main)
        main.wait_stream(side)

    def run_host(self, topk_h, w_h, x_h, out_h, stream=None, grads=True, fused=True, chunks=8):
        """The step fed from pinned host buffers: host->device copies of the
        routing and hidden rows, the path, and the combined rows back to host.

        With chunks > 1 the token rows move in `chunks` slices on two copy
        streams: slice i is copied in, dispatched and combined while slice i+1
        is still arriving and slice i-1 is already going out (the host link is
        full duplex), so the transfers overlap each other and the kernels.
        Dispatch and combine of a token slice touch only that slice's pairs, so
        the slices are independent.  The routing and gate weights go first on
        the same copy stream as the token slices, ahead of them, so the route
        never waits behind the hidden rows (copied on the compute stream
        instead, they did so in every other step on B200, which then ran the
        two copy directions one after the other: 4.97 against 3.32 ms for the
        moderate EP8 workload).  The caller's stream waits for the last copy
        out before anything queued after this call."""
        main = stream if stream is not None else torch.cuda.current_stream(self.device)
        if chunks <= 1 or self.T < chunks:
            with torch.cuda.stream(main):
                self.topk_ids.copy_(topk_h, non_blocking=True)
                self.w.copy_(w_h, non_blocking=True)
                self.x.copy_(x_h, non_blocking=True)
                self.step(main, grads, fused)
                out_h.copy_(self.out, non_blocking=True)
            return
        h2d, d2h = self._copy_streams()
        h2d.wait_stream(main)  # buffers are free once the caller's earlier work is done
        d2h.wait_stream(main)
        with torch.cuda.stream(h2d):
            self.topk_ids.copy_(topk_h, non_blocking=True)
            self.w.copy_(w_h, non_blocking=True)
            routed = torch.cuda.Event()
            routed.record(h2d)
        main.wait_event(routed)
        self.route(main, fused)
        bounds = slice_bounds(self.T, chunks)
        K = self.K
        for t0, t1 in zip(bounds[:-1], bounds[1:]):
            with torch.cuda.stream(h2d):
                self.x[t0:t1].copy_(x_h[t0:t1], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(h2d)
            main.wait_event(arrived)
            ep_dispatch(self.x[t0:t1], K, self.pos[t0 * K:t1 * K], self.buf, self.dev_status, main)
            ep_combine(self.buf, self.w[t0:t1], self.pos[t0 * K:t1 * K], self.out[t0:t1], self.dev_status, main)
            combined = torch.cuda.Event()
            combined.record(main)
            d2h.wait_event(combined)
            with torch.cuda.stream(d2h):
                out_h[t0:t1].copy_(self.out[t0:t1], non_blocking=True)
        if grads:
            self.grad_reduce(False, main)
        main.wait_stream(d2h)
        main.wait_stream(h2d)

    def status(self, stream=None):
        return ep_status_read(self.dev_status, stream)

    def _copy_streams(self):
        if not hasattr(self, "_h2d"):
            self._h2d = torch.cuda.Stream(self.device)
            self._d2h = torch.cuda.Stream(self.device)
        return self._h2d, self._d2h

    # --- plan views -------------------------------------------------------
    def plan_view(self, name, count):
        off = self.plan_layout[name]
        return self.plan[off:off + count]


def run_host_layers(layers, topk_hs, w_hs, x_hs, out_hs, stream=None, grads=True, fused=True, chunks=8):
    """Several layers' host-fed passes (each as EpLayer.run_host: its routing,
    gate weights and hidden rows in from pinned host memory, its combined rows
    out), with the layers' copies overlapping one another.

    The layers may share their row buffers (EpLayer(share=...)): then layer
    l+1's slice j of hidden rows may arrive as soon as layer l has dispatched
    its slice j, and layer l+1 may combine slice j as soon as layer l's slice j
    has left for the host, so layer l+1's inbound copies run while layer l's
    outbound copies drain (the host link is full duplex).  Within a layer the
    slices pipeline exactly as in run_host.  Results: out_hs[l] holds layer
    l's combined rows (the same tensor may be given for every layer; it then
    ends with the last layer's).  The caller's stream waits for every copy."""
    n = len(layers)
    if not (len(topk_hs) == len(w_hs) == len(x_hs) == len(out_hs) == n):
        raise ValueError("one routing, weight, hidden and output buffer per layer")
    if n == 0:
        return
    first = layers[0]
    main = stream if stream is not None else torch.cuda.current_stream(first.device)
    h2d, d2h = first._copy_streams()
    h2d.wait_stream(main)
    d2h.wait_stream(main)
    prev = None  # (x, out, [dispatched events], [sent events]) of the layer before
    for ly, topk_h, w_h, x_h, out_h in zip(layers, topk_hs, w_hs, x_hs, out_hs):
        with torch.cuda.stream(h2d):
            ly.topk_ids.copy_(topk_h, non_blocking=True)
            ly.w.copy_(w_h, non_blocking=True)
            routed = torch.cuda.Event()
            routed.record(h2d)
        main.wait_event(routed)
        ly.route(main, fused)
        bounds = slice_bounds(ly.T, max(1, min(chunks, ly.T)))
        K = ly.K
        ptr = (lambda t: t.data_ptr())
        same_x = prev is not None and ptr(prev[0]) == ptr(ly.x)
        x_is_prev_out = prev is not None and ptr(prev[1]) == ptr(ly.x)  # chained layers (chain_buffers)
        same_out = prev is not None and ptr(prev[1]) == ptr(ly.out)
        dispatched, sent = [], []
        for j, (t0, t1) in enumerate(zip(bounds[:-1], bounds[1:])):
            with torch.cuda.stream(h2d):
                if same_x:
                    h2d.wait_event(prev[2][j])  # the layer before has read these rows of x
                if x_is_prev_out:
                    h2d.wait_event(prev[3][j])  # the layer before's rows here have left for the host
                ly.x[t0:t1].copy_(x_h[t0:t1], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(h2d)
            main.wait_event(arrived)
            ep_dispatch(ly.x[t0:t1], K, ly.pos[t0 * K:t1 * K], ly.buf, ly.dev_status, main)
            ev = torch.cuda.Event()
            ev.record(main)
            dispatched.append(ev)
            if same_out:
                main.wait_event(prev[3][j])  # the layer before's rows of out have left
            ep_combine(ly.buf, ly.w[t0:t1], ly.pos[t0 * K:t1 * K], ly.out[t0:t1], ly.dev_status, main)
            combined = torch.cuda.Event()
            combined.record(main)
            d2h.wait_event(combined)
            with torch.cuda.stream(d2h):
                out_h[t0:t1].copy_(ly.out[t0:t1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(d2h)
                sent.append(ev)
        if grads:
            ly.grad_reduce(False, main)
        prev = (ly.x, ly.out, dispatched, sent)
    main.wait_stream(d2h)
    main.wait_stream(h2d)


def chain_buffers(layers):
    """Make consecutive layers a chain on two row buffers: layer l reads its
    hidden rows from the buffer layer l-1 combined into (layer 0 from the first
    one), as the MoE layers of one forward pass do.  The layers must share
    their row buffers (EpLayer(share=...)); nothing is copied."""
    if not layers:
        return
    a, b = layers[0].x, layers[0].out
    for i, ly in enumerate(layers):
        if ly.x.data_ptr() not in (a.data_ptr(), b.data_ptr()) or ly.out.data_ptr() not in (a.data_ptr(), b.data_ptr()):
            raise ValueError("chained layers must share their row buffers")
        ly.x, ly.out = (a, b) if i % 2 == 0 else (b, a)


def run_host_chain(layers, topk_hs, w_hs, x_h, out_h, stream=None, grads=True, fused=True, chunks=8):
    """A chain of layers (chain_buffers) fed from pinned host memory: every
    layer's routing and gate weights and the batch's hidden rows in, the last
    layer's combined rows out.

    The hidden rows arrive in token slices and the first layer dispatches and
    combines each slice as it lands; the middle layers run on the device; the
    last layer combines slice by slice and each slice leaves as soon as it is
    combined.  Routing for the later layers is copied behind the first layer's
    rows on the same copy stream.  With one layer this is EpLayer.run_host.
    The caller's stream waits for the last copy out.  (run_host_batches with
    one batch, the rows arriving in the first layer's x and leaving from the
    last layer's out.)"""
    run_host_batches(layers, [(topk_hs, w_hs, x_h, out_h)], None, None, stream, grads, fused, chunks)


def _record(stream):
    ev = torch.cuda.Event()
    ev.record(stream)
    return ev


def _routing_stage(ly):
    """Device copies of a layer's routing and gate weights that the next
    batch's may land in while this batch still reads the layer's own."""
    if not hasattr(ly, "_rt_stage"):
        ly._rt_stage = (torch.empty_like(ly.topk_ids), torch.empty_like(ly.w))
    return ly._rt_stage


def batch_gating(layer_bufs, x_stage, out_stage):
    """The waits run_host_batches takes between batch b and batch b+1, from
    which storage each buffer is.  layer_bufs: (x, out) storage identities of
    every layer, in order; x_stage, out_stage: those of the stage buffers.

    x_last_use: the last layer of a batch that reads or writes x_stage's
    storage (layer 0 reads it); out_first_write: the first layer that writes
    out_stage's storage; x_waits_sent: x_stage is out_stage's storage, so the
    next rows also wait for the rows before to have left; x_by_slice: the next
    batch's slice j may come in once this batch's slice j is dispatched (one
    layer only: on a chain the rows wait for the whole first layer, which
    measured faster); out_by_slice: the last layer's slice j may be combined
    once the batch before's slice j has left (no other layer writes
    out_stage's storage)."""
    n = len(layer_bufs)
    if n == 0:
        raise ValueError("no layers")
    x_waits_sent = x_stage == out_stage
    x_last_use = max([0] + [l for l, (x, o) in enumerate(layer_bufs) if x_stage in (x, o)])
    out_first_write = min([n - 1] + [l for l, (x, o) in enumerate(layer_bufs) if o == out_stage])
    return {"x_last_use": x_last_use, "out_first_write": out_first_write, "x_waits_sent": x_waits_sent,
            "x_by_slice": n == 1 and x_last_use == 0 and not x_waits_sent,
            "out_by_slice": out_first_write == n - 1 and not x_waits_sent}


def run_host_batches(layers, batches, x_stage=None, out_stage=None, stream=None, grads=True, fused=True, chunks=8):
    """A chain of layers (chain_buffers) over a sequence of batches fed from
    pinned host memory, the batches overlapping on the host link.

    batches: (topk_hs, w_hs, x_h, out_h) per batch -- every layer's routing
    and gate weights, the batch's hidden rows, and the host buffer for the last
    layer's combined rows.  Each batch runs as in run_host_chain: its rows
    arrive in token slices that the first layer dispatches and combines as
    they land, the middle layers run on the device, and the last layer's
    slices leave as soon as they are combined.

    x_stage and out_stage are the device buffers [T, H] the first layer
    dispatches from and the last layer combines into (default: the first
    layer's x and the last layer's out).  Given apart from the chain's two row
    buffers, batch b+1's rows come in while batch b's later layers still run
    and batch b's rows go out while batch b+1's layers run: the inbound copies
    wait for batch b's first layer to have read x_stage (with one layer, slice
    j waits only for batch b's slice j to have been dispatched), and the last
    layer of batch b+1 writes slice j of out_stage once batch b's slice j has
    left.  With several batches a layer's routing and gate weights for batch
    b+1 arrive in a device copy of their own and move into the layer's buffers
    on the compute stream, so they never wait for batch b.  With the default
    buffers every wait falls on the last layer that uses the buffer, so the
    batches run one after another.  The caller's stream waits for every copy."""
    batches = list(batches)
    n = len(layers)
    if n == 0:
        raise ValueError("no layers")
    first, last = layers[0], layers[-1]
    x_stage = first.x if x_stage is None else x_stage
    out_stage = last.out if out_stage is None else out_stage
    for t in (x_stage, out_stage):
        if t.shape != first.x.shape or t.dtype != first.x.dtype or t.device != first.x.device:
            raise ValueError("x_stage and out_stage must be [T, H] bf16 buffers on the layers' device")
    ptr = (lambda t: t.data_ptr())
    g = batch_gating([(ptr(ly.x), ptr(ly.out)) for ly in layers], ptr(x_stage), ptr(out_stage))
    x_waits_sent, x_last_use, out_first_write = g["x_waits_sent"], g["x_last_use"], g["out_first_write"]
    x_by_slice, out_by_slice = g["x_by_slice"], g["out_by_slice"]
    staged_routing = len(batches) > 1
    main = stream if stream is not None else torch.cuda.current_stream(first.device)
    h2d, d2h = first._copy_streams()
    h2d.wait_stream(main)
    d2h.wait_stream(main)
    T, K = first.T, first.K
    bounds = slice_bounds(T, max(1, min(chunks, T)))
    spans = list(zip(bounds[:-1], bounds[1:]))
    layer_done = [None] * n          # main finished layer l of the batch before
    rt_taken = [None] * n            # main moved the batch before's staged routing of layer l into the layer
    dispatched = [None] * len(spans)  # the batch before's first layer dispatched slice j (its rows are free)
    left = [None] * len(spans)       # the batch before's slice j has left out_stage
    sent = None                      # the batch before's rows have all left out_stage

    def routing_in(l, topk_h, w_h):
        ly = layers[l]
        if staged_routing:
            if rt_taken[l] is not None:
                h2d.wait_event(rt_taken[l])
            st_t, st_w = _routing_stage(ly)
        else:
            if layer_done[l] is not None:
                h2d.wait_event(layer_done[l])
            st_t, st_w = ly.topk_ids, ly.w
        st_t.copy_(topk_h, non_blocking=True)
        st_w.copy_(w_h, non_blocking=True)
        return _record(h2d)

    for topk_hs, w_hs, x_h, out_h in batches:
        if not (len(topk_hs) == len(w_hs) == n):
            raise ValueError("one routing and weight buffer per layer")
        routed, arrived = [None] * n, []
        with torch.cuda.stream(h2d):
            routed[0] = routing_in(0, topk_hs[0], w_hs[0])
            if not x_by_slice:
                if layer_done[x_last_use] is not None:
                    h2d.wait_event(layer_done[x_last_use])
                if x_waits_sent and sent is not None:
                    h2d.wait_event(sent)
            for j, (t0, t1) in enumerate(spans):
                if x_by_slice and dispatched[j] is not None:
                    h2d.wait_event(dispatched[j])
                x_stage[t0:t1].copy_(x_h[t0:t1], non_blocking=True)
                arrived.append(_record(h2d))
            for l in range(1, n):
                routed[l] = routing_in(l, topk_hs[l], w_hs[l])
        for l, ly in enumerate(layers):
            main.wait_event(routed[l])
            if staged_routing:
                st_t, st_w = _routing_stage(ly)
                with torch.cuda.stream(main):
                    ly.topk_ids.copy_(st_t, non_blocking=True)
                    ly.w.copy_(st_w, non_blocking=True)
                rt_taken[l] = _record(main)
            ly.route(main, fused)
            if l == out_first_write and sent is not None and not out_by_slice:
                main.wait_event(sent)
            if l == 0 or l == n - 1:
                # a token slice's combine reads only the rows its own dispatch wrote
                rows_in = x_stage if l == 0 else ly.x
                rows_out = out_stage if l == n - 1 else ly.out
                for j, (t0, t1) in enumerate(spans):
                    if l == 0:
                        main.wait_event(arrived[j])
                    ep_dispatch(rows_in[t0:t1], K, ly.pos[t0 * K:t1 * K], ly.buf, ly.dev_status, main)
                    if l == 0:
                        dispatched[j] = _record(main)
                    if l == n - 1 and out_by_slice and left[j] is not None:
                        main.wait_event(left[j])
                    ep_combine(ly.buf, ly.w[t0:t1], ly.pos[t0 * K:t1 * K], rows_out[t0:t1], ly.dev_status, main)
                    if l == n - 1:
                        d2h.wait_event(_record(main))
                        with torch.cuda.stream(d2h):
                            out_h[t0:t1].copy_(rows_out[t0:t1], non_blocking=True)
                            left[j] = _record(d2h)
            else:
                ly.dispatch(main)
                ly.combine(main)
            layer_done[l] = _record(main)
            if grads:
                ly.grad_reduce(False, main)
        sent = _record(d2h)
    main.wait_stream(d2h)
    main.wait_stream(h2d)
