"""Pins for the CPU oracle: checks against facts fixed by the source pages and
by mathematics, never against the oracle itself.

Each pin takes a loaded oracle library `L` (so the mutation tests can run the
same pins on deliberately broken copies) and raises AssertionError on failure.

Kinds of pin used:
  * the hand-worked 4-rank example (tests/golden/hand_example_4rank.json), every
    value derived by hand from the definitions;
  * brute force: all P! row permutations of tiny cases, filtered by the
    layout's defining predicates -- exactly one must survive;
  * reductions to library routines in special cases (numpy stable argsort,
    fancy indexing, float32 adds);
  * closed forms (max_vio of uniform / single-expert routing) and fp64 error
    bounds for the fp32 sums;
  * invariants the pages state (S*K rows per rank, routing unchanged, copies of
    an expert add up to T_e).
"""
import itertools
import json
import math
import os

import numpy as np

import oracle as O
import workload as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example_4rank.json")
QUOTA_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quota_hand_example_4rank.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- helpers

def unit_plan(loads, R, S, K, E):
    """Independent statement of the replica rule at the level of single pairs:
    list the excess pairs one by one (overloaded ranks ascending, within a rank
    its home experts by descending id, each expert giving up to what is still
    in excess), list the missing pairs one by one (underloaded ranks ascending),
    pair them up position by position, and merge runs of equal (expert, rank)."""
    ER, SK = E // R, S * K
    excess_units, deficit_units = [], []
    for r in range(R):
        Lr = sum(int(loads[e]) for e in range(r * ER, (r + 1) * ER))
        if Lr > SK:
            rem = Lr - SK
            for e in reversed(range(r * ER, (r + 1) * ER)):
                take = min(int(loads[e]), rem)
                excess_units += [e] * take
                rem -= take
        elif Lr < SK:
            deficit_units += [r] * (SK - Lr)
    assert len(excess_units) == len(deficit_units)
    reps = []
    for e, r in zip(excess_units, deficit_units):
        if reps and reps[-1][0] == e and reps[-1][1] == r:
            reps[-1][2] += 1
        else:
            reps.append([e, r, 1])
    return reps


def slots_from_plan(pl, R, S, K, E):
    """Buffer slots in order: (slot id, logical expert, first row, rows)."""
    ER, SK = E // R, S * K
    out = []
    for r in range(R):
        row = r * SK
        for e in range(r * ER, (r + 1) * ER):
            out.append((e, e, row, int(pl["home_count"][e])))
            row += int(pl["home_count"][e])
        for m in range(pl["n_rep"]):
            if pl["rep_rank"][m] == r:
                out.append((E + m, int(pl["rep_expert"][m]), row, int(pl["rep_count"][m])))
                row += int(pl["rep_count"][m])
        assert row == (r + 1) * SK, "rank does not hold exactly S*K rows"
    return out


def layout_predicates_hold(pos, topk_flat, pl, R, S, K, E):
    """The defining predicates of the layout, given the plan."""
    slots = slots_from_plan(pl, R, S, K, E)
    P = len(topk_flat)
    row_slot = np.empty(P, dtype=np.int64)
    row_expert = np.empty(P, dtype=np.int64)
    for sid, e, first, n in slots:
        row_slot[first:first + n] = sid
        row_expert[first:first + n] = e
    # routing unchanged: the row's copy is a copy of the pair's expert
    if not np.array_equal(row_expert[pos], topk_flat):
        return False
    # within a slot, rows follow ascending p
    src = np.empty(P, dtype=np.int64)
    src[pos] = np.arange(P)
    for sid, e, first, n in slots:
        if n > 1 and not np.all(np.diff(src[first:first + n]) > 0):
            return False
    # an expert's copies take consecutive ranges of its pairs: home first, then
    # replicas in match order
    for e in range(E):
        copies = [s for s in slots if s[1] == e and s[0] == e] + sorted(
            [s for s in slots if s[1] == e and s[0] >= E], key=lambda s: s[0])
        last = -1
        for sid, _, first, n in copies:
            if n == 0:
                continue
            ps = src[first:first + n]
            if ps.min() <= last:
                return False
            last = ps.max()
    return True


def check_layout_invariants(topk, pl, lo, R, S, K, E):
    topk_flat = np.asarray(topk, dtype=np.int64).reshape(-1)
    P = topk_flat.size
    SK = S * K
    pos, src = lo["pos"].astype(np.int64), lo["src"].astype(np.int64)
    # pos is a permutation of [0, P) and src its inverse
    assert np.array_equal(np.sort(pos), np.arange(P))
    assert np.array_equal(src[pos], np.arange(P))
    # S*K rows per rank: every row index in [r*SK, (r+1)*SK) is used once (permutation)
    # and the slot lengths of each rank add up to S*K
    cu = lo["cu_seqlens"].astype(np.int64)
    order = lo["slot_order"]
    n_rep = pl["n_rep"]
    assert len(order) == E + n_rep and cu[0] == 0 and cu[-1] == P and np.all(np.diff(cu) >= 0)
    # slot -> logical expert
    slot_expert = np.concatenate([np.arange(E), np.asarray(pl["rep_expert"], dtype=np.int64)])
    assert np.array_equal(slot_expert[lo["pair_slot"]], topk_flat), "routing changed"
    # each pair's row lies inside its slot's range
    where = np.empty(E + n_rep, dtype=np.int64)
    where[order] = np.arange(E + n_rep)
    i = where[lo["pair_slot"]]
    assert np.all(cu[i] <= pos) and np.all(pos < cu[i + 1])
    # rank sizes: slot ranges of rank r stay in [r*SK, (r+1)*SK)
    ER = E // R
    for r in range(R):
        assert np.sum((pos >= r * SK) & (pos < (r + 1) * SK)) == SK
    # copies of each expert add up to T_e
    loads = np.bincount(topk_flat, minlength=E)
    per = np.asarray(pl["home_count"], dtype=np.int64).copy()
    np.add.at(per, np.asarray(pl["rep_expert"], dtype=np.int64), np.asarray(pl["rep_count"], dtype=np.int64))
    assert np.array_equal(per, loads)
    # replicas go from overloaded home ranks to underloaded ranks
    rank_load = loads.reshape(R, ER).sum(1)
    for m in range(n_rep):
        e, r = int(pl["rep_expert"][m]), int(pl["rep_rank"][m])
        assert rank_load[e // ER] > SK and rank_load[r] < SK and r != e // ER
        assert pl["rep_count"][m] > 0
    return True


# ------------------------------------------------------------------- pins

def pin_hand_example(L):
    g = golden()
    R, S, K, E, bm = g["R"], g["S"], g["K"], g["E"], g["block_m"]
    topk = np.array(g["topk_ids"], dtype=np.int32)
    loads, mv, bad = O.route_stats(topk, E, L=L)
    assert bad == 0
    assert loads.tolist() == g["loads"]
    assert mv == g["max_vio"]
    pl = O.plan(loads, R, S, K, E, L=L)
    assert [[int(a), int(b), int(c)] for a, b, c in zip(pl["rep_expert"], pl["rep_rank"], pl["rep_count"])] == \
        g["replicas"]
    assert pl["home_count"].tolist() == g["home_count"]
    lo = O.layout(topk, pl, R, S, E, L=L)
    assert lo["pos"].tolist() == g["pos"]
    assert lo["slot_order"].tolist() == g["slot_order"]
    assert lo["cu_seqlens"].tolist() == g["cu_seqlens"]
    ids, eids, n = O.align_sort(topk, E, bm, L=L)
    assert n == g["align_num_tokens_post_pad"]
    assert len(ids) == g["align_capacity"]
    pre = g["align_sorted_token_ids_prefix"]
    assert ids[:len(pre)].tolist() == pre
    assert np.all(ids[len(pre):] == g["align_sentinel"])
    assert eids.tolist() == g["align_expert_ids"]


def pin_max_vio_closed_forms(L):
    # uniform routing: every expert gets P/E pairs -> 0 (perfect balance)
    for (T, E, K) in [(64, 16, 2), (96, 8, 4), (256, 64, 8)]:
        topk, _ = W.routing_from(T, E, K, seed=1, uniform=True)
        loads, mv, _ = O.route_stats(topk, E, L=L)
        assert np.all(loads == T * K // E) and mv == 0.0
    # all tokens on one expert with K = 1: max T_e = P, mean P/E -> E - 1
    for E in (2, 7, 64):
        topk = np.full((40, 1), E - 1, dtype=np.int32)
        loads, mv, _ = O.route_stats(topk, E, L=L)
        assert loads[E - 1] == 40 and loads[:E - 1].sum() == 0 and mv == float(E - 1)
    # ids out of range are reported, not counted
    topk = np.array([[0, 1], [2, 9]], dtype=np.int32)
    loads, mv, bad = O.route_stats(topk, 4, L=L)
    assert bad == 1 and loads.tolist() == [1, 1, 1, 0]
    # a generic case against exact rational arithmetic: max_e T_e / (P/E) - 1
    topk, _ = W.routing_from(300, 12, 3, seed=5, bias_e=np.linspace(1, -1, 12))
    loads, mv, _ = O.route_stats(topk, 12, L=L)
    ref = np.bincount(topk.ravel(), minlength=12)
    from fractions import Fraction
    exact = Fraction(int(ref.max()), 1) / Fraction(900, 12) - 1
    assert loads.tolist() == ref.tolist()
    assert abs(mv - float(exact)) <= 2 * math.ulp(float(exact) + 1.0)


def _rand_loads(rng, R, ER, SK):
    E = R * ER
    total = R * SK
    mode = rng.integers(0, 4)
    if mode == 0:  # multinomial with a random skew
        p = rng.dirichlet(np.full(E, rng.uniform(0.1, 3.0)))
        return rng.multinomial(total, p).astype(np.int32)
    if mode == 1:  # one hot expert
        loads = np.zeros(E, dtype=np.int32)
        loads[rng.integers(0, E)] = total
        return loads
    if mode == 2:  # balanced
        loads = np.zeros(E, dtype=np.int32)
        for r in range(R):
            part = rng.multinomial(SK, np.full(ER, 1.0 / ER))
            loads[r * ER:(r + 1) * ER] = part
        return loads
    loads = rng.multinomial(total, np.full(E, 1.0 / E)).astype(np.int32)  # near uniform
    return loads


def pin_plan_unit_restatement(L):
    rng = np.random.default_rng(1234)
    for it in range(400):
        R = int(rng.choice([1, 2, 3, 4, 5, 8]))
        ER = int(rng.integers(1, 6))
        SK = int(rng.integers(1, 40))
        E = R * ER
        K = int(rng.integers(1, 4))
        if SK % K:
            SK = K * max(1, SK // K)
        S = SK // K
        loads = _rand_loads(rng, R, ER, SK)
        pl = O.plan(loads, R, S, K, E, L=L)
        ref = unit_plan(loads, R, S, K, E)
        got = [[int(a), int(b), int(c)] for a, b, c in zip(pl["rep_expert"], pl["rep_rank"], pl["rep_count"])]
        assert got == ref, (loads.tolist(), R, S, K, got, ref)
        # every rank ends with exactly S*K pairs
        rows = np.zeros(R, dtype=np.int64)
        for e in range(E):
            rows[e // ER] += pl["home_count"][e]
        for e, r, c in got:
            rows[r] += c
        assert np.all(rows == SK)
        assert np.all(pl["home_count"] >= 0)
        n_chunks = len({e for e, _, _ in got})
        n_def = len({r for _, r, _ in got})
        assert len(got) <= max(0, n_chunks + n_def - 1)
        assert len(got) <= E + R - 1
    # uniform loads: no replica at all
    pl = O.plan(np.full(16, 8, dtype=np.int32), 4, 16, 2, 16, L=L)
    assert pl["n_rep"] == 0 and np.all(pl["home_count"] == 8)


def pin_layout_brute_force(L):
    """All P! permutations of the rows of tiny cases; exactly one satisfies the
    layout's defining predicates, and it is the oracle's."""
    rng = np.random.default_rng(7)
    cases = []
    for R, E, S, K in [(2, 2, 2, 2), (2, 4, 2, 2), (2, 4, 4, 1), (2, 2, 4, 1), (1, 3, 2, 2), (2, 4, 1, 2)]:
        for _ in range(3):
            T = R * S
            topk = np.stack([rng.choice(E, size=K, replace=False) for _ in range(T)]).astype(np.int32)
            cases.append((R, E, S, K, topk))
    # a degenerate one: all pairs on expert 0
    cases.append((2, 2, 4, 1, np.zeros((8, 1), dtype=np.int32)))
    for R, E, S, K, topk in cases:
        P = R * S * K
        loads, _, _ = O.route_stats(topk, E, L=L)
        pl = O.plan(loads, R, S, K, E, L=L)
        lo = O.layout(topk, pl, R, S, E, L=L)
        flat = topk.reshape(-1).astype(np.int64)
        survivors = [np.array(perm) for perm in itertools.permutations(range(P))
                     if layout_predicates_hold(np.array(perm), flat, pl, R, S, K, E)]
        assert len(survivors) == 1, (topk.tolist(), len(survivors))
        assert np.array_equal(survivors[0], lo["pos"])


def pin_layout_library_reductions(L):
    """With no replicas (one rank, or balanced ranks), rows are the pairs sorted
    by expert, stable in p: the inverse of numpy's stable argsort."""
    for seed, (R, S, K, E) in enumerate([(1, 50, 3, 7), (1, 300, 8, 64), (4, 10, 2, 8)]):
        if R == 1:
            topk, _ = W.routing_from(R * S, E, K, seed=seed, bias_e=np.linspace(2, -2, E))
        else:
            topk, _ = W.routing_from(R * S, E, K, seed=seed, uniform=True)
        loads, _, _ = O.route_stats(topk, E, L=L)
        pl = O.plan(loads, R, S, K, E, L=L)
        assert pl["n_rep"] == 0
        lo = O.layout(topk, pl, R, S, E, L=L)
        src = np.argsort(topk.reshape(-1), kind="stable")
        assert np.array_equal(lo["src"], src)
        assert np.array_equal(lo["pos"][src], np.arange(R * S * K))


def pin_layout_invariants(L):
    rng = np.random.default_rng(99)
    for it in range(40):
        R = int(rng.choice([1, 2, 3, 4, 8]))
        ER = int(rng.integers(1, 7))
        E = R * ER
        K = int(rng.integers(1, min(8, E) + 1))
        S = int(rng.integers(1, 50))
        variant = rng.integers(0, 3)
        if variant == 0:
            topk, _ = W.routing_from(R * S, E, K, seed=it, bias_e=rng.normal(0, 2, E))
        elif variant == 1:
            topk, _ = W.routing_from(R * S, E, K, seed=it, uniform=True)
        else:
            topk, _ = W.routing_from(R * S, E, K, seed=it, force_expert0=True)
        loads, _, _ = O.route_stats(topk, E, L=L)
        pl = O.plan(loads, R, S, K, E, L=L)
        lo = O.layout(topk, pl, R, S, E, L=L)
        check_layout_invariants(topk, pl, lo, R, S, K, E)


def pin_align_sort(L):
    # block_m = 1: no padding; the ids are numpy's stable argsort by expert
    for seed, (T, K, E) in enumerate([(37, 3, 9), (200, 8, 64), (16, 2, 8)]):
        topk, _ = W.routing_from(T, E, K, seed=seed, bias_e=np.linspace(1.5, -1.5, E))
        ids, eids, n = O.align_sort(topk, E, 1, L=L)
        P = T * K
        assert n == P
        assert np.array_equal(ids[:P], np.argsort(topk.reshape(-1), kind="stable"))
        assert np.array_equal(eids[:P], np.sort(topk.reshape(-1)))
    # invariants at several block sizes, including experts with no pairs
    rng = np.random.default_rng(3)
    for it in range(30):
        E = int(rng.integers(1, 40))
        K = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(0, 200))
        bm = int(rng.choice([1, 2, 3, 4, 16, 64, 128]))
        topk, _ = W.routing_from(T, E, K, seed=it, bias_e=rng.normal(0, 2, E)) if T else \
            (np.zeros((0, K), np.int32), None)
        P = T * K
        ids, eids, n = O.align_sort(topk, E, bm, L=L)
        cap, capb = O.align_sort_capacity(P, E, bm)
        assert len(ids) == cap and len(eids) == capb
        assert n % bm == 0
        counts = np.bincount(topk.reshape(-1), minlength=E)
        assert n == sum(-(-int(c) // bm) * bm for c in counts)
        assert np.all(ids[n:] == P) and np.all(eids[n // bm:] == -1)
        valid = ids[:n][ids[:n] != P]
        assert np.array_equal(np.sort(valid), np.arange(P))
        flat = topk.reshape(-1)
        for b in range(n // bm):
            blk = ids[b * bm:(b + 1) * bm]
            blk = blk[blk != P]
            assert len(blk) > 0  # no block is padding only
            assert np.all(flat[blk] == eids[b])
            assert np.all(np.diff(blk) > 0)
        assert np.all(np.diff(eids[:n // bm]) >= 0)


def pin_dispatch(L):
    rng = np.random.default_rng(11)
    for (R, S, K, E, H) in [(2, 3, 2, 4, 8), (4, 16, 4, 16, 64), (1, 5, 1, 3, 16)]:
        topk, _ = W.routing_from(R * S, E, K, seed=int(rng.integers(1 << 30)), bias_e=rng.normal(0, 1, E))
        loads, _, _ = O.route_stats(topk, E, L=L)
        pl = O.plan(loads, R, S, K, E, L=L)
        lo = O.layout(topk, pl, R, S, E, L=L)
        x = W.hidden(R * S, H, seed=3)
        buf = O.dispatch(x, lo["pos"], K, R * S * K, L=L)
        ref = np.zeros_like(buf)
        ref[lo["pos"]] = np.repeat(x, K, axis=0)  # numpy scatter
        assert np.array_equal(buf, ref)


def pin_combine(L):
    rng = np.random.default_rng(5)
    # hand-computed rounding cases, K = 1, y = 1.0: the result is bf16_rn(w).
    # bf16 keeps 8 significant bits, so in [1, 2) its spacing is 2^-7:
    #   1 + 2^-8      is halfway between 1 and 1 + 2^-7       -> ties to even: 1.0
    #   1 + 3*2^-8    is halfway between 1 + 2^-7 and 1 + 2^-6 -> ties to even: 1 + 2^-6
    #   1 + 2^-8 + 2^-20 is above halfway                       -> 1 + 2^-7
    #   -(1 + 2^-8)   ties to even, sign kept                    -> -1.0
    ws = np.array([[1 + 2.0 ** -8], [1 + 3 * 2.0 ** -8], [1 + 2.0 ** -8 + 2.0 ** -20], [-(1 + 2.0 ** -8)]],
                  dtype=np.float32)
    one = np.full((4, 1), 0x3F80, dtype=np.uint16)  # bf16 1.0
    out = O.combine(one, ws, np.arange(4, dtype=np.int32), 1, L=L)
    assert O.bf16_to_f32(out[:, 0]).tolist() == [1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7, -1.0]
    # K = 1, w = 1: out is the y row itself, bit for bit
    T, H, E = 20, 32, 6
    topk = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    y = W.hidden(T, H, seed=9)
    pos = rng.permutation(T).astype(np.int32)
    out = O.combine(y, np.ones((T, 1), np.float32), pos, 1, L=L)
    assert np.array_equal(out, y[pos])
    # general K: within fp32-sum error bound of the fp64 sum, then one bf16 rounding
    for (R, S, K, E, H) in [(2, 8, 4, 8, 16), (4, 12, 3, 12, 40), (2, 4, 2, 2, 8)]:
        T = R * S
        topk, w = W.routing_from(T, E, K, seed=int(rng.integers(1 << 30)), bias_e=rng.normal(0, 1, E))
        loads, _, _ = O.route_stats(topk, E, L=L)
        pl = O.plan(loads, R, S, K, E, L=L)
        lo = O.layout(topk, pl, R, S, E, L=L)
        y = W.hidden(T * K, H, seed=17)
        out = O.combine(y, w, lo["pos"], K, L=L)
        yf = O.bf16_to_f32(y).astype(np.float64)
        rows = yf[lo["pos"].reshape(T, K)]                       # [T, K, H]
        exact = np.einsum("tk,tkh->th", w.astype(np.float64), rows)
        absum = np.einsum("tk,tkh->th", np.abs(w.astype(np.float64)), np.abs(rows))
        got = O.bf16_to_f32(out).astype(np.float64)
        # fp32 error of K products and K-1 adds, plus half a bf16 ulp of the result
        bound = 2 * K * 2.0 ** -24 * absum + np.abs(exact) * 2.0 ** -8 + 1e-30
        assert np.all(np.abs(got - exact) <= bound)
        # the stand-in expert's closed form agrees with the definition through the layout
        scale = W.expert_scale(E)
        x = W.hidden(T, H, seed=21)
        buf = O.dispatch(x, lo["pos"], K, T * K, L=L)
        y2 = O.expert_standin(buf, lo["src"], topk, scale, L=L)
        out_def = O.combine(y2, w, lo["pos"], K, L=L)
        out_cf = O.combine_closed(x, w, topk, scale, L=L)
        assert np.array_equal(out_def, out_cf)
        # and the closed form is the bf16 rounding of an fp32 sum within the bound
        xf = O.bf16_to_f32(x).astype(np.float64)
        yv = O.bf16_to_f32(
            _bf16_rne((O.bf16_to_f32(x)[:, None, :] * scale[topk][:, :, None]).astype(np.float32))
        ).astype(np.float64)
        exact = np.einsum("tk,tkh->th", w.astype(np.float64), yv)
        absum = np.einsum("tk,tkh->th", np.abs(w.astype(np.float64)), np.abs(yv))
        got = O.bf16_to_f32(out_cf).astype(np.float64)
        assert np.all(np.abs(got - exact) <= 2 * K * 2.0 ** -24 * absum + np.abs(exact) * 2.0 ** -8 + 1e-30)
        del xf


def _bf16_rne(f32):
    u = np.asarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def pin_grad_reduce(L):
    rng = np.random.default_rng(8)
    E, n = 6, 257
    g_home = W.grad_rows(1, W.STREAM_GHOME, n, E)
    # no replica: unchanged
    gh, _ = O.grad_reduce(g_home, np.zeros((1, n), np.float32), [], L=L)
    assert np.array_equal(gh, g_home)
    # one replica: the single fp32 add (numpy float32 addition)
    g_rep = W.grad_rows(2, W.STREAM_GREP, n, 1)
    gh, _ = O.grad_reduce(g_home, g_rep, [4], L=L)
    ref = g_home.copy()
    ref[4] = (g_home[4] + g_rep[0]).astype(np.float32)
    assert np.array_equal(gh, ref)
    # several replicas per expert, in match order, fp32 and bf16 replica rows
    rep_expert = [2, 2, 5, 0, 2]
    for dt in ("f32", "bf16"):
        g_rep = W.grad_rows(3, W.STREAM_GREP, n, len(rep_expert), dtype=dt)
        gr_f = g_rep if dt == "f32" else O.bf16_to_f32(g_rep)
        gh, gr2 = O.grad_reduce(g_home, g_rep, rep_expert, clear=True, L=L)
        ref = g_home.copy()
        for m, e in enumerate(rep_expert):  # home first, then replicas in match order
            ref[e] = (ref[e] + gr_f[m]).astype(np.float32)
        assert np.array_equal(gh, ref)
        assert not np.any(gr2)  # cleared
        # fp64 bound: at most 3 fp32 adds per element
        exact = g_home.astype(np.float64).copy()
        absum = np.abs(exact).copy()
        for m, e in enumerate(rep_expert):
            exact[e] += gr_f[m]
            absum[e] += np.abs(gr_f[m])
        assert np.all(np.abs(gh - exact) <= 3 * 2.0 ** -24 * absum + 1e-30)
        _ = rng


def pin_dispatch_backward(L):
    rng = np.random.default_rng(21)
    # K = 1: the gradient of a pure permutation is the inverse permutation
    T, H = 30, 24
    dbuf = W.hidden(T, H, seed=31)
    pos = rng.permutation(T).astype(np.int32)
    np.testing.assert_array_equal(O.dispatch_backward(dbuf, pos, T, 1, L=L), dbuf[pos])
    # backward of dispatch applied to dispatch(x): every token gets K copies of x,
    # and j*x is exact in fp32 for a bf16 x, so dx = bf16_rn(K * x) in closed form
    for K in (2, 3, 4, 6, 8):
        T, H = 20, 16
        x = W.hidden(T, H, seed=K)
        pos = rng.permutation(T * K).astype(np.int32)
        buf = O.dispatch(x, pos, K, T * K, L=L)
        dx = O.dispatch_backward(buf, pos, T, K, L=L)
        ref = _bf16_rne(O.bf16_to_f32(x) * np.float32(K))
        np.testing.assert_array_equal(dx, ref)
    # general rows: fp32 sum of K terms within its error bound of the fp64 sum
    T, K, H = 25, 5, 40
    dbuf = W.hidden(T * K, H, seed=41)
    pos = rng.permutation(T * K).astype(np.int32)
    pos[7] = -1  # a pair without a row contributes nothing
    dx = O.bf16_to_f32(O.dispatch_backward(dbuf, pos, T, K, L=L)).astype(np.float64)
    rows = O.bf16_to_f32(dbuf).astype(np.float64)[np.maximum(pos, 0)].reshape(T, K, H)
    rows[7 // K, 7 % K] = 0.0
    exact = rows.sum(1)
    assert np.all(np.abs(dx - exact) <= K * 2.0 ** -24 * np.abs(rows).sum(1) + np.abs(exact) * 2.0 ** -8 + 1e-30)


def pin_combine_backward(L):
    rng = np.random.default_rng(22)
    T, K, H = 16, 3, 32
    P = T * K
    dout = W.hidden(T, H, seed=51)
    y = W.hidden(P, H, seed=52)
    pos = rng.permutation(P).astype(np.int32)
    # w = 1: dy rows are dout rows, exactly
    dy, dw = O.combine_backward(dout, np.ones((T, K), np.float32), y, pos, L=L)
    np.testing.assert_array_equal(dy[pos].reshape(T, K, H), np.repeat(dout[:, None, :], K, axis=1))
    # general weights: dy = bf16_rn(float32 product), dw = the fp64 dot product
    w = rng.uniform(-2, 2, (T, K)).astype(np.float32)
    init = np.full((P + 5, H), 0x1234, dtype=np.uint16)
    y5 = np.concatenate([y, W.hidden(5, H, seed=53)])
    dy, dw = O.combine_backward(dout, w, y5, pos, dy_init=init, L=L)
    ref = _bf16_rne(O.bf16_to_f32(dout)[:, None, :] * w[:, :, None])       # [T, K, H]
    np.testing.assert_array_equal(dy[pos].reshape(T, K, H), ref)
    assert np.all(dy[P:] == 0x1234)  # rows no pair addresses are left alone
    dref = np.einsum("th,tkh->tk", O.bf16_to_f32(dout).astype(np.float64),
                     O.bf16_to_f32(y5).astype(np.float64)[pos].reshape(T, K, H))
    np.testing.assert_allclose(dw, dref, rtol=1e-12, atol=1e-12)
    # y rows equal to their token's dout row: dw is the squared norm
    y_same = np.repeat(dout, K, axis=0)[np.argsort(pos)]
    _, dw2 = O.combine_backward(dout, w, y_same, pos, L=L)
    sq = (O.bf16_to_f32(dout).astype(np.float64) ** 2).sum(1)
    np.testing.assert_allclose(dw2, np.repeat(sq[:, None], K, axis=1), rtol=1e-12)


def pin_prefetch_slots(L):
    g = golden()
    R, S, K, E = g["R"], g["S"], g["K"], g["E"]
    SK = S * K
    topk = np.array(g["topk_ids"], dtype=np.int32)
    loads, _, _ = O.route_stats(topk, E, L=L)
    pl = O.plan(loads, R, S, K, E, L=L)
    # hand example: m0 (expert 1, 4 pairs) -> rank 1; m1 (expert 0, 2 pairs) and
    # m2 (expert 5, 4 pairs) -> rank 3
    slot, nrem, capped = O.prefetch_slots(pl, E, R, 2, SK, L=L)
    assert slot.tolist() == [8, 8, 9] and nrem.tolist() == [0, 0, 0, 0] and capped.tolist() == [8, 8, 8, 8]
    slot, nrem, capped = O.prefetch_slots(pl, E, R, 1, SK, L=L)
    assert slot.tolist() == [8, 8, -1] and nrem.tolist() == [0, 0, 0, 1]
    assert capped.tolist() == [8, 8, 12, 4]  # expert 5's 4 pairs back on rank 2
    slot, nrem, capped = O.prefetch_slots(pl, E, R, 0, SK, L=L)
    assert slot.tolist() == [-1, -1, -1] and nrem.tolist() == [0, 1, 0, 2]
    assert capped.tolist() == g["rank_loads"]  # no replica: the unplanned loads
    # random plans: slots on a rank are E, E+1, ... in match order up to B; the
    # remote count is what does not fit; B = 0 gives each rank the sum of its
    # experts' loads, a B above every rank's replica count gives S*K, and the
    # capped loads always sum to R*S*K
    rng = np.random.default_rng(17)
    for it in range(100):
        R = int(rng.choice([2, 4, 8])); ER = int(rng.integers(1, 5)); E = R * ER
        SK = int(rng.integers(4, 40)); loads = _rand_loads(rng, R, ER, SK)
        pl = O.plan(loads, R, SK, 1, E, L=L)
        B = int(rng.integers(0, 4))
        slot, nrem, capped = O.prefetch_slots(pl, E, R, B, SK, L=L)
        for r in range(R):
            mine = [m for m in range(pl["n_rep"]) if pl["rep_rank"][m] == r]
            want = [E + j if j < B else -1 for j in range(len(mine))]
            assert [int(slot[m]) for m in mine] == want
            assert nrem[r] == max(0, len(mine) - B)
        assert int(capped.sum()) == R * SK
        unplanned = loads.reshape(R, ER).sum(axis=1)
        assert O.prefetch_slots(pl, E, R, 0, SK, L=L)[2].tolist() == unplanned.tolist()
        assert O.prefetch_slots(pl, E, R, E + R, SK, L=L)[2].tolist() == [SK] * R


# ------------------------------------------------------- quota planner

def pin_quota_hand_example(L):
    g = golden()
    with open(QUOTA_GOLDEN) as f:
        q = json.load(f)
    R, S, K, E = g["R"], g["S"], g["K"], g["E"]
    topk = np.array(g["topk_ids"], dtype=np.int32)
    assert O.load_matrix(topk, R, S, K, E, L=L).tolist() == q["load_matrix"]
    loads = np.array(g["loads"], dtype=np.int32)
    for key, B in (("B1", 1), ("B2", 2), ("B0", 0)):
        want = q[key]
        qp = O.quota_plan(loads, R, S, K, E, B, L=L)
        assert qp["tau"] == want["tau"], (key, qp["tau"])
        reps = [[int(a), int(b), int(c)] for a, b, c in zip(qp["rep_expert"], qp["rep_rank"], qp["rep_count"])]
        assert reps == want["replicas"], (key, reps)
        if "home_quota" in want:
            assert qp["home_quota"].tolist() == want["home_quota"]
        lo = O.quota_layout(topk, qp, R, S, K, E, L=L)
        assert lo["rank_load"].tolist() == want["rank_load"]
        assert lo["n_local"] == want["n_local"]
        for name in ("pos", "slot_order", "cu_seqlens"):
            if name in want:
                assert lo[name].tolist() == want[name], (key, name)


def pin_quota_threshold_closed_forms(L):
    """R = 2: one rank sheds, the other takes every chunk as one piece, so tau is
    feasible iff the B heaviest experts of the heavier rank cover its excess:
    tau* = max(ceil(P/2), H_o - (sum of its B largest loads)).  Any R: B = 0
    leaves only tau = max H_r (nothing shed); unlimited slots make ceil(P/R)
    feasible (the rooms then hold at least the excess)."""
    rng = np.random.default_rng(31)
    for it in range(300):
        R = 2 if it < 200 else int(rng.choice([3, 4, 8]))
        ER = int(rng.integers(1, 6))
        E = R * ER
        P = int(rng.integers(1, 200))
        loads = rng.multinomial(P, rng.dirichlet(np.full(E, rng.uniform(0.1, 3.0)))).astype(np.int32)
        H = loads.reshape(R, ER).sum(axis=1)
        lo = -(-P // R)
        B = int(rng.integers(0, ER + 2))
        if R == 2:
            o = int(np.argmax(H))
            top = int(np.sort(loads[o * ER:(o + 1) * ER])[::-1][:B].sum())
            assert O.quota_threshold(loads, E, R, P, B, L=L) == max(lo, int(H[o]) - top), (loads.tolist(), B)
        assert O.quota_threshold(loads, E, R, P, 0, L=L) == max(lo, int(H.max()))
        assert O.quota_threshold(loads, E, R, P, E + R, L=L) == lo


def _quota_case(rng, it):
    R = int(rng.choice([1, 2, 3, 4, 8]))
    ER = int(rng.integers(1, 5))
    E = R * ER
    S = int(rng.integers(1, 24))
    K = int(rng.integers(1, min(E, 4) + 1))
    bias = rng.normal(0.0, rng.uniform(0.0, 3.0), E).astype(np.float32)
    topk, _ = W.routing_from(R * S, E, K, seed=500 + it, bias_e=bias)
    return R, S, K, E, ER, topk


def pin_quota_invariants(L):
    """What the page states (every rank at or under the threshold, copies only
    with work, a replica budget per rank, local instances first, routing
    unchanged), checked on random routings with numpy doing the counting."""
    rng = np.random.default_rng(32)
    for it in range(80):
        R, S, K, E, ER, topk = _quota_case(rng, it)
        SK, P = S * K, R * S * K
        loads = np.bincount(topk.ravel(), minlength=E).astype(np.int32)
        H = loads.reshape(R, ER).sum(axis=1)
        B = int(rng.integers(0, 4))
        qp = O.quota_plan(loads, R, S, K, E, B, L=L)
        tau, n = qp["tau"], qp["n_rep"]
        re, rr, rc, hq = qp["rep_expert"], qp["rep_rank"], qp["rep_count"], qp["home_quota"]
        assert -(-P // R) <= tau <= max(-(-P // R), int(H.max()))
        assert np.all(rc > 0) and np.all(hq >= 0)
        assert np.all(np.bincount(rr, minlength=R) <= B)
        assert all(H[rr[m]] < tau and H[re[m] // ER] > tau for m in range(n))
        assert np.array_equal(hq + np.bincount(re, weights=rc, minlength=E).astype(np.int64), loads)
        assert O.quota_plan_at(loads, E, R, tau - 1, B, L=L) is None or tau == -(-P // R)
        lo = O.quota_layout(topk, qp, R, S, K, E, L=L)
        pos, src = lo["pos"], lo["src"]
        assert np.array_equal(np.sort(pos), np.arange(P)) and np.array_equal(src[pos], np.arange(P))
        order, cu = lo["slot_order"], lo["cu_seqlens"]
        q = np.diff(cu)
        slot_e = np.where(order < E, order, re[np.maximum(order - E, 0)] if n else order)
        slot_r = np.where(order < E, order // ER, rr[np.maximum(order - E, 0)] if n else order // ER)
        row_slot = np.repeat(np.arange(len(order)), q)
        assert np.array_equal(slot_e[row_slot[pos]], topk.ravel())  # routing unchanged
        row_rank = slot_r[row_slot]
        assert np.all(np.diff(row_rank) >= 0)  # ranks in order
        assert np.array_equal(np.bincount(row_rank, minlength=R), lo["rank_load"])
        assert np.all(lo["rank_load"] <= tau) and lo["rank_load"].sum() == P
        for r in range(R):  # home experts by id, then received replicas by match order
            mine = order[slot_r == r]
            homes = mine[mine < E]
            assert homes.tolist() == list(range(r * ER, (r + 1) * ER))
            assert mine[ER:].tolist() == sorted(mine[ER:].tolist()) and np.all(mine[ER:] >= E)
        Lm = np.zeros((R, E), dtype=np.int64)
        np.add.at(Lm, (np.arange(P) // SK, topk.ravel()), 1)
        want_local = 0
        for i, sid in enumerate(order):
            ps = src[cu[i]:cu[i + 1]]
            e, r = slot_e[i], slot_r[i]
            nloc = int(min(q[i], Lm[r, e]))
            want_local += nloc
            assert np.all(ps[:nloc] // SK == r)  # local pairs first
            assert np.all(np.diff(ps[:nloc]) > 0) and np.all(np.diff(ps[nloc:]) > 0)
        assert lo["n_local"] == want_local == int(np.sum(row_rank[pos] == np.arange(P) // SK))
        for e in range(E):  # the looked-up pairs of e, instance after instance, are e's other pairs in order
            inst = [i for i in range(len(order)) if slot_e[i] == e]
            inst.sort(key=lambda i: (order[i] >= E, order[i]))
            rest = np.concatenate([src[cu[i] + int(min(q[i], Lm[slot_r[i], e])):cu[i + 1]] for i in inst])
            local = set(np.concatenate([src[cu[i]:cu[i] + int(min(q[i], Lm[slot_r[i], e]))] for i in inst]).tolist())
            mine = [p for p in np.flatnonzero(topk.ravel() == e).tolist() if p not in local]
            assert rest.tolist() == mine


def unit_quota_plan(loads, R, E, tau, B):
    """Independent statement of the quota rule at threshold tau, one pair at a
    time: every rank above tau lists its excess pairs (ranks ascending; within a
    rank its home experts heaviest first, ties to the lower id, each giving up to
    what is still in excess); the ranks below tau are rooms (ascending) of
    tau - H_r pairs and at most B pieces.  Each pair goes to the current room;
    a pair that would open a new piece (another expert's chunk, or a new room)
    moves on to the next room when the current one is full or holds B pieces.
    Returns [expert, room rank, pairs] per piece in walk order, or None when
    the rooms run out first."""
    ER = E // R
    H = [int(sum(int(loads[e]) for e in range(r * ER, (r + 1) * ER))) for r in range(R)]
    units = []  # (chunk id, expert)
    for r in range(R):
        rem = H[r] - tau
        if rem <= 0:
            continue
        for e in sorted(range(r * ER, (r + 1) * ER), key=lambda x: (-int(loads[x]), x)):
            take = min(int(loads[e]), rem)
            units += [((r, e), e)] * take
            rem -= take
            if rem == 0:
                break
    rooms = [r for r in range(R) if H[r] < tau]
    j, left, pieces, reps, last = 0, (tau - H[rooms[0]] if rooms else 0), 0, [], None
    for chunk, e in units:
        new_piece = last != (chunk, j)
        while j < len(rooms) and (left == 0 or (new_piece and pieces == B)):
            j += 1
            left = tau - H[rooms[j]] if j < len(rooms) else 0
            pieces, new_piece = 0, True
        if j >= len(rooms):
            return None
        if new_piece:
            reps.append([e, rooms[j], 0])
            pieces += 1
        reps[-1][2] += 1
        left -= 1
        last = (chunk, j)
    return reps


def pin_quota_unit_restatement(L):
    """The oracle's threshold and plan against unit_quota_plan: tau* is the
    smallest tau from ceil(P/R) up at which every excess pair finds a room
    (the largest H_r always does), and the replicas, in match order, and the
    home quotas are those of the pair-by-pair walk at tau*."""
    rng = np.random.default_rng(34)
    for it in range(400):
        R = int(rng.choice([1, 2, 3, 4, 5, 8]))
        ER = int(rng.integers(1, 6))
        E = R * ER
        SK = int(rng.integers(1, 30))
        loads = _rand_loads(rng, R, ER, SK) if it % 2 else rng.multinomial(
            R * SK, rng.dirichlet(np.full(E, rng.uniform(0.1, 3.0)))).astype(np.int32)
        P = R * SK
        B = int(rng.choice([0, 1, 2, 3, E]))
        H = loads.reshape(R, ER).sum(axis=1)
        lo, hi = -(-P // R), max(-(-P // R), int(H.max()))
        want_tau = next(t for t in range(lo, hi + 1) if t == hi or unit_quota_plan(loads, R, E, t, B) is not None)
        qp = O.quota_plan(loads, R, SK, 1, E, B, L=L)
        assert qp["tau"] == want_tau, (loads.tolist(), R, B, qp["tau"], want_tau)
        want = unit_quota_plan(loads, R, E, want_tau, B) or []
        got = [[int(a), int(b), int(c)] for a, b, c in zip(qp["rep_expert"], qp["rep_rank"], qp["rep_count"])]
        assert got == want, (loads.tolist(), R, B, want_tau, got, want)
        hq = loads.astype(np.int64).copy()
        for e, _, c in want:
            hq[e] -= c
        assert qp["home_quota"].tolist() == hq.tolist()


def pin_quota_no_replica_is_a_sort(L):
    """B = 0: no copy, so the layout is a stable sort by (expert, pair not from
    the expert's home rank) -- numpy's lexsort."""
    rng = np.random.default_rng(33)
    for it in range(40):
        R, S, K, E, ER, topk = _quota_case(rng, 100 + it)
        SK, P = S * K, R * S * K
        loads = np.bincount(topk.ravel(), minlength=E).astype(np.int32)
        qp = O.quota_plan(loads, R, S, K, E, 0, L=L)
        assert qp["n_rep"] == 0
        lo = O.quota_layout(topk, qp, R, S, K, E, L=L)
        e = topk.ravel()
        p = np.arange(P)
        order = np.lexsort((p, (p // SK) != (e // ER), e))
        want = np.empty(P, dtype=np.int64)
        want[order] = p
        assert np.array_equal(lo["pos"], want)


ALL_PINS = [pin_hand_example, pin_max_vio_closed_forms, pin_plan_unit_restatement, pin_layout_brute_force,
            pin_layout_library_reductions, pin_layout_invariants, pin_align_sort, pin_dispatch, pin_combine,
            pin_grad_reduce, pin_dispatch_backward, pin_combine_backward, pin_prefetch_slots, pin_quota_hand_example,
            pin_quota_threshold_closed_forms, pin_quota_invariants, pin_quota_no_replica_is_a_sort,
            pin_quota_unit_restatement]
