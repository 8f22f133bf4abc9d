"""Discrete-event model of the forward kernel's barrier protocol (csrc/fwd_sm100.cu): one
persistent CTA working through several units, its TMA producer, MMA issuer (dense and
block-sparse issue orders) and two softmax warpgroups, the in-order tensor pipe with its
commits, and TMA loads that land in any order.  In the block-sparse mode a unit is one query
tile whose active key tiles alternate between the two slots, and warpgroup 0 merges both
slots' results (merge_ready / merge_free with warpgroup 1, o_done and o_free of both slots).

Waits have the hardware's semantics: a wait for phase k of an mbarrier returns when the
current phase's parity differs from k's, so a barrier that completes two phases before a
waiter polls it looks unchanged, and one that is two phases behind looks complete.  The
scheduler picks a random ready actor at each step (the slowest-poller worst case), and the
run fails on a deadlock, on a wait that returns before its phase completed, or on a data
hazard: a product reading a K/V/Q tile that is not loaded, a load overwriting a tile that a
pending product still reads, P read before it was published, S read before it was
computed, an S product issued over a P (same TMEM columns) that no PV has read yet, a
softmax step (which may rescale O) while the previous PV of its tile still runs, O
overwritten before its epilogue read it, or O read before its products ended.

The roles follow the kernel's issue logic step by step (names as in the kernel), so a
change to the kernel's barrier protocol must be mirrored here.  Test infrastructure only.
"""
import random


class Deadlock(Exception):
    pass


class Hazard(Exception):
    pass


class Sim:
    def __init__(self, rng):
        self.rng = rng
        self.done = {}        # barrier -> completed phases
        self.pipe = []        # in-order tensor pipe: ("S", t, pos, unit) / ("PV", ...) / ("C", bar)
        self.tma = []         # pending loads: (bar, kind, pos)
        # data state
        self.k_loaded = {}    # ring pos -> loaded
        self.v_loaded = {}
        self.k_reads_pending = {}  # ring pos -> number of S products not yet executed
        self.v_reads_pending = {}
        self.q_unit = -1
        self.q_reads_pending = 0
        self.s_done = [0, 0]   # S products executed per tile
        self.p_pub = [0, 0]    # P published per tile
        self.pv_done = [0, 0]  # PV executed per tile
        self.pv_issued = [0, 0]
        self.p_half_pub = [0, 0]
        self.s_issued = [0, 0]
        self.o_read_units = [0, 0]   # epilogues done per tile
        self.merge_pub = 0           # block-sparse: units whose slot-1 values are published
        self.merge_read = 0          # ... and read by warpgroup 0
        self.o_unit_pv = [{}, {}]    # unit -> PVs executed

    def completed(self, bar):
        return self.done.get(bar, 0)

    def complete(self, bar):
        self.done[bar] = self.completed(bar) + 1

    def parity_ok(self, bar, k):
        # Hardware: the wait returns iff the current phase's parity differs from k's.
        return (self.completed(bar) - k) % 2 == 1

    def truly_ok(self, bar, k):
        return self.completed(bar) >= k + 1


def run(mode, masks0, masks1, nkv_list, seed, stages=4, empty_tile_waits_o_free=True,
        split_p=False, max_steps=200000):
    """mode 'dense' (nkv_list: (nkv0, nkv1) per unit) or 'sparse' (masks0: the unit's query
    tile's sorted active key tiles, per unit; masks1 unused).  `stages` is the K/V ring depth
    (2 at head dim 128, 4 at 64).  `empty_tile_waits_o_free=False` signals an empty slot's O
    without waiting for o_free (the race the kernel avoids).
    `split_p` (dense only): P is published in two halves (p_half, then p_full) and each half
    of PV is issued after its half, as on the 8-bit path.
    Returns "ok" or raises Deadlock / Hazard."""
    S_STAGES = stages
    # Block-sparse units hold one query tile, and the kernel turns the second Q slot into one
    # more K stage: K runs stages + 1 deep, V stages deep.
    KS = stages + 1 if mode == "sparse" else stages
    VS = stages
    rng = random.Random(seed)
    sim = Sim(rng)
    units = len(nkv_list) if mode == "dense" else len(masks0)

    def tile_lists(u):
        if mode == "dense":
            n0, n1 = nkv_list[u]
            return list(range(n0)), list(range(n1))
        lst = list(masks0[u])
        return lst[0::2], lst[1::2]   # the slots' key tiles

    # ------------------------------------------------------------------ roles
    def loader():
        g = 0
        for u in range(units):
            if u > 0:
                yield ("wait", "q_empty", u - 1)
            if sim.q_reads_pending:
                raise Hazard("Q overwritten while S products still read it")
            sim.tma.append(("q_full", "Q", u))
            l0, l1 = tile_lists(u)
            for j in (sorted(set(l0) | set(l1)) if mode == "dense" else masks0[u]):
                s = g % KS
                if g >= KS:
                    yield ("wait", f"k_empty{s}", g // KS - 1)
                old = g - KS
                if old >= 0 and sim.k_reads_pending.get(old, 0):
                    raise Hazard(f"K slot {s} reloaded while pos {old} still read")
                sim.tma.append((f"k_full{s}", "K", g))
                sv = g % VS
                if g >= VS:
                    yield ("wait", f"v_empty{sv}", g // VS - 1)
                old = g - VS
                if old >= 0 and sim.v_reads_pending.get(old, 0):
                    raise Hazard(f"V slot {sv} reloaded while pos {old} still read")
                sim.tma.append((f"v_full{sv}", "V", g))
                g += 1

    def issue_s(t, pos, u):
        # S_t shares its TMEM columns with P_t: every earlier P_t must already be read by an
        # issued PV (the pipe runs in issue order).
        if sim.pv_issued[t] < sim.s_issued[t]:
            raise Hazard(f"S{t} issued over a P{t} that no PV has read yet")
        sim.s_issued[t] += 1
        if not sim.k_loaded.get(pos):
            raise Hazard(f"S{t} issued on K pos {pos} not loaded")
        if sim.q_unit != u:
            raise Hazard(f"S{t} of unit {u} issued with Q of unit {sim.q_unit}")
        sim.k_reads_pending[pos] = sim.k_reads_pending.get(pos, 0) + 1
        sim.q_reads_pending += 1
        sim.pipe.append(("S", t, pos, u))
        sim.pipe.append(("C", f"s_full{t}"))

    def issue_pv(t, pos, u, first):
        if not sim.v_loaded.get(pos):
            raise Hazard(f"PV{t} issued on V pos {pos} not loaded")
        if sim.p_pub[t] <= sim.pv_issued[t]:
            raise Hazard(f"PV{t} issued before its P was published")
        if first and sim.o_read_units[t] < u:
            raise Hazard(f"PV{t} overwrites O of unit {u - 1} before its epilogue")
        sim.pv_issued[t] += 1
        sim.v_reads_pending[pos] = sim.v_reads_pending.get(pos, 0) + 1
        sim.pipe.append(("PV", t, pos, u))

    def commit(bar):
        sim.pipe.append(("C", bar))

    def mma_dense():
        g = 0
        np_ = [0, 0]
        for u in range(units):
            n0, n1 = nkv_list[u]
            yield ("wait", "q_full", u)
            s = g % S_STAGES
            yield ("wait", f"k_full{s}", g // S_STAGES)
            issue_s(0, g, u)
            issue_s(1, g, u)
            commit(f"k_empty{s}")
            if n1 == 1:
                commit("q_empty")
            for j in range(n1):
                s = (g + j) % S_STAGES
                s1 = (g + j + 1) % S_STAGES
                more = j + 1 < n1
                yield ("wait", f"v_full{s}", (g + j) // S_STAGES)
                if more:
                    yield ("wait", f"k_full{s1}", (g + j + 1) // S_STAGES)
                if j < n0:
                    if j == 0 and u > 0:
                        yield ("wait", "o_free0", u - 1)
                    if split_p:
                        yield ("wait", "p_half0", np_[0])
                        if sim.p_half_pub[0] <= sim.pv_issued[0]:
                            raise Hazard("first half of PV0 issued before its half of P")
                    yield ("wait", "p_full0", np_[0])
                    issue_pv(0, g + j, u, j == 0)
                    np_[0] += 1
                    if j + 1 < n0:
                        issue_s(0, g + j + 1, u)
                    else:
                        commit("o_done0")
                if j == 0 and u > 0:
                    yield ("wait", "o_free1", u - 1)
                if split_p:
                    yield ("wait", "p_half1", np_[1])
                    if sim.p_half_pub[1] <= sim.pv_issued[1]:
                        raise Hazard("first half of PV1 issued before its half of P")
                yield ("wait", "p_full1", np_[1])
                issue_pv(1, g + j, u, j == 0)
                np_[1] += 1
                commit(f"v_empty{s}")
                if more:
                    issue_s(1, g + j + 1, u)
                    commit(f"k_empty{s1}")
                    if j + 2 == n1:
                        commit("q_empty")
                else:
                    commit("o_done1")
            g += n1

    def mma_sparse():
        g = 0
        np_ = [0, 0]
        for u in range(units):
            cnt = len(masks0[u])
            yield ("wait", "q_full", u)
            for t in (0, 1):
                if cnt <= t:
                    if empty_tile_waits_o_free and u > 0:
                        yield ("wait", f"o_free{t}", u - 1)
                    commit(f"o_done{t}")
            if cnt == 0:
                commit("q_empty")

            def issue_s_at(k):
                pos = g + k
                s = pos % KS
                yield ("wait", f"k_full{s}", pos // KS)
                issue_s(k & 1, pos, u)
                commit(f"k_empty{s}")
                if k == cnt - 1:
                    commit("q_empty")
            if cnt >= 1:
                yield from issue_s_at(0)
            if cnt >= 2:
                yield from issue_s_at(1)
            for k in range(cnt):
                t = k & 1
                pos = g + k
                s = pos % VS
                yield ("wait", f"v_full{s}", pos // VS)
                if k < 2 and u > 0:
                    yield ("wait", f"o_free{t}", u - 1)
                yield ("wait", f"p_full{t}", np_[t])
                issue_pv(t, pos, u, k < 2)
                np_[t] += 1
                commit(f"v_empty{s}")
                if k + 2 < cnt:
                    yield from issue_s_at(k + 2)
                else:
                    commit(f"o_done{t}")
            g += cnt

    def softmax(t):
        ns = 0
        for u in range(units):
            lst = tile_lists(u)[t]
            for _ in lst:
                yield ("wait", f"s_full{t}", ns)
                ns += 1
                if sim.s_done[t] < ns:
                    raise Hazard(f"softmax{t} read S before it was computed")
                # A step may rescale O in place: the previous step's PV must have landed.
                if sim.pv_done[t] < ns - 1:
                    raise Hazard(f"softmax{t} may rescale O while PV{t} of its last step runs")
                # P overwrites S in place; publish (in two halves on the split path)
                if split_p:
                    sim.p_half_pub[t] += 1
                    sim.complete(f"p_half{t}")
                    yield ("step",)
                sim.p_pub[t] += 1
                sim.complete(f"p_full{t}")
            if mode == "dense":
                yield ("wait", f"o_done{t}", u)
                if sim.o_unit_pv[t].get(u, 0) != len(lst):
                    raise Hazard(f"softmax{t} read O of unit {u} before its PVs finished")
                sim.o_read_units[t] += 1
                sim.complete(f"o_free{t}")
            elif t == 1:
                # publish this slot's max and sum for the merge
                if u > 0:
                    yield ("wait", "merge_free", u - 1)
                if sim.merge_read < u:
                    raise Hazard(f"warpgroup 1 overwrote the merge values of unit {u - 1} unread")
                sim.merge_pub = u + 1
                sim.complete("merge_ready")
            else:
                # warpgroup 0 merges both slots' O and hands both back
                lists = tile_lists(u)
                yield ("wait", "o_done0", u)
                yield ("wait", "o_done1", u)
                yield ("wait", "merge_ready", u)
                for tt in (0, 1):
                    if sim.o_unit_pv[tt].get(u, 0) != len(lists[tt]):
                        raise Hazard(f"merge read O{tt} of unit {u} before its PVs finished")
                if sim.merge_pub < u + 1:
                    raise Hazard(f"merge read warpgroup 1's values of unit {u} unpublished")
                sim.merge_read = u + 1
                sim.complete("merge_free")
                for tt in (0, 1):
                    sim.o_read_units[tt] += 1
                    sim.complete(f"o_free{tt}")

    # ------------------------------------------------------------------ scheduler
    roles = {"load": loader(), "mma": mma_dense() if mode == "dense" else mma_sparse(),
             "sm0": softmax(0), "sm1": softmax(1)}
    pending = {r: None for r in roles}   # current wait request
    finished = set()

    def step_pipe():
        op = sim.pipe.pop(0)
        if op[0] == "S":
            _, t, pos, u = op
            sim.s_done[t] += 1
            sim.k_reads_pending[pos] -= 1
            sim.q_reads_pending -= 1
        elif op[0] == "PV":
            _, t, pos, u = op
            sim.pv_done[t] += 1
            sim.v_reads_pending[pos] -= 1
            sim.o_unit_pv[t][u] = sim.o_unit_pv[t].get(u, 0) + 1
        else:
            sim.complete(op[1])

    def step_tma():
        i = rng.randrange(len(sim.tma))
        bar, kind, pos = sim.tma.pop(i)
        if kind == "K":
            sim.k_loaded[pos] = True
        elif kind == "V":
            sim.v_loaded[pos] = True
        else:
            sim.q_unit = pos
        sim.complete(bar)

    for _ in range(max_steps):
        ready = []
        for r, gen in roles.items():
            if r in finished:
                continue
            w = pending[r]
            if w is None or sim.parity_ok(w[1], w[2]):
                ready.append(r)
        choices = ready + (["pipe"] if sim.pipe else []) + (["tma"] if sim.tma else [])
        if not choices:
            if len(finished) == len(roles):
                return "ok"
            raise Deadlock({r: pending[r] for r in roles if r not in finished})
        c = rng.choice(choices)
        if c == "pipe":
            step_pipe()
            continue
        if c == "tma":
            step_tma()
            continue
        w = pending[c]
        if w is not None and not sim.truly_ok(w[1], w[2]):
            raise Hazard(f"{c}: wait on {w[1]} phase {w[2]} returned early (parity alias; "
                         f"completed {sim.completed(w[1])})")
        try:
            req = next(roles[c])
            pending[c] = None if req[0] == "step" else req
        except StopIteration:
            finished.add(c)
            pending[c] = None
    raise RuntimeError("step limit")


def random_masks(rng, units, nt, causal, density):
    """Block-sparse units: per unit, one query tile's sorted active key tiles."""
    out = []
    for u in range(units):
        qt = rng.randrange(max(1, nt))
        vis = range(nt) if not causal else range(min(nt, qt + 1))
        out.append(sorted(j for j in vis if rng.random() < density))
    return out
