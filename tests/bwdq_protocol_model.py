"""Discrete-event model of the deterministic dQ kernel's barrier protocol
(csrc/bwd_dq_sm100.cu, `bwd_dq_kernel`): one CTA (one query tile) walking its key tiles,
with its TMA producer (Q and dO once; K through a three-stage ring, V through a two-stage
ring), the MMA issuer (prologue S(0), dP(0), S(1); then per key tile [ds_ready j] dP(j+1),
dQ(j), S(j+2)), the compute warps, the in-order tensor pipe with its commits, and TMA loads
that land in any order.  S has two TMEM buffers (tile j uses j % 2), each with its own
s_full barrier.

Waits have the hardware's parity semantics, the scheduler picks a random ready actor at each
step, and a run fails on a deadlock, a wait that returns before its phase completed, or a data
hazard: a product reading a K / V / Q / dO tile that is not loaded, a load overwriting a tile a
pending product reads, an S product overwriting a buffer whose dS has not been read by its dQ,
a dP product overwriting dP before the compute warps read it, the compute warps reading S or dP
before they were computed, dQ reading dS before it was written, or the epilogue reading dQ
early.  Test infrastructure only.
"""
import random


class Deadlock(Exception):
    pass


class Hazard(Exception):
    pass


def run(nkv, seed, kstages=3, vstages=2, max_steps=200000):
    rng = random.Random(seed)
    done = {}
    pipe, tma = [], []
    st = {"qd": False, "k": {}, "v": {}, "k_pending": {}, "v_pending": {},
          "exec": {"S": 0, "dP": 0, "dQ": 0}, "issued": {"S": 0, "dP": 0, "dQ": 0},
          "ds_written": 0, "dp_read": 0, "s_read": 0}

    def completed(bar):
        return done.get(bar, 0)

    def complete(bar):
        done[bar] = completed(bar) + 1

    def loader():
        tma.append(("qd_full", "QD", 0))
        for j in range(nkv):
            sk, sv = j % kstages, j % vstages
            if j >= kstages:
                yield ("wait", f"k_empty{sk}", j // kstages - 1)
                if st["k_pending"].get(j - kstages, 0):
                    raise Hazard(f"K stage {sk} reloaded while tile {j - kstages} is read")
            tma.append((f"k_full{sk}", "K", j))
            if j >= vstages:
                yield ("wait", f"v_empty{sv}", j // vstages - 1)
                if st["v_pending"].get(j - vstages, 0):
                    raise Hazard(f"V stage {sv} reloaded while tile {j - vstages} is read")
            tma.append((f"v_full{sv}", "V", j))

    def mma():
        def issue_s(j):
            yield ("wait", f"k_full{j % kstages}", j // kstages)
            if not st["k"].get(j) or not st["qd"]:
                raise Hazard(f"S({j}) issued before K_{j} / Q landed")
            # buffer j % 2 held dS_{j-2}: its dQ must be issued before (pipe order)
            if j >= 2 and st["issued"]["dQ"] < j - 1:
                raise Hazard(f"S({j}) issued over dS_{j - 2} before dQ({j - 2}) read it")
            st["issued"]["S"] += 1
            st["k_pending"][j] = st["k_pending"].get(j, 0) + 1
            pipe.append(("S", j))
            pipe.append(("C", f"s_full{j & 1}"))

        def issue_dp(j):
            yield ("wait", f"v_full{j % vstages}", j // vstages)
            if not st["v"].get(j) or not st["qd"]:
                raise Hazard(f"dP({j}) issued before V_{j} / dO landed")
            if j >= 1 and st["dp_read"] < j:
                raise Hazard(f"dP({j}) issued over dP({j - 1}) still being read")
            st["issued"]["dP"] += 1
            st["v_pending"][j] = st["v_pending"].get(j, 0) + 1
            pipe.append(("dP", j))
            pipe.append(("C", "dp_full"))
            pipe.append(("C", f"v_empty{j % vstages}"))

        yield ("wait", "qd_full", 0)
        yield from issue_s(0)
        yield from issue_dp(0)
        if nkv >= 2:
            yield from issue_s(1)
        for j in range(nkv):
            yield ("wait", "ds_ready", j)
            if st["ds_written"] < j + 1:
                raise Hazard(f"dQ({j}) issued before dS_{j} was written")
            if j + 1 < nkv:
                yield from issue_dp(j + 1)
            st["issued"]["dQ"] += 1
            st["k_pending"][j] = st["k_pending"].get(j, 0) + 1
            pipe.append(("dQ", j))
            pipe.append(("C", f"k_empty{j % kstages}"))
            if j + 2 < nkv:
                yield from issue_s(j + 2)
        pipe.append(("C", "dq_done"))

    def compute():
        for j in range(nkv):
            yield ("wait", f"s_full{j & 1}", j >> 1)
            yield ("wait", "dp_full", j)
            if st["exec"]["S"] < j + 1 or st["exec"]["dP"] < j + 1:
                raise Hazard(f"compute read S / dP of tile {j} before they were computed")
            st["s_read"] += 1
            st["dp_read"] += 1
            st["ds_written"] += 1
            complete("ds_ready")
        yield ("wait", "dq_done", 0)
        if st["exec"]["dQ"] < nkv:
            raise Hazard("epilogue read dQ before its last product ended")

    roles = {"load": loader(), "mma": mma(), "comp": compute()}
    pending = {r: None for r in roles}
    finished = set()
    for _ in range(max_steps):
        ready = [r for r in roles if r not in finished and
                 (pending[r] is None or (completed(pending[r][1]) - pending[r][2]) % 2 == 1)]
        choices = ready + (["pipe"] if pipe else []) + (["tma"] if tma else [])
        if not choices:
            if len(finished) == len(roles):
                return "ok"
            raise Deadlock({r: pending[r] for r in roles if r not in finished})
        c = rng.choice(choices)
        if c == "pipe":
            op = pipe.pop(0)
            if op[0] == "C":
                complete(op[1])
            else:
                kind, j = op
                if kind in ("S", "dQ"):
                    if not st["k"].get(j):
                        raise Hazard(f"{kind}({j}) ran on a K stage that no longer holds K_{j}")
                    st["k_pending"][j] -= 1
                if kind == "dP":
                    if not st["v"].get(j):
                        raise Hazard(f"dP({j}) ran on a V stage that no longer holds V_{j}")
                    st["v_pending"][j] -= 1
                if kind == "dQ" and st["ds_written"] < j + 1:
                    raise Hazard(f"dQ({j}) read dS_{j} before it was written")
                if kind == "S" and j >= 2 and st["exec"]["dQ"] < j - 1:
                    raise Hazard(f"S({j}) overwrote dS_{j - 2} before dQ({j - 2}) ran")
                st["exec"][kind] += 1
            continue
        if c == "tma":
            bar, kind, j = tma.pop(rng.randrange(len(tma)))
            if kind == "QD":
                st["qd"] = True
            elif kind == "K":
                st["k"].pop(j - kstages, None)
                st["k"][j] = True
            else:
                st["v"].pop(j - vstages, None)
                st["v"][j] = True
            complete(bar)
            continue
        w = pending[c]
        if w is not None and completed(w[1]) < w[2] + 1:
            raise Hazard(f"{c}: wait on {w[1]} phase {w[2]} returned early")
        try:
            req = next(roles[c])
            pending[c] = req
        except StopIteration:
            finished.add(c)
            pending[c] = None
    raise RuntimeError("step limit")
