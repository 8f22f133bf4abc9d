"""Discrete-event model of the backward key-tile kernel's barrier protocol
(csrc/bwd_sm100.cu, `bwd_main_kernel`): one CTA (one key tile) walking its query tiles,
with its TMA producer (K and V once; Q with its lse2 / D vectors and dO through two-stage
rings), the MMA issuer, the two compute warpgroups and the dQ drain warpgroup, the in-order
tensor pipe with its commits, and TMA loads that land in any order.

Waits have the hardware's semantics (a wait for phase k returns when the current phase's
parity differs from k's), the scheduler picks a random ready actor at each step, and a run
fails on a deadlock, a wait returning before its phase completed, or a data hazard: a
product reading a tile that is not loaded or a TMEM / shared-memory region that is not yet
written, a product overwriting a region (S^T/P^T columns, dP^T/dQ columns, the dS^T tile)
that is still to be read, a load overwriting a Q / dO stage (or its lse2 / D vectors) still
in use, the drain reading dQ before its product ended, or the epilogue reading dK / dV
early.  The roles follow the kernel's code step by step (names as in the kernel).  Test
infrastructure only.
"""
import random


class Deadlock(Exception):
    pass


class Hazard(Exception):
    pass


def run(nq, seed, with_dq=True, max_steps=200000):
    """One CTA with `nq` query tiles.  Returns "ok" or raises Deadlock / Hazard."""
    rng = random.Random(seed)
    done = {}
    pipe = []          # in-order tensor pipe: (kind, n) or ("C", barrier)
    tma = []           # pending loads: (barrier, kind, n)
    st = {
        "kv": False, "q_loaded": {}, "do_loaded": {},
        "exec": {k: 0 for k in ("S", "dP", "dV", "dQ", "dK")},   # products executed
        "issued": {k: 0 for k in ("S", "dP", "dV", "dQ", "dK")},
        "p_pub": 0, "ds_pub": 0,       # steps whose P^T / dS^T both warpgroups have written
        "p_half": [0, 0], "ds_half": [0, 0],
        "s_read": [0, 0], "dp_read": [0, 0], "vec_read": [0, 0],
        "dq_read": 0,
    }

    def completed(bar):
        return done.get(bar, 0)

    def complete(bar):
        done[bar] = completed(bar) + 1

    def commit(bar):
        pipe.append(("C", bar))

    def issue(kind, n):
        st["issued"][kind] += 1
        pipe.append((kind, n))

    # ---------------------------------------------------------------- roles
    def loader():
        tma.append(("kv_full", "KV", 0))
        for n in range(nq):
            sq = n % 2
            if n >= 2:
                yield ("wait", f"q_empty{sq}", n // 2 - 1)
                # The stage's Q and vectors of step n-2 must be done with.
                if st["exec"]["S"] < n - 1 or st["exec"]["dK"] < n - 1:
                    raise Hazard(f"Q stage {sq} reloaded while products of step {n - 2} read it")
                if min(st["vec_read"]) < n - 1:
                    raise Hazard(f"lse2/D of step {n - 2} overwritten while still read")
            tma.append((f"q_full{sq}", "Q", n))
            sd = n % 2
            if n >= 2:
                yield ("wait", f"do_empty{sd}", n // 2 - 1)
                if st["exec"]["dP"] < n - 1 or st["exec"]["dV"] < n - 1:
                    raise Hazard(f"dO stage {sd} reloaded while products of step {n - 2} read it")
            tma.append((f"do_full{sd}", "dO", n))

    def mma():
        def issue_s(n):
            yield ("wait", f"q_full{n % 2}", n // 2)
            if not st["kv"] or not st["q_loaded"].get(n):
                raise Hazard(f"S^T_{n} issued before K / Q_{n} landed")
            # S^T columns hold P^T_{n-1}: dV_{n-1} must be issued before (pipe order), and
            # both warpgroups must be done reading S^T_{n-1}.
            if st["issued"]["dV"] < n:
                raise Hazard(f"S^T_{n} issued over P^T_{n - 1} before dV read it")
            issue("S", n)
            commit("s_full")

        def issue_dp(n):
            yield ("wait", f"do_full{n % 2}", n // 2)
            if with_dq and n > 0:
                yield ("wait", "dq_empty", n - 1)
            if with_dq and st["dq_read"] < n:
                raise Hazard(f"dP^T_{n} issued over dQ_{n - 1} before the drain read it")
            if not st["do_loaded"].get(n):
                raise Hazard(f"dP^T_{n} issued before dO_{n} landed")
            if n > 0 and min(st["dp_read"]) < n:
                raise Hazard(f"dP^T_{n} issued over dP^T_{n - 1} still being read")
            issue("dP", n)
            commit("dp_full")

        yield ("wait", "kv_full", 0)
        yield from issue_s(0)
        yield from issue_dp(0)
        for n in range(nq):
            yield ("wait", "p_ready", n)
            if st["p_pub"] < n + 1:
                raise Hazard(f"dV_{n} issued before P^T_{n} was written")
            issue("dV", n)
            commit(f"do_empty{n % 2}")
            if n + 1 < nq:
                yield from issue_s(n + 1)
            yield ("wait", "ds_ready", n)
            if st["ds_pub"] < n + 1:
                raise Hazard(f"dQ/dK_{n} issued before dS^T_{n} was written")
            if with_dq:
                issue("dQ", n)
                commit("dq_full")
            issue("dK", n)
            commit(f"q_empty{n % 2}")
            if n + 1 < nq:
                yield from issue_dp(n + 1)
        commit("dkdv_done")

    def compute(half):
        for n in range(nq):
            yield ("wait", "s_full", n)
            yield ("wait", f"q_full{n % 2}", n // 2)
            if st["exec"]["S"] < n + 1:
                raise Hazard(f"warpgroup {half} read S^T_{n} before it was computed")
            if not st["q_loaded"].get(n):
                raise Hazard(f"warpgroup {half} read lse2_{n} before it landed")
            st["s_read"][half] += 1
            # P^T written over this half's S^T columns
            st["p_half"][half] += 1
            if min(st["p_half"]) == n + 1:
                st["p_pub"] = n + 1
            complete("p_ready_arrive")
            if completed("p_ready_arrive") % 2 == 0:
                complete("p_ready")
            yield ("step",)
            yield ("wait", "dp_full", n)
            if st["exec"]["dP"] < n + 1:
                raise Hazard(f"warpgroup {half} read dP^T_{n} before it was computed")
            # dS^T_n into the shared tile: dQ_{n-1} and dK_{n-1} must have read dS^T_{n-1}
            if n > 0 and (st["exec"]["dK"] < n or (with_dq and st["exec"]["dQ"] < n)):
                raise Hazard(f"warpgroup {half} overwrote dS^T_{n - 1} still being read")
            st["dp_read"][half] += 1
            st["vec_read"][half] += 1
            st["ds_half"][half] += 1
            if min(st["ds_half"]) == n + 1:
                st["ds_pub"] = n + 1
            complete("ds_ready_arrive")
            if completed("ds_ready_arrive") % 2 == 0:
                complete("ds_ready")
        yield ("wait", "dkdv_done", 0)
        if st["exec"]["dK"] < nq or st["exec"]["dV"] < nq:
            raise Hazard("dK / dV read before their last products ended")

    def drain():
        for n in range(nq if with_dq else 0):
            yield ("wait", "dq_full", n)
            if st["exec"]["dQ"] < n + 1:
                raise Hazard(f"drain read dQ_{n} before it was computed")
            st["dq_read"] += 1
            complete("dq_empty")

    roles = {"load": loader(), "mma": mma(), "c0": compute(0), "c1": compute(1),
             "drain": drain()}
    pending = {r: None for r in roles}
    finished = set()

    def parity_ok(bar, k):
        return (completed(bar) - k) % 2 == 1

    for _ in range(max_steps):
        ready = [r for r in roles if r not in finished
                 and (pending[r] is None or parity_ok(pending[r][1], pending[r][2]))]
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
                st["exec"][op[0]] += 1
            continue
        if c == "tma":
            bar, kind, n = tma.pop(rng.randrange(len(tma)))
            if kind == "KV":
                st["kv"] = True
            elif kind == "Q":
                st["q_loaded"][n] = True
                st["q_loaded"].pop(n - 2, None)
            else:
                st["do_loaded"][n] = True
                st["do_loaded"].pop(n - 2, None)
            complete(bar)
            continue
        w = pending[c]
        if w is not None and completed(w[1]) < w[2] + 1:
            raise Hazard(f"{c}: wait on {w[1]} phase {w[2]} returned early "
                         f"(completed {completed(w[1])})")
        try:
            req = next(roles[c])
            pending[c] = None if req[0] == "step" else req
        except StopIteration:
            finished.add(c)
            pending[c] = None
    raise RuntimeError("step limit")
