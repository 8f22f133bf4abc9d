"""Discrete-event model of the split-KV decoding kernel's barrier protocol
(csrc/fwd_splitkv_sm100.cu): one CTA (one query tile, one key slice of `nkv` tiles) with its
TMA producer (Q once; K and V through a ring), the MMA issuer (S two tiles ahead in two
TMEM buffers, PV after each P), the softmax warps (which wait for the previous PV only on
the steps where they rescale O) and the in-order tensor pipe with its commits.

Waits have the hardware's parity semantics, the scheduler picks a random ready actor at
each step, and a run fails on a deadlock, a wait returning before its phase completed, or a
data hazard: S or PV on a tile that is not loaded, S over a buffer whose P no PV has read,
P read before published, a rescale of O while a PV into it runs, a ring slot reloaded while
a product still reads it, or O read before its products ended.  Test infrastructure only.
"""
import random


class Deadlock(Exception):
    pass


class Hazard(Exception):
    pass


def run(nkv, seed, stages=3, need_prob=0.3, max_steps=100000):
    """`nkv` key tiles in the slice; `need_prob` is the chance that a softmax step rescales
    O (the kernel does so when a row maximum jumps).  Returns "ok" or raises."""
    rng = random.Random(seed)
    done = {}
    pipe, tma = [], []
    st = {"q": False, "k": {}, "v": {}, "exec_s": 0, "exec_pv": 0, "iss_pv": 0, "p_pub": 0}

    def completed(bar):
        return done.get(bar, 0)

    def complete(bar):
        done[bar] = completed(bar) + 1

    def loader():
        tma.append(("q_full", "Q", 0))
        for n in range(nkv):
            s = n % stages
            if n >= stages:
                yield ("wait", f"kv_empty{s}", n // stages - 1)
                if st["exec_s"] < n - stages + 1 or st["exec_pv"] < n - stages + 1:
                    raise Hazard(f"ring slot {s} reloaded while tile {n - stages} is read")
            tma.append((f"k_full{s}", "K", n))
            tma.append((f"v_full{s}", "V", n))

    def mma():
        def issue_s(n):
            s = n % stages
            yield ("wait", f"k_full{s}", n // stages)
            if not st["q"] or not st["k"].get(n):
                raise Hazard(f"S_{n} issued before Q / K_{n} landed")
            if st["iss_pv"] < n - 1:
                raise Hazard(f"S_{n} issued over P_{n - 2} before its PV")
            pipe.append(("S", n))
            pipe.append(("C", f"s_full{n & 1}"))

        yield ("wait", "q_full", 0)
        yield from issue_s(0)
        for n in range(nkv):
            if n + 1 < nkv:
                yield from issue_s(n + 1)
            s = n % stages
            yield ("wait", f"p_full{n & 1}", n >> 1)
            yield ("wait", f"v_full{s}", n // stages)
            if st["p_pub"] < n + 1:
                raise Hazard(f"PV_{n} issued before P_{n} was published")
            if not st["v"].get(n):
                raise Hazard(f"PV_{n} issued before V_{n} landed")
            st["iss_pv"] += 1
            pipe.append(("PV", n))
            pipe.append(("C", f"kv_empty{s}"))
            pipe.append(("C", "pv_done"))
        pipe.append(("C", "o_done"))

    def softmax():
        for n in range(nkv):
            yield ("wait", f"s_full{n & 1}", n >> 1)
            if st["exec_s"] < n + 1:
                raise Hazard(f"softmax read S_{n} before it was computed")
            if n > 0 and rng.random() < need_prob:
                yield ("wait", "pv_done", n - 1)
                if st["exec_pv"] < n:
                    raise Hazard(f"O rescaled while PV_{n - 1} runs")
            st["p_pub"] += 1
            complete(f"p_full{n & 1}")
        if nkv > 0:
            yield ("wait", "o_done", 0)
            if st["exec_pv"] < nkv:
                raise Hazard("O read before its last PV ended")

    roles = {"load": loader(), "mma": mma(), "sm": softmax()} if nkv > 0 else {"sm": softmax()}
    pending = {r: None for r in roles}
    finished = set()
    for _ in range(max_steps):
        ready = [r for r in roles if r not in finished and (
            pending[r] is None or (completed(pending[r][1]) - pending[r][2]) % 2 == 1)]
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
            elif op[0] == "S":
                st["exec_s"] += 1
            else:
                st["exec_pv"] += 1
            continue
        if c == "tma":
            bar, kind, n = tma.pop(rng.randrange(len(tma)))
            if kind == "Q":
                st["q"] = True
            else:
                st[kind.lower()][n] = True
                st[kind.lower()].pop(n - stages, None)
            complete(bar)
            continue
        w = pending[c]
        if w is not None and completed(w[1]) < w[2] + 1:
            raise Hazard(f"{c}: wait on {w[1]} phase {w[2]} returned early "
                         f"(completed {completed(w[1])})")
        try:
            pending[c] = next(roles[c])
        except StopIteration:
            finished.add(c)
            pending[c] = None
    raise RuntimeError("step limit")
