"""A randomised model of the prefill kernel's barrier protocol (one CTA pair of one launch).

Test infrastructure: ``tests/test_prefill_protocol.py`` runs it on the CPU.  It mirrors the
roles of ``rma_prefill.cu`` (the TMA producer of each CTA, the odd CTA's cleaner, the even CTA's
two Q K^T issuers and its P V issuer, the two softmax groups of each CTA, and each CTA's tail)
and the mbarriers they share.  Asynchronous work completes later, in a random order that keeps the
hardware's guarantees: TMA bytes land in any order; the pair's tensor pipe runs its MMAs in issue
order; a tcgen05 commit arrives once every earlier MMA of its issuing thread is done.

What it checks, over many random schedules:
  * every parity wait is sound: it is made while its barrier has completed P or P + 1 phases (a
    barrier two phases ahead would let a parity wait pass on the wrong phase, and one whose phase
    P - 1 is still open would let it pass at once);
  * nothing deadlocks (an abort-aware wait that can never complete is timed out, as the kernel's
    bounded wait would, and its CTA abandons its tile; a drain wait that can never complete is an
    error);
  * when a CTA passes the final cluster barrier (after which it frees tensor memory and reuses its
    stage area), no TMA load into it, no MMA of its pair and no commit into its barriers is still
    in flight.

``abort_rate`` makes random abort-aware waits time out; ``async_bias`` sets how quickly the
asynchronous work completes next to the warps; ``drain`` selects the kernel's drain (waits on the
operations' own barriers) or a fixed delay, which the model shows unsafe once the copies and MMAs
are slow.
"""
import random


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.done = count, 0, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self, n=1, tx=0):
        self.pending -= n
        self.tx += tx
        if self.pending < 0:
            raise Hazard(f"{self.name}: more arrivals than its count in one phase")
        self._check()

    def complete_tx(self, b):
        self.tx -= b
        self._check()


class Hazard(Exception):
    pass


def run(n_chunks, seed, stages=5, abort_rate=0.0, drain=True, async_bias=0.5, max_steps=400000):
    """One launch of one CTA pair over n_chunks chunks (0 = an empty bank).  async_bias is the
    chance that a scheduling step completes pending asynchronous work rather than advancing a role
    (small values make copies and MMAs slow next to the warps)."""
    rng = random.Random(seed)
    E, O = 0, 1
    S = stages
    bar = {}
    for c in (E, O):
        bar[c] = {"Full": [Barrier(f"c{c}.Full{i}", 1) for i in range(S)],
                  "Empty": [Barrier(f"c{c}.Empty{i}", 1) for i in range(S)],
                  "SFull": [Barrier(f"c{c}.SFull{i}", 1) for i in range(2)],
                  "OFinal": Barrier(f"c{c}.OFinal", 1), "Drain": Barrier(f"c{c}.Drain", 3),
                  "Xfer": Barrier(f"c{c}.Xfer", 1)}
    bar[E].update({"Peer": [Barrier(f"E.Peer{i}", 1) for i in range(S)], "QReady": Barrier("E.QReady", 16),
                   "PFull": [Barrier(f"E.PFull{i}", 8) for i in range(2)],
                   "SFree": [Barrier(f"E.SFree{i}", 8) for i in range(2)]})
    abort = {E: False, O: False}
    events = []                 # pending asynchronous completions: (kind, target cta, callable)
    pipe = []                   # the pair's tensor pipe: ("mma", issuer) / ("commit", issuer, fn, targets)
    issued = {E: 0, O: 0}       # chunks whose loads each producer issued
    passed_final = set()
    flags = set()

    def pipe_fire_commits():
        for op in list(pipe):
            if op[0] == "commit" and not any(o[0] == "mma" and o[1] == op[1] for o in pipe[:pipe.index(op)]):
                pipe.remove(op)
                for c in op[3]:
                    if c in passed_final:
                        raise Hazard(f"a commit arrives in CTA {c} after it passed the final barrier")
                op[2]()

    def pipe_step():
        for i, op in enumerate(pipe):
            if op[0] == "mma":
                pipe.pop(i)
                break
        pipe_fire_commits()

    def mma(issuer):
        pipe.append(("mma", issuer))
        events.append(("mma", None, pipe_step))

    def commit(issuer, key, idx=None):
        def fn():
            for c in (E, O):
                (bar[c][key] if idx is None else bar[c][key][idx]).arrive()
        pipe.append(("commit", issuer, fn, (E, O)))
        pipe_fire_commits()

    # a wait is ("wait", cta, barrier, phase, drain?): drain waits ignore the abort flag
    def wait(c, b, phase, is_drain=False):
        return ("wait", c, b, phase, is_drain)

    # ---------------- roles ----------------
    def producer(c):
        ok = True
        for j in range(n_chunks):
            st = j % S
            if j >= S:
                ok = yield wait(c, bar[c]["Empty"][st], j // S - 1)
                if not ok:
                    break
            bar[c]["Full"][st].arrive(1, tx=32)
            events.append(("tma", c, lambda b=bar[c]["Full"][st]: b.complete_tx(32)))
            issued[c] += 1
        if drain and n_chunks > 0:
            for jj in range(max(0, issued[c] - S), issued[c]):
                yield wait(c, bar[c]["Full"][jj % S], jj // S, True)
            yield wait(c, bar[c]["Drain"], 0, True)
        flags.add(("roles_done", c, "prod"))

    def cleaner():
        for j in range(n_chunks):
            st = j % S
            ok = yield wait(O, bar[O]["Full"][st], j // S)
            if not ok:
                break
            bar[E]["Peer"][st].arrive()
        for jj in range(max(0, n_chunks - S), n_chunks):
            ok = yield wait(O, bar[O]["Empty"][jj % S], jj // S)
            if not ok:
                break
        flags.add(("roles_done", O, "clean"))

    def qk(mine):
        ok = yield wait(E, bar[E]["QReady"], 0)
        for j in range(mine, n_chunks, 2):
            if not ok:
                break
            st = j % S
            if j >= 2:
                ok = yield wait(E, bar[E]["SFree"][j & 1], (j - 2) >> 1)
                if not ok:
                    break
            ok = yield wait(E, bar[E]["Full"][st], j // S)
            if not ok:
                break
            ok = yield wait(E, bar[E]["Peer"][st], j // S)
            if not ok:
                break
            mma(f"qk{mine}")
            commit(f"qk{mine}", "SFull", j & 1)
        if drain:
            commit(f"qk{mine}", "Drain")
        flags.add(("roles_done", E, f"qk{mine}"))

    def pv():
        ok = True
        for j in range(n_chunks):
            ok = yield wait(E, bar[E]["PFull"][j & 1], j >> 1)
            if not ok:
                break
            mma("pv")
            commit("pv", "Empty", j % S)
        if ok:
            commit("pv", "OFinal")
            for jj in range(max(0, n_chunks - S), n_chunks):
                ok = yield wait(E, bar[E]["Empty"][jj % S], jj // S)
                if not ok:
                    break
        if drain:
            commit("pv", "Drain")
        flags.add(("roles_done", E, "pv"))

    def group(c, wg):
        bar[E]["QReady"].arrive(4)
        ok = True
        for j in range(wg, n_chunks, 2):
            if ok:
                ok = yield wait(c, bar[c]["SFull"][wg], j >> 1)
            if ok:
                bar[E]["SFree"][wg].arrive(4)
            if j >= 1:
                yield ("flag", ("m", c, j - 1))          # the reference max handed over by the other group
            flags.add(("m", c, j))
            if not ok:
                continue
            if j >= 1 and rng.random() < 0.3:              # a rescale of O waits for P V of chunk j - 1
                ok = yield wait(c, bar[c]["Empty"][(j - 1) % S], (j - 1) // S)
            if ok and j >= 2:                              # this group's P buffer: P V of chunk j - 2 done
                ok = yield wait(c, bar[c]["Empty"][(j - 2) % S], (j - 2) // S)
            if not ok:
                continue
            bar[E]["PFull"][wg].arrive(4)

    def softmax_end(c):
        # both groups meet (named barrier 1), then the final O
        yield ("flag", ("grpdone", c, 0))
        yield ("flag", ("grpdone", c, 1))
        ok = not abort[c]
        if ok and n_chunks > 0:
            ok = yield wait(c, bar[c]["OFinal"], 0)
        flags.add(("roles_done", c, "softmax"))

    def tail(c):
        names = ["prod", "softmax"] + (["qk0", "qk1", "pv"] if c == E else ["clean"])
        for other in (E, O):            # the cluster barrier: every role of both CTAs has arrived
            for n in (["prod", "softmax"] + (["qk0", "qk1", "pv"] if other == E else ["clean"])):
                yield ("flag", ("roles_done", other, n))
        if not drain:
            for _ in range(rng.randint(0, 3)):   # the fixed sleep: some completions land, maybe not all
                yield ("sleep",)
        passed_final.add(c)
        # invariants: nothing still in flight into this CTA
        if any(k == "tma" and t == c for (k, t, _) in events):
            raise Hazard(f"CTA {c} passes the final barrier with a TMA load into it in flight")
        if any(op[0] == "mma" for op in pipe):
            raise Hazard(f"CTA {c} passes the final barrier with an MMA of its pair in flight")
        if any(op[0] == "commit" for op in pipe):
            raise Hazard(f"CTA {c} passes the final barrier with a commit into it pending")
        # the exchange: the partner's copy into this CTA lands; wait for it before exiting
        bar[c]["Xfer"].arrive(1, tx=64)
        events.append(("xfer", c, lambda b=bar[c]["Xfer"]: b.complete_tx(64)))
        yield wait(c, bar[c]["Xfer"], 0, True)
        flags.add(("exit", c))

    # group completion flags come from the group processes
    def group_done(c, wg):
        g = group(c, wg)
        res = None
        try:
            while True:
                res = yield g.send(res) if res is not None else next(g)
        except StopIteration:
            pass
        flags.add(("grpdone", c, wg))

    procs = [("prod", E, producer(E)), ("prod", O, producer(O)), ("clean", O, cleaner()), ("qk0", E, qk(0)),
             ("qk1", E, qk(1)), ("pv", E, pv()), ("g0", E, group_done(E, 0)), ("g1", E, group_done(E, 1)),
             ("g0", O, group_done(O, 0)), ("g1", O, group_done(O, 1)), ("sm", E, softmax_end(E)),
             ("sm", O, softmax_end(O)), ("tail", E, tail(E)), ("tail", O, tail(O))]
    if n_chunks == 0:
        # an empty bank: no tensor memory, no roles but the tails (the kernel skips everything)
        procs = [p for p in procs if p[0] in ("tail",)]
        for c in (E, O):
            for n in ["prod", "softmax"] + (["qk0", "qk1", "pv"] if c == E else ["clean"]):
                flags.add(("roles_done", c, n))
    state = {p: None for p in procs}
    started = set()

    def ready(w):
        if w is None:
            return True
        if w[0] == "flag":
            return w[1] in flags
        if w[0] == "sleep":
            return True
        _, c, b, phase, is_drain = w
        return b.done > phase or (abort[c] and not is_drain)

    live = list(procs)
    steps = 0
    while live:
        steps += 1
        if steps > max_steps:
            raise Hazard("no progress")
        runnable = [p for p in live if ready(state[p])]
        choices = [("p", p) for p in runnable] + [("e", i) for i in range(len(events))]
        if not choices:
            # every process is blocked: the kernel's bounded waits run out; abort-aware ones give up
            blocked = [p for p in live if state[p] and state[p][0] == "wait" and not state[p][4]]
            if not blocked:
                names = ", ".join(f"{p[0]}@{p[1]} {state[p][2].name if state[p][0] == 'wait' else state[p]}"
                                  for p in live)
                raise Hazard("a drain wait can never complete: " + names)
            p = rng.choice(blocked)
            abort[state[p][1]] = True
            continue
        if runnable and events:
            kind, ch = ("e", rng.randrange(len(events))) if rng.random() < async_bias else ("p", rng.choice(runnable))
        else:
            kind, ch = rng.choice(choices)
        if kind == "e":
            events.pop(ch)[2]()
            continue
        p = ch
        w = state[p]
        result = None
        if w is not None and w[0] == "wait":
            _, c, b, phase, is_drain = w
            if b.done > phase + 1:
                raise Hazard(f"{p[0]}@{p[1]} waits phase {phase} of {b.name}, which has completed {b.done}")
            result = b.done > phase
            if not result and not is_drain:
                abort[c] = True
            elif result and not is_drain and abort_rate and rng.random() < abort_rate:
                result = False                    # this wait timed out after all (a slow phase)
                abort[c] = True
        try:
            if p not in started:
                started.add(p)
                state[p] = next(p[2])
            else:
                state[p] = p[2].send(result)
        except StopIteration:
            live.remove(p)
            state[p] = None
            continue
        nw = state[p]
        if nw is not None and nw[0] == "wait" and nw[2].done < nw[3] and not (abort[nw[1]] and not nw[4]):
            # the phase before the awaited one is still open: its parity differs from the awaited
            # phase's, so the hardware's parity wait would pass at once
            raise Hazard(f"{p[0]}@{p[1]} waits phase {nw[3]} of {nw[2].name}, which has completed only "
                         f"{nw[2].done}")
    return steps
