"""A randomised model of the prefill attention kernel's barrier protocol (one cluster of 2 CTAs
of one launch, looping over its work items).

Test infrastructure: ``tests/test_prefill_protocol.py`` runs it on the CPU.  It mirrors the roles
of ``prefill_attn_kernel`` in ``rma_prefill.cu``: the TMA producer of each CTA, the odd CTA's
cleaner, the even CTA's two Q K^T issuers and its P V issuer, the two softmax groups of each CTA
(which also load each item's Q into tensor memory and drain its O), and each CTA's exit, with the
mbarriers they share.  Asynchronous work completes later, in a random order that keeps the
hardware's guarantees: TMA bytes land in any order; the pair's tensor pipe runs its MMAs in issue
order; a tcgen05 commit arrives once every earlier MMA of its issuing thread is done.

What it checks, over many random schedules and item lists:
  * every parity wait is sound: when it is issued its barrier has completed P or P + 1 phases (a
    barrier two phases ahead would let a parity wait pass on the wrong phase, and one whose phase
    P - 1 is still open would let it pass at once);
  * tensor-memory and shared-memory hazards: Q of an item is written only when no Q K^T is queued
    in the pipe; a Q K^T runs only on the Q of its own item; a P V of an item runs only after every
    group of both CTAs has drained O of the previous item; a P V reads only a P its group wrote
    for that chunk;
  * nothing deadlocks (an abort-aware wait that can never complete is timed out, as the kernel's
    bounded wait would, and its CTA abandons its work; a drain wait that can never complete is an
    error);
  * when a CTA passes the final cluster barrier (after which it frees tensor memory), no TMA load
    into it, no MMA of its pair and no commit into its barriers is still in flight.

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


def run(items, seed, stages=5, abort_rate=0.0, drain=True, async_bias=0.5, max_steps=2_000_000):
    """One cluster's launch over `items`, the chunk count of each of its work items in order (0 = an
    item without chunks: an empty bank).  async_bias is the chance that a scheduling step completes
    pending asynchronous work rather than advancing a role."""
    rng = random.Random(seed)
    E, O = 0, 1
    S = stages
    bar = {}
    for c in (E, O):
        bar[c] = {"Full": [Barrier(f"c{c}.Full{i}", 1) for i in range(S)],
                  "Empty": [Barrier(f"c{c}.Empty{i}", 1) for i in range(S)],
                  "SFull": [Barrier(f"c{c}.SFull{i}", 1) for i in range(2)],
                  "OFinal": Barrier(f"c{c}.OFinal", 1), "Drain": Barrier(f"c{c}.Drain", 3)}
    bar[E].update({"Peer": [Barrier(f"E.Peer{i}", 1) for i in range(S)], "QReady": Barrier("E.QReady", 16),
                   "PFull": [Barrier(f"E.PFull{i}", 8) for i in range(2)],
                   "SFree": [Barrier(f"E.SFree{i}", 8) for i in range(2)],
                   "ODrained": Barrier("E.ODrained", 16)})
    abort = {E: False, O: False}
    events = []                 # pending asynchronous completions: (kind, target cta, callable)
    pipe = []                   # the pair's tensor pipe: ("mma", issuer, check) / ("commit", issuer, fn, targets)
    issued = {E: 0, O: 0}       # chunks whose loads each producer issued
    passed_final = set()
    flags = set()
    n_items = len(items)
    base = [sum(items[:i]) for i in range(n_items + 1)]          # global index of each item's first chunk
    with_chunks = [i for i in range(n_items) if items[i] > 0]
    # tensor-memory contents: whose Q is in it (per CTA), which item's O each group has drained
    q_of = {E: None, O: None}
    drained = {(c, wg): -1 for c in (E, O) for wg in (0, 1)}   # last item with chunks whose O the group drained
    p_of = {(c, wg): None for c in (E, O) for wg in (0, 1)}    # global chunk whose P is in the group's buffer

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
                if op[2] is not None:
                    op[2]()
                break
        pipe_fire_commits()

    def mma(issuer, check=None):
        pipe.append(("mma", issuer, check))
        events.append(("mma", None, pipe_step))

    def commit(issuer, key, idx=None):
        def fn():
            for c in (E, O):
                (bar[c][key] if idx is None else bar[c][key][idx]).arrive()
        pipe.append(("commit", issuer, fn, (E, O)))
        pipe_fire_commits()

    def wait(c, b, phase, is_drain=False):
        return ("wait", c, b, phase, is_drain)

    # ---------------- roles ----------------
    def producer(c):
        ok = True
        jg = 0
        for it in range(n_items):
            for j in range(items[it]):
                st = jg % S
                if jg >= S:
                    ok = yield wait(c, bar[c]["Empty"][st], jg // S - 1)
                    if not ok:
                        break
                bar[c]["Full"][st].arrive(1, tx=32)
                events.append(("tma", c, lambda b=bar[c]["Full"][st]: b.complete_tx(32)))
                issued[c] = jg + 1
                jg += 1
            if not ok:
                break
        if drain and issued[c] > 0:
            for jj in range(max(0, issued[c] - S), issued[c]):
                yield wait(c, bar[c]["Full"][jj % S], jj // S, True)
        if drain:
            yield wait(c, bar[c]["Drain"], 0, True)
        flags.add(("roles_done", c, "prod"))

    def cleaner():
        jg = 0
        ok = True
        for it in range(n_items):
            for j in range(items[it]):
                st = jg % S
                ok = yield wait(O, bar[O]["Full"][st], jg // S)
                if not ok:
                    break
                bar[E]["Peer"][st].arrive()
                jg += 1
            if not ok:
                break
        for jj in range(max(0, jg - S), jg):
            if not ok:
                break
            ok = yield wait(O, bar[O]["Empty"][jj % S], jj // S)
        flags.add(("roles_done", O, "clean"))

    def qk(mine):
        jg, kw = 0, 0
        ok = True
        for it in range(n_items):
            if items[it] == 0:
                continue
            ok = yield wait(E, bar[E]["QReady"], kw)
            kw += 1
            for j in range(items[it]):
                g = jg
                jg += 1
                if not ok:
                    break
                if (g & 1) != mine:
                    continue
                st = g % S
                if g >= 2:
                    ok = yield wait(E, bar[E]["SFree"][g & 1], (g - 2) >> 1)
                    if not ok:
                        break
                ok = yield wait(E, bar[E]["Full"][st], g // S)
                if not ok:
                    break
                ok = yield wait(E, bar[E]["Peer"][st], g // S)
                if not ok:
                    break

                def check(it=it):
                    if abort[E] or abort[O]:
                        return
                    for c in (E, O):
                        if q_of[c] != it:
                            raise Hazard(f"Q K^T of item {it} runs on CTA {c}'s Q of item {q_of[c]}")
                mma(f"qk{mine}", check)
                commit(f"qk{mine}", "SFull", g & 1)
            if not ok:
                break
        if drain:
            commit(f"qk{mine}", "Drain")
        flags.add(("roles_done", E, f"qk{mine}"))

    def pv():
        jg, kw = 0, 0
        ok = True
        for it in range(n_items):
            if items[it] == 0:
                continue
            if kw >= 1:
                ok = yield wait(E, bar[E]["ODrained"], kw - 1)
            prev = with_chunks[kw - 1] if kw >= 1 else -1
            kw += 1
            for j in range(items[it]):
                g = jg
                jg += 1
                if not ok:
                    break
                ok = yield wait(E, bar[E]["PFull"][g & 1], g >> 1)
                if not ok:
                    break

                def check(it=it, g=g, prev=prev):
                    if abort[E] or abort[O]:
                        return
                    for c in (E, O):
                        for wg in (0, 1):
                            if drained[(c, wg)] < prev:
                                raise Hazard(f"P V of item {it} runs before CTA {c} group {wg} drained O of item {prev}")
                        if p_of[(c, g & 1)] != g:
                            raise Hazard(f"P V of chunk {g} reads CTA {c}'s P of chunk {p_of[(c, g & 1)]}")
                mma("pv", check)
                commit("pv", "Empty", g % S)
            if ok:
                commit("pv", "OFinal")
            else:
                break
        for jj in range(max(0, jg - S), jg):
            if not ok:
                break
            ok = yield wait(E, bar[E]["Empty"][jj % S], jj // S)
        if drain:
            commit("pv", "Drain")
        flags.add(("roles_done", E, "pv"))

    def load_q(c, wg, it):
        # the group's half of its rows' Q: no Q K^T may still be queued
        if not (abort[E] or abort[O]) and any(op[0] == "mma" and op[1].startswith("qk") for op in pipe):
            raise Hazard(f"CTA {c} group {wg} writes Q of item {it} while a Q K^T is queued")
        flags.add(("q", c, wg, it))
        if all(("q", cc, w, it) in flags for cc in (E, O) for w in (0, 1)):
            q_of[E] = q_of[O] = it
        bar[E]["QReady"].arrive(4)

    def group(c, wg):
        ok = True
        jg, kw = 0, 0
        if n_items and items[0] > 0:
            load_q(c, wg, 0)
        for it in range(n_items):
            x = items[it]
            for j in range(x):
                g = jg + j
                if (g & 1) != wg:
                    continue
                if ok:
                    ok = yield wait(c, bar[c]["SFull"][wg], g >> 1)
                if ok:
                    bar[E]["SFree"][wg].arrive(4)
                if j >= 1:
                    yield ("flag", ("m", c, g - 1))          # the reference max handed over by the other group
                flags.add(("m", c, g))
                if not ok:
                    continue
                if j >= 1 and rng.random() < 0.3:              # a rescale of O waits for P V of chunk g - 1
                    ok = yield wait(c, bar[c]["Empty"][(g - 1) % S], (g - 1) // S)
                if ok and g >= 2:                              # this group's P buffer: P V of chunk g - 2 done
                    ok = yield wait(c, bar[c]["Empty"][(g - 2) % S], (g - 2) // S)
                if not ok:
                    continue
                p_of[(c, wg)] = g
                bar[E]["PFull"][wg].arrive(4)
            jg += x
            # both groups meet (named barrier 1), then the final O of the item
            flags.add(("met", c, wg, it))
            yield ("flag", ("met", c, wg ^ 1, it))
            have_o = False
            if x > 0 and ok:
                ok = yield wait(c, bar[c]["OFinal"], kw)
                have_o = ok
            # the next item's Q (every Q K^T of this item has completed), then the drain of O
            if it + 1 < n_items and items[it + 1] > 0:
                if ok:
                    load_q(c, wg, it + 1)
                else:
                    bar[E]["QReady"].arrive(4)                # abandoned: the contents no longer matter
            p_of[(c, wg)] = "drain"                          # the drain stages O in the group's P buffer
            for _ in range(4):                               # four steps of 32 columns, each taking a while
                yield ("sleep",)
            if x > 0:
                if have_o:
                    drained[(c, wg)] = it
                bar[E]["ODrained"].arrive(4)
                kw += 1

    def softmax(c, wg):
        g = group(c, wg)
        res = None
        try:
            while True:
                res = yield g.send(res) if res is not None else next(g)
        except StopIteration:
            pass
        flags.add(("roles_done", c, f"g{wg}"))

    def tail(c):
        for other in (E, O):            # the cluster barrier: every role of both CTAs has arrived
            for n in (["prod", "g0", "g1"] + (["qk0", "qk1", "pv"] if other == E else ["clean"])):
                yield ("flag", ("roles_done", other, n))
        if not drain:
            for _ in range(rng.randint(0, 3)):   # a fixed delay: some completions land, maybe not all
                yield ("sleep",)
        passed_final.add(c)
        if any(k == "tma" and t == c for (k, t, _) in events):
            raise Hazard(f"CTA {c} passes the final barrier with a TMA load into it in flight")
        if any(op[0] == "mma" for op in pipe):
            raise Hazard(f"CTA {c} passes the final barrier with an MMA of its pair in flight")
        if any(op[0] == "commit" for op in pipe):
            raise Hazard(f"CTA {c} passes the final barrier with a commit into it pending")
        flags.add(("exit", c))

    procs = [("prod", E, producer(E)), ("prod", O, producer(O)), ("clean", O, cleaner()), ("qk0", E, qk(0)),
             ("qk1", E, qk(1)), ("pv", E, pv()), ("g0", E, softmax(E, 0)), ("g1", E, softmax(E, 1)),
             ("g0", O, softmax(O, 0)), ("g1", O, softmax(O, 1)), ("tail", E, tail(E)), ("tail", O, tail(O))]
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
            raise Hazard(f"{p[0]}@{p[1]} waits phase {nw[3]} of {nw[2].name}, which has completed only "
                         f"{nw[2].done}")
    return steps
