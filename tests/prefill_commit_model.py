"""A randomised model of the prefill call's cross-launch hand-off through each (sequence, group)'s
ticket word (one launch of the attention kernel, one of the commit kernel, all groups).

Test infrastructure: ``tests/test_prefill_protocol.py`` runs it on the CPU.  It mirrors
``rma_prefill.cu``: attention clusters take items in the kernel's order (group-major, a cluster's
items permuted within each wave); every softmax warp of an item's CTA pair, once its stores of the
item's rows have completed, adds 1 << 16 to the group's word.  The commit's slices wait until the
high half reaches 16 arrivals per item of their group, then read the rows and write the ring; the
admit CTA does not wait; every commit CTA then adds 1 and the one that sees the low half reach the
slice count writes the group's counters and clears the word.  Warps, slices and the admit run in a
random interleaving.

What it checks: a slice reads a group's rows only after every item of the group has stored them;
the counters are written only after every item of the group has finished (the items read them);
the word is zero again after the call (the next call, and the decode's split merge, start from 0);
no wait can block for good.
"""
import random


class Hazard(Exception):
    pass


def run(n_groups, npairs, n_clusters, slices, seed, max_steps=200_000):
    rng = random.Random(seed)
    per_group = 2 * npairs
    n_items = n_groups * per_group
    warps_per_item = 16
    need = warps_per_item * per_group
    word = [0] * n_groups
    counters_written = [False] * n_groups
    items_done = [0] * n_groups          # items whose every warp has signalled
    items_started = [0] * n_groups
    events = []

    def item_at(c, k):
        return k * n_clusters + (c + 2 * k) % n_clusters

    def cluster(c):
        k = 0
        while k * n_clusters < n_items:
            it = item_at(c, k)
            k += 1
            if it >= n_items:
                continue
            g = it // per_group
            if counters_written[g]:
                raise Hazard(f"item {it} of group {g} starts after the group's counters were written")
            items_started[g] += 1
            yield "work"
            # the item's 16 warps signal one by one, each after its own stores completed
            for _ in range(warps_per_item):
                yield "store"
                word[g] += 1 << 16
            items_done[g] += 1

    def slice_cta(g):
        yield "pre-wait work"
        while (word[g] >> 16) < need:
            yield "spin"
        if items_done[g] != per_group:
            raise Hazard(f"a slice of group {g} reads rows with {items_done[g]} of {per_group} items done")
        yield "combine and ring write"
        yield from arrive(g)

    def admit_cta(g):
        yield "competition"
        yield from arrive(g)

    def arrive(g):
        old = word[g]
        word[g] += 1
        if (old & 0xFFFF) == slices:
            if items_done[g] != per_group or items_started[g] != per_group:
                raise Hazard(f"group {g}'s counters written with {items_done[g]} items done")
            if (word[g] >> 16) != need:
                raise Hazard(f"group {g}'s word cleared with {word[g] >> 16} of {need} row arrivals")
            counters_written[g] = True
            word[g] = 0
        yield "arrived"

    procs = [cluster(c) for c in range(min(n_clusters, n_items))]
    for g in range(n_groups):
        procs.append(admit_cta(g))
        procs += [slice_cta(g) for _ in range(slices)]
    live = list(procs)
    steps = 0
    while live:
        steps += 1
        if steps > max_steps:
            raise Hazard("no progress")
        p = rng.choice(live)
        try:
            next(p)
        except StopIteration:
            live.remove(p)
    for g in range(n_groups):
        if word[g] != 0 or not counters_written[g]:
            raise Hazard(f"group {g}: word {word[g]:#x} after the call, counters written {counters_written[g]}")
    return steps
