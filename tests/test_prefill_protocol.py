"""The prefill attention kernel's barrier protocol, on the CPU, through a randomised model.

``prefill_protocol_model.py`` plays every role of one cluster of the persistent attention launch
(TMA producers, the odd CTA's cleaner, the Q K^T and P V issuers, both softmax groups of both CTAs,
the exits) over a list of work items, against the kernel's mbarriers, with copies, MMAs and commits
completing in random order.  A GPU test cannot make a bounded wait run out without hanging work on
purpose, so the abandon-and-drain path is exercised here: waits are made to time out at random, and
the model checks that no copy, MMA or commit into a CTA is still in flight when that CTA passes the
final cluster barrier (after which it frees tensor memory).  Planted mistakes show what the checks
catch.
"""
import random

import pytest

import prefill_protocol_model as model

CHUNKS = [0, 1, 2, 3, 5, 16, 17, 19, 20]


def _items(seed, lo=1, hi=5):
    r = random.Random(seed)
    return [r.choice(CHUNKS) for _ in range(r.randint(lo, hi))]


@pytest.mark.parametrize("async_bias", [0.5, 0.1, 0.02])
def test_protocol_is_sound_without_timeouts(async_bias):
    for seed in range(120):
        model.run(_items(seed), seed, async_bias=async_bias)


@pytest.mark.parametrize("async_bias", [0.5, 0.1, 0.02])
def test_abandoned_items_drain_before_the_final_barrier(async_bias):
    for seed in range(120):
        model.run(_items(seed), seed, abort_rate=0.05, async_bias=async_bias)


def test_bench_shaped_item_lists():
    """The items a cluster gets at the bench's steady state: 3 or 4 items of 16 to 20 chunks."""
    for seed in range(60):
        r = random.Random(seed)
        items = [r.choice([16, 17, 18, 19, 20]) for _ in range(r.choice([3, 4]))]
        model.run(items, seed, async_bias=r.choice([0.5, 0.1]))


def test_a_fixed_delay_instead_of_the_drain_is_caught():
    """The check that guards the drain: with a fixed delay in its place and slow asynchronous work,
    some schedules pass the final barrier with a load still landing."""
    caught = 0
    for seed in range(200):
        try:
            model.run(_items(seed), seed, abort_rate=0.05, drain=False, async_bias=0.02)
        except model.Hazard as e:
            assert "in flight" in str(e) or "after it passed" in str(e) or "pending" in str(e)
            caught += 1
    assert caught > 0


def _planted(old, new):
    src = open(model.__file__).read()
    assert src.count(old) == 1
    ns = {}
    exec(compile(src.replace(old, new), "planted_model", "exec"), ns)
    return ns


def _caught(ns, runs=200, lo=2):
    caught, msgs = 0, []
    for seed in range(runs):
        try:
            ns["run"](_items(seed, lo=lo), seed)
        except ns["Hazard"] as e:
            caught += 1
            msgs.append(str(e))
    return caught, msgs


def test_an_issuer_that_skips_the_q_wait_of_an_item_without_its_chunks_is_caught():
    """The odd-chunk Q K^T issuer skipping the Q barrier's phase of a one-chunk item: its next wait
    is then on a phase whose predecessor may still be open, and passes at once on the hardware."""
    ns = _planted('            ok = yield wait(E, bar[E]["QReady"], kw)\n            kw += 1',
                  '            if mine == 0 or items[it] > 1:\n                ok = yield wait(E, bar[E]["QReady"], kw)\n'
                  '            kw += 1')
    caught, _ = _caught(ns)
    assert caught > 0


def test_loading_the_next_q_before_the_items_last_p_v_is_caught():
    ns = _planted('            if x > 0 and ok:\n                ok = yield wait(c, bar[c]["OFinal"], kw)\n'
                  '                have_o = ok\n',
                  '')
    caught, _ = _caught(ns)
    assert caught > 0


def test_p_v_before_o_is_drained_is_caught():
    ns = _planted('                ok = yield wait(E, bar[E]["ODrained"], kw - 1)', '                pass')
    caught, msgs = _caught(ns)
    assert caught > 0 and any("drained" in m for m in msgs)


def test_a_producer_reusing_a_stage_one_phase_early_is_caught():
    ns = _planted('                    ok = yield wait(c, bar[c]["Empty"][st], jg // S - 1)',
                  '                    ok = yield wait(c, bar[c]["Empty"][st], max(0, jg // S - 2))')
    caught = 0
    for seed in range(100):
        try:
            ns["run"]([17, 9], seed, stages=2)
        except ns["Hazard"]:
            caught += 1
    assert caught > 0


def test_commit_hand_off_through_the_ticket_word():
    """The prefill call's cross-launch hand-off (``prefill_commit_model.py``): slices read a group's
    rows only after every item stored them, the counters change only after every item finished, and
    the word is zero after the call, over random interleavings and shapes."""
    import prefill_commit_model as cm
    for seed in range(200):
        r = random.Random(seed)
        cm.run(n_groups=r.choice([1, 3, 8]), npairs=r.choice([1, 2, 4]), n_clusters=r.choice([1, 5, 16, 64]),
               slices=r.choice([1, 4, 32]), seed=seed)


def test_a_slice_waiting_for_too_few_arrivals_is_caught():
    """A planted mistake: the slices' wait counts one softmax group per item instead of every warp."""
    import prefill_commit_model as cm
    src = open(cm.__file__).read()
    bad = src.replace("    need = warps_per_item * per_group", "    need = 2 * per_group")
    assert bad != src
    ns = {}
    exec(compile(bad, "planted_commit_model", "exec"), ns)
    caught = 0
    for seed in range(50):
        try:
            ns["run"](n_groups=3, npairs=2, n_clusters=5, slices=4, seed=seed)
        except ns["Hazard"]:
            caught += 1
    assert caught > 0
