"""The prefill kernel's barrier protocol, on the CPU, through a randomised model.

``prefill_protocol_model.py`` plays every role of one CTA pair (TMA producers, the odd CTA's
cleaner, the Q K^T and P V issuers, both softmax groups, the tails) against the kernel's mbarriers,
with copies, MMAs and commits completing in random order.  A GPU test cannot make a bounded wait
run out without hanging work on purpose, so the abandon-and-drain path is exercised here: waits are
made to time out at random, and the model checks that no copy, MMA or commit into a CTA is still
in flight when that CTA passes the final cluster barrier (after which it frees tensor memory and
reuses its stage area).
"""
import random

import pytest

import prefill_protocol_model as model

CHUNKS = [0, 1, 2, 3, 5, 6, 9, 16, 17, 20]


@pytest.mark.parametrize("async_bias", [0.5, 0.1, 0.02])
def test_protocol_is_sound_without_timeouts(async_bias):
    for seed in range(150):
        n = random.Random(seed).choice(CHUNKS)
        model.run(n, seed, async_bias=async_bias)


@pytest.mark.parametrize("async_bias", [0.5, 0.1, 0.02])
def test_abandoned_tiles_drain_before_the_final_barrier(async_bias):
    for seed in range(150):
        n = random.Random(seed).choice(CHUNKS)
        model.run(n, seed, abort_rate=0.05, async_bias=async_bias)


def test_a_fixed_delay_instead_of_the_drain_is_caught():
    """The check that guards the drain: with a fixed delay in its place and slow asynchronous work,
    some schedules pass the final barrier with a load still landing."""
    caught = 0
    for seed in range(200):
        n = random.Random(seed).choice(CHUNKS[1:])
        try:
            model.run(n, seed, abort_rate=0.05, drain=False, async_bias=0.02)
        except model.Hazard as e:
            assert "in flight" in str(e) or "after it passed" in str(e)
            caught += 1
    assert caught > 0


def test_a_parity_wait_two_phases_behind_is_caught():
    """A planted protocol mistake: the producer reuses a stage one phase early (it waits on the
    empty barrier of the chunk before the one that used the stage)."""
    src = open(model.__file__).read()
    bad = src.replace('ok = yield wait(c, bar[c]["Empty"][st], j // S - 1)',
                      'ok = yield wait(c, bar[c]["Empty"][st], max(0, j // S - 2))')
    assert bad != src
    ns = {}
    exec(compile(bad, "planted_model", "exec"), ns)
    caught = 0
    for seed in range(100):
        try:
            ns["run"](17, seed, stages=2)
        except ns["Hazard"]:
            caught += 1
    assert caught > 0


def test_a_parity_wait_on_a_phase_not_yet_open_is_caught():
    """A planted protocol mistake: the P V issuer waits on the P buffer's next phase (the phase
    before it still open, so the hardware's parity wait would pass at once and P V would read a P
    not yet written)."""
    src = open(model.__file__).read()
    bad = src.replace('ok = yield wait(E, bar[E]["PFull"][j & 1], j >> 1)',
                      'ok = yield wait(E, bar[E]["PFull"][j & 1], (j >> 1) + 1)')
    assert bad != src
    ns = {}
    exec(compile(bad, "planted_model", "exec"), ns)
    caught = 0
    for seed in range(50):
        try:
            ns["run"](9, seed)
        except ns["Hazard"] as e:
            assert "completed only" in str(e)
            caught += 1
    assert caught > 0
