"""The persistent prefill's barrier protocol, checked on the host with the
discrete-event model in tests/persist_protocol_model.py (which issues the
kernel's waits, arrivals, commits, copies and MMAs in the kernel's order)."""
import pytest

from tests.persist_protocol_model import (MUTATIONS, PAGED_MUTATIONS, ProtocolError, random_case,
                                          random_paged_case, simulate)


def test_random_item_mixes_run_clean():
    for seed in range(400):
        items, claimed, NS, F8 = random_case(seed)
        simulate(items, claimed, NS, F8, seed=seed)


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_protocol_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(200):
        items, claimed, NS, F8 = random_case(seed)
        try:
            simulate(items, claimed, NS, F8, seed=seed, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"model misses {mutation}"


def test_paged_tail_handoff_runs_clean():
    for seed in range(400):
        items, claimed, NS, tails = random_paged_case(seed)
        simulate(items, claimed, NS, False, seed=seed, tails=tails)


@pytest.mark.parametrize("mutation", PAGED_MUTATIONS)
def test_paged_tail_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(200):
        items, claimed, NS, tails = random_paged_case(seed)
        try:
            simulate(items, claimed, NS, False, seed=seed, mutation=mutation, tails=tails)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"model misses {mutation}"
