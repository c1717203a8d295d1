"""The grid-form prefill kernel's barrier protocol, checked on the host with
the discrete-event model in tests/prefill_grid_protocol_model.py (which issues
the kernel's waits, arrivals, commits, copies and MMAs in the kernel's order)."""
import itertools
import random

import pytest

from tests.prefill_grid_protocol_model import MUTATIONS, REDUNDANT, ProtocolError, random_case, simulate


def test_random_cases_run_clean():
    for seed in range(400):
        simulate(*random_case(seed), seed=seed)


@pytest.mark.parametrize("NS,f8,tail", [(5, False, False), (5, False, True), (8, False, False),
                                        (8, False, True), (8, True, False)])
def test_every_pair_of_key_tile_counts(NS, f8, tail):
    """The kernel's ring depths and input kinds; slot 0 with 1-9 key tiles and
    slot 1 with none up to one more than slot 0 (fewer, as many and more key
    tiles than ring slots)."""
    r = random.Random(NS * 10 + f8 * 2 + tail)
    for n0, n1 in itertools.product(range(1, 10), range(0, 11)):
        if n1 > n0 + 1:
            continue
        rescale = [[[r.random() < 0.3 for _ in range(max(n0, n1) + 1)] for _ in range(4)] for _ in range(2)]
        simulate((n0, n1), NS, f8, tail, rescale, seed=n0 * 16 + n1)


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_protocol_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(400):
        try:
            simulate(*random_case(seed), seed=seed, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"model misses {mutation}"


@pytest.mark.parametrize("mutation", REDUNDANT)
def test_redundant_waits_never_matter(mutation):
    """Waits the earlier commits already imply: dropping one is never seen."""
    for seed in range(400):
        simulate(*random_case(seed), seed=seed, mutation=mutation)
