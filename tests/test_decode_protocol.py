"""The tensor-core split decode's barrier protocol, checked on the host with
the discrete-event model in tests/decode_protocol_model.py (which issues the
kernel's waits, arrivals, commits, copies and MMAs in the kernel's order)."""
import itertools

import pytest

from tests.decode_protocol_model import MUTATIONS, REDUNDANT, ProtocolError, random_case, simulate


def test_random_cases_run_clean():
    for seed in range(400):
        simulate(*random_case(seed), seed=seed)


@pytest.mark.parametrize("items,kv8", [(3, False), (6, False), (6, True), (12, True)])
@pytest.mark.parametrize("tail", [False, True])
def test_every_ring_depth_and_tile_count(items, kv8, tail):
    """The kernel's ring depths, 1 to 13 key tiles (fewer, as many and more
    tiles than ring slots), with and without a partly filled last page."""
    for n_tiles, seed in itertools.product(range(1, 14), range(3)):
        grew = [False] + [(seed + j) % 3 == 0 for j in range(1, n_tiles)]
        simulate(n_tiles, items, kv8, tail, grew, seed=seed)


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_protocol_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(300):
        try:
            simulate(*random_case(seed), seed=seed, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"model misses {mutation}"


@pytest.mark.parametrize("mutation", REDUNDANT)
def test_redundant_waits_never_matter(mutation):
    """Waits the earlier commits already imply: dropping one is never seen."""
    for seed in range(300):
        simulate(*random_case(seed), seed=seed, mutation=mutation)
