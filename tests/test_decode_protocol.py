"""The split decode kernels' barrier protocols (tensor-core and CUDA-core),
checked on the host with the discrete-event models in
tests/decode_protocol_model.py (which issue each kernel's waits, arrivals,
commits, copies, MMAs and shared-memory accesses in the kernel's order)."""
import itertools

import pytest

from tests.decode_protocol_model import (CC_MUTATIONS, MUTATIONS, REDUNDANT, ProtocolError, random_case,
                                         random_cc_case, simulate, simulate_cc)


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


def test_cuda_core_kernel_runs_clean():
    for seed in range(300):
        simulate_cc(*random_cc_case(seed), seed=seed)


@pytest.mark.parametrize("d,kv8", [(64, False), (128, False), (64, True), (128, True)])
@pytest.mark.parametrize("gc", [1, 2, 4, 8])
def test_cuda_core_every_configuration(d, gc, kv8):
    """Every head size, heads-per-CTA and cache type (so every way the combine
    scratch overlaps the consumers' rows of the first ring slot), 1 to 14
    pages (fewer, as many and more pages than ring slots)."""
    for num_pages, seed in itertools.product(range(1, 15), range(2)):
        simulate_cc(num_pages, d, gc, kv8, seed=seed)


@pytest.mark.parametrize("mutation", CC_MUTATIONS)
def test_cuda_core_planted_mistakes_are_caught(mutation):
    caught = 0
    for seed in range(300):
        try:
            simulate_cc(*random_cc_case(seed), seed=seed, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"model misses {mutation}"
