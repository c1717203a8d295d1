"""bench.py's DRAM-traffic attribution on the host: a decode batch whose
requests share pages (a common prefix) must not take the K/V-scaled traffic of
the 16-request capture, whose requests own their pages."""
import numpy as np

import bench
import workloads as W


def test_private_pages_are_not_shared():
    inp = W.make_decode([70, 1, 640, 129], 4, 2, 64, seed=5)
    assert not bench.pages_shared(inp)


def test_shared_prefix_pages_are_detected():
    casc = W.make_cascade(128, [64, 3, 200], 4, 2, 64, seed=6)
    assert bench.pages_shared(casc.as_plain_decode())


def test_unused_slots_do_not_count():
    # a page id repeated only past a request's length is not read twice
    inp = W.make_decode([64, 64], 4, 2, 64, seed=7, extra_pages=2)
    inp.block_table = np.concatenate([inp.block_table, inp.block_table[::-1]], axis=1)
    assert not bench.pages_shared(inp)
    inp.cache_seqlens = np.array([65, 64], dtype=np.int32)   # row 0 now reads row 1's page
    assert bench.pages_shared(inp)


def test_shared_batch_gets_no_scaled_traffic():
    casc = W.make_cascade(128, [64, 3, 200], 4, 2, 64, seed=6)

    class Case:
        fp8 = False
        inp = casc.as_plain_decode()

    assert bench.measured_traffic("decode_tc", Case.inp.name, Case) == (None, None)


def test_private_batch_gets_scaled_traffic():
    # the control for the test above: the same lookup with private pages
    class Case:
        fp8 = False
        inp = W.make_decode([70, 1, 640, 129], 4, 2, 64, seed=5)

    traffic, source = bench.measured_traffic("decode_tc", Case.inp.name, Case)
    assert traffic is not None and traffic > 0
    assert "scaled by K/V bytes" in source
