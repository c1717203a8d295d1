"""GPU parity of fa_merge_states against the oracle's LSE merge."""
import numpy as np
import pytest

import oracle
from tests.gpu_util import compare

pytestmark = pytest.mark.gpu


def run_merge(o_parts, lse_parts):
    import torch
    import exact_attention_148_b200 as fa
    o = torch.from_numpy(o_parts.astype(np.float32)).cuda()
    l = torch.from_numpy(lse_parts.astype(np.float32)).cuda()
    out, lse = fa.merge_states(o, l)
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("S", [1, 2, 3, 17, 64])
@pytest.mark.parametrize("d", [64, 128])
def test_merge_matches_oracle(S, d):
    g = np.random.default_rng(S * 1000 + d)
    R, H = 5, 3
    o_parts = g.standard_normal((S, R, H, d)).astype(np.float32)
    lse_parts = (g.standard_normal((S, R, H)) * 4 + 10).astype(np.float32)
    if S > 2:
        lse_parts[1, 0, 0] = -np.inf          # an empty split carries no weight
    out, lse = run_merge(o_parts, lse_parts)
    o_ref, l_ref = oracle.merge_states_ref(o_parts.astype(np.float64), lse_parts.astype(np.float64))
    compare(out, lse, o_ref, l_ref, f"merge S={S} d={d}")


def test_merge_all_empty_row():
    S, R, H, d = 4, 2, 2, 128
    o_parts = np.ones((S, R, H, d), dtype=np.float32)
    lse_parts = np.zeros((S, R, H), dtype=np.float32)
    lse_parts[:, 1, 0] = -np.inf
    out, lse = run_merge(o_parts, lse_parts)
    assert np.all(out[1, 0] == 0) and np.isneginf(lse[1, 0])
    assert np.allclose(out[0, 0], 1.0) and abs(lse[0, 0] - np.log(4)) < 1e-6


def test_merge_large_lse_offsets():
    g = np.random.default_rng(9)
    o_parts = g.standard_normal((3, 2, 2, 128)).astype(np.float32)
    lse_parts = np.array([1000.0, 1001.0, 999.5], dtype=np.float32)[:, None, None] * np.ones((3, 2, 2), np.float32)
    out, lse = run_merge(o_parts, lse_parts)
    o_ref, l_ref = oracle.merge_states_ref(o_parts.astype(np.float64), lse_parts.astype(np.float64))
    compare(out, lse, o_ref, l_ref, "merge large LSE")
