"""Integer part of the step on the GPU -- position decode and cache rows -- bit-exact
against the oracle ("Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", Section 3.3.3; Algorithm 3, step 3)."""
import numpy as np
import pytest
import torch

import oracle
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu


def _gpu_decode(tb, te, s, T, H, W, C, slot):
    out = torch.empty((te - tb, 4), dtype=torch.int64, device="cuda")
    rope3d.rope3d_decode_positions(tb, te, s, T, H, W, C, slot, out)
    return out.cpu().numpy()


@pytest.mark.parametrize("grid", [(3, 4, 6), (3, 30, 52), (3, 45, 80), (21, 30, 52), (1, 1, 1),
                                  (2, 1, 9), (5, 7, 1)])
@pytest.mark.parametrize("s", [0, 3, 18, 237])
def test_decode_matches_oracle(grid, s):
    T, H, W = grid
    n = T * H * W
    orc = oracle.default()
    C = max(n, 144)
    slot = (s * H * W) % C
    got = _gpu_decode(0, n, s, T, H, W, C, slot)
    idx = range(n) if n <= 5000 else sorted(set(np.random.default_rng(s).integers(0, n, 2000).tolist()) | {0, n - 1})
    for i in idx:
        assert tuple(got[i, :3]) == orc.decode(i, s, T, H, W), i
        assert got[i, 3] == orc.cache_row(i, slot, C), i


def test_decode_sub_ranges_and_wrap():
    orc = oracle.default()
    T, H, W = 3, 30, 52
    for (tb, te) in wl.slices(T * H * W, 7) + [(4679, 4680), (1559, 1561)]:
        got = _gpu_decode(tb, te, 9, T, H, W, 2000, 1990)
        for r, i in enumerate(range(tb, te)):
            assert tuple(got[r, :3]) == orc.decode(i, 9, T, H, W)
            assert got[r, 3] == orc.cache_row(i, 1990, 2000)


def test_decode_large_indices_use_64_bit():
    # a grid whose indices pass 2^31 -- the decode must not overflow
    T, H, W = 600, 2000, 2000
    n = T * H * W
    assert n > 2 ** 31
    orc = oracle.default()
    tb, te = n - 1000, n
    got = _gpu_decode(tb, te, 5, T, H, W, 3_000_000_001, 2_999_999_000)
    for r in range(0, 1000, 37):
        i = tb + r
        assert tuple(got[r, :3]) == orc.decode(i, 5, T, H, W)
        assert got[r, 3] == orc.cache_row(i, 2_999_999_000, 3_000_000_001)
