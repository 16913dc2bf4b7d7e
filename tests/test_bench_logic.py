"""Host logic of the benchmark that needs no GPU: the FLOPs accounting of the
layer and the rank of the FLOPs-matched static baseline ([DyRA] App. E.4:
a static low-rank layer of rank r + k + k' with the same FLOPs as DyRA)."""

import dataclasses
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from synth import CONFIGS  # noqa: E402


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_static_matched_rank(name):
    s = CONFIGS[name]
    rs = bench.static_matched_rank(s)
    _, _, dyra_flops, _ = bench.algorithmic(s)
    per_rank = 2.0 * s.N * (s.d_in + s.d_out)
    cap = min(s.d_in, s.d_out) // 8 * 8
    assert rs % 8 == 0
    # the static layer has at least the ranks DyRA applies (r static + k correction)
    assert s.r + s.k <= rs <= cap
    # the largest multiple of 8 whose FLOPs do not exceed DyRA's, unless capped
    if rs < cap:
        assert rs * per_rank <= dyra_flops < (rs + 8) * per_rank
    else:
        assert rs * per_rank <= dyra_flops or rs == cap


def test_algorithmic_counts_the_correction():
    """With k = 0 the layer's FLOPs are exactly the static part's."""
    s = dataclasses.replace(CONFIGS["vit_fc1"], k=0)
    flops, _, total, _ = bench.algorithmic(s)
    assert flops["gram"] == 0 and flops["solve"] == 0 and flops["rfactor"] == 0
    assert total == pytest.approx(2.0 * s.N * s.r * (s.d_in + s.d_out))
