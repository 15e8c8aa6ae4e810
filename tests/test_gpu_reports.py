"""The enhancement-share diagnostic computed from the CUDA path agrees with
the same statistics computed from the fp64 oracle's outputs."""
import dataclasses

import numpy as np
import pytest

import bench
from sfa_harness import Pair
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def test_enhancement_share_matches_the_oracle():
    base = WORKLOADS["tiny"]
    got, ref = {}, {}
    for ab in (0.0, 10.0):
        w = base.replace(values=dataclasses.replace(base.values, alpha_base=ab))
        pair = Pair(w)
        g, r = pair.prefill(128)
        got[ab], ref[ab] = g, r
    sg = bench.enhancement_stats(got[0.0], got[10.0])
    sr = bench.enhancement_stats(ref[0.0], ref[10.0])
    for key in ("cos_median", "share_median", "share_p90"):
        assert abs(sg[key] - sr[key]) < 1e-3, (key, sg[key], sr[key])
    # the enhancement is bounded by eps * alpha_layer (0.5 * 0.3 * 10 at L = 1)
    assert np.abs(got[10.0] - got[0.0]).max() <= 0.5 * 0.3 * 10.0 + 1e-6
