"""The device Philox4x32-10 uniforms equal the oracle's bit for bit."""

import numpy as np
import pytest
import torch

from oracle.philox import uniform

pytestmark = pytest.mark.gpu


def test_device_uniforms_match_oracle():
    import tree_verification_verify_b200 as tv
    from tree_verification_verify_b200 import build
    build.build()
    rng = np.random.default_rng(0)
    n = 20000
    b = rng.integers(0, 64, n).astype(np.int32)
    node = rng.integers(0, 1 << 20, n).astype(np.int32)
    draw = rng.integers(0, 1 << 27, n).astype(np.int32)
    tag = rng.integers(1, 4, n).astype(np.int32)
    for seed, step in ((0, 0), (123456789, 7), ((1 << 64) - 1, (1 << 40) + 3)):
        dev = [torch.from_numpy(x).cuda() for x in (b, node, draw, tag)]
        got = tv.philox_uniforms(seed, step, *dev).cpu().numpy()
        ref = uniform(seed, step, b.astype(np.uint64), node.astype(np.uint64),
                      draw.astype(np.uint64), tag.astype(np.uint64))
        np.testing.assert_array_equal(got, ref)
