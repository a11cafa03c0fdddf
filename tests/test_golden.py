"""The oracle against its stored regression fixture.

The pages print no worked numeric example, so the fixture is not a pin: it
was written by tests/golden/make_golden.py, which calls only the oracle and
the seeded input generator, and it guards the oracle against unintended
changes between commits."""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402
from sparse_hierarchical_attention_chunk_b200 import configs  # noqa: E402


def test_oracle_reproduces_stored_tiny_fixture():
    with open(os.path.join(HERE, "golden", "oracle_tiny_f32_seed7.json")) as f:
        ref = json.load(f)
    cur = make_golden.compute(configs.TINY_F32, seed=ref["seed"])
    assert cur["positions"] == ref["positions"]
    assert cur["mask"] == ref["mask"]
    for key in ("kbar_c3_first8", "w", "o_first8", "lse"):
        np.testing.assert_allclose(np.array(cur[key]), np.array(ref[key]), rtol=1e-12, atol=1e-12)
    # the fixture is not degenerate: some position routes, rows sum to 1
    w = np.array(ref["w"])
    assert (w.sum(axis=-1)[2:] > 0.999).all() and (w[:2] == 0).all()
