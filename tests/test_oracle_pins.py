"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.fixture(autouse=True)
def _no_mutation():
    oracle.set_mutation(oracle.MUTATION_NONE)
    yield
    oracle.set_mutation(oracle.MUTATION_NONE)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_golden_tree_shape_matches_generator():
    """The level tree the generator draws has the shape printed on the pages."""
    import os
    from tree_masked_verification_b200.inputs import LONGSPEC_TREE_SHAPE, WORKLOADS
    path = os.path.join(os.path.dirname(__file__), "golden", "longspec_tree_shape.txt")
    kv = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.split()
    widths = tuple(int(x) for x in kv["widths"])
    assert widths == LONGSPEC_TREE_SHAPE
    assert int(kv["nodes"][0]) == sum(widths) == WORKLOADS["llama3-8b-32k"].T
    par = WORKLOADS["llama3-8b-32k"].parents()[0]
    depth = np.zeros(len(par), dtype=int)
    for i, p in enumerate(par):
        depth[i] = 1 if p == -1 else depth[p] + 1
    assert depth.max() == int(kv["depth"][0])
    assert np.bincount(depth)[1:].tolist() == list(widths)


@pytest.mark.parametrize("par", [[0], [-1, 1], [-1, 0, 3], [-2, 0], [-1, 2, 0]])
def test_mask_rejects_bad_parent(par):
    with pytest.raises(oracle.OracleError) as e:
        oracle.tree_mask(par)
    assert e.value.code == oracle.BAD_PARENT


def test_rows_subset_matches_full():
    from tree_masked_verification_b200.inputs import Workload
    w = Workload("rows", B=2, Hq=4, Hkv=2, D=8, T=6, L_cap=10, seed=3,
                 tree="random", prefix_range=(0, 10))
    p = pins.problem_from(w.generate())
    out, lse = p.attention()
    rows = np.array([[1, 3, 5], [0, 0, 0], [1, 1, 2]], dtype=np.int32)
    o2, l2 = p.attention(rows)
    for i, (b, h, t) in enumerate(rows):
        np.testing.assert_array_equal(o2[i], out[b, h, t])
        assert l2[i] == lse[b, h, t]


def test_empty_prefix_chunk_is_empty_partial():
    from tree_masked_verification_b200.inputs import Workload
    w = Workload("empty", B=1, Hq=2, Hkv=1, D=4, T=3, L_cap=6, seed=4,
                 tree="random", prefix_range=(3, 3))
    p = pins.problem_from(w.generate())
    o, l = p.prefix_partial(3, 6)
    assert np.all(l == -np.inf) and np.all(o == 0)
