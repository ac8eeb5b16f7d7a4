"""Every tree of 1 to 6 nodes (each parent array with parent[i] in {-1, 0, .., i-1}: 873
trees) in one batch, through both verify kernels and the commit, compared in full with the
oracle."""
import itertools

import pytest

from linear_attention_tree_b200 import workloads as W
from tests.test_parity_gpu import _full_check

pytestmark = pytest.mark.gpu


def _all_trees(max_n):
    trees = []
    for n in range(1, max_n + 1):
        for par in itertools.product(*[range(-1, i) for i in range(n)]):
            trees.append(list(par))
    return trees


@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_every_tree_up_to_six_nodes(kernel):
    trees = _all_trees(6)
    assert len(trees) == 1 + 2 + 6 + 24 + 120 + 720
    w = W.synthetic(trees, H=1, dk=128, dv=128, seed=6, name="all-trees-6")
    _full_check(w, kernel)
