"""Batch-wide verification budget (host policy): optimality against brute force, the
cap-the-largest rule against its literal loop and the ragged workload's recipe, the cost
model's fit, and pruning checked through the oracle.

The pages (Twig abstract, "batch-wide verification budgeting"; Bole summary, 批级验证预算校准)
give the budget no formula; the expected-token objective and greedy rule are the plain reading
stated in the module's docstring, and these tests pin the code to that reading by brute force.
"""
import itertools

import numpy as np
import pytest

from linear_attention_tree_b200 import budget as Bd
from linear_attention_tree_b200 import workloads as W
from oracle import oracle as O


def _walk_probability(parent, p, n):
    out = 1.0
    while n >= 0:
        out *= p[n]
        n = parent[n]
    return out


def _closed_subsets(parent):
    """Every ancestor-closed node set of one small tree, with its size."""
    n = len(parent)
    for mask in range(1 << n):
        keep = [i for i in range(n) if mask >> i & 1]
        if all(parent[i] < 0 or (mask >> parent[i] & 1) for i in keep):
            yield keep


def _best_by_size(parent, p, cap=None):
    """Brute force: best sum of walk probabilities over closed subsets of each size."""
    best = {}
    for keep in _closed_subsets(parent):
        if cap is not None and len(keep) > cap:
            continue
        val = sum(_walk_probability(parent, p, i) for i in keep)
        best[len(keep)] = max(best.get(len(keep), -1.0), val)
    return best


def _random_trees(rng, n_trees, max_n, ties=True):
    trees = []
    for _ in range(n_trees):
        n = int(rng.integers(0, max_n + 1))
        parent = W.uniform_parent_tree(rng, n, 4)
        p = rng.uniform(0.0, 1.0, n)
        if ties and n:
            p[rng.random(n) < 0.3] = 1.0      # equal path probabilities down a chain
            p[rng.random(n) < 0.1] = 0.0
            p = np.round(p, 1)                 # many exact ties across trees
        trees.append((parent, p))
    return trees


def _closed(parent, keep):
    ks = set(int(x) for x in keep)
    return all(parent[i] < 0 or parent[i] in ks for i in ks)


def test_path_probability_is_the_product_along_the_path():
    rng = np.random.default_rng(1)
    for _ in range(20):
        parent, p = _random_trees(rng, 1, 30, ties=False)[0]
        P = Bd.path_probability(parent, p)
        for i in range(len(parent)):
            assert P[i] == pytest.approx(_walk_probability(parent, p, i), rel=1e-12)
            if parent[i] >= 0:
                assert P[i] <= P[parent[i]]
    with pytest.raises(ValueError):
        Bd.path_probability([-1, 1], [0.5, 0.5])
    with pytest.raises(ValueError):
        Bd.path_probability([-1], [1.5])


@pytest.mark.parametrize("cap", [None, 2, 4])
def test_greedy_selection_is_optimal_by_brute_force(cap):
    rng = np.random.default_rng(7 if cap is None else cap)
    for trial in range(40):
        trees = _random_trees(rng, int(rng.integers(1, 4)), 7)
        per_tree = [_best_by_size(par, p, cap) for par, p in trees]
        total = sum(max(b) for b in per_tree)
        for budget in range(total + 2):
            keeps = Bd.select_nodes(trees, budget, cap=cap)
            assert sum(len(k) for k in keeps) == min(budget, total)
            for (par, _), k in zip(trees, keeps):
                assert _closed(par, k)
                assert cap is None or len(k) <= cap
            brute = max(sum(b[c] for b, c in zip(per_tree, combo))
                        for combo in itertools.product(*[sorted(b) for b in per_tree])
                        if sum(combo) <= budget)
            got = Bd.expected_tokens(trees, keeps) - len(trees)
            assert got == pytest.approx(brute, abs=1e-12), (trial, budget)


def test_reserve_keeps_every_tree_alive():
    rng = np.random.default_rng(3)
    trees = _random_trees(rng, 6, 9)
    need = sum(min(2, len(par)) for par, _ in trees)
    keeps = Bd.select_nodes(trees, need + 3, min_nodes=2)
    for (par, _), k in zip(trees, keeps):
        assert len(k) >= min(2, len(par)) and _closed(par, k)
    assert sum(len(k) for k in keeps) == min(need + 3, sum(len(par) for par, _ in trees))
    with pytest.raises(ValueError):
        Bd.select_nodes(trees, need - 1, min_nodes=2)


def _cap_loop(sizes, budget):
    n = list(sizes)
    while sum(n) > budget:
        j = int(np.argmax(n))
        n[j] -= 1
    return n


def test_cap_largest_equals_its_loop():
    rng = np.random.default_rng(11)
    for _ in range(300):
        sizes = rng.integers(0, 20, size=int(rng.integers(1, 12)))
        budget = int(rng.integers(0, int(sizes.sum()) + 5))
        assert list(Bd.cap_largest(sizes, budget)) == _cap_loop(list(sizes), budget)


def test_cap_largest_reproduces_the_ragged_workload():
    """The ragged workload draws 128 sizes U{8..48} as the first draw of its data generator
    (PCG64 seeded 1000·4 + seed) and shrinks the largest until they sum to 3072."""
    for seed in (0, 1):
        raw = np.random.Generator(np.random.PCG64(4000 + seed)).integers(8, 49, size=128)
        w = W.config(4, seed)
        assert list(Bd.cap_largest(raw, 3072)) == [int(x) for x in np.diff(w.node_offsets)]


def test_prune_and_pack():
    parents = [[-1, 0, 0, 1, -1, 4], [-1, -1, 1], []]
    keeps = [[0, 1, 3, 4], [1, 2], []]
    par, offs, rows = Bd.pack(parents, keeps)
    assert list(par) == [-1, 0, 1, -1, -1, 0]
    assert list(offs) == [0, 4, 6, 6]
    assert list(rows) == [0, 1, 3, 4, 7, 8]
    with pytest.raises(ValueError):
        Bd.prune([-1, 0, 1], [0, 2])        # node 2's parent is not kept
    with pytest.raises(ValueError):
        Bd.prune([-1, 0, 1], [1, 0])        # not ascending


def test_pruned_batch_has_the_full_batch_outputs_at_kept_nodes():
    """Outputs of a node depend on its root path only, so the oracle on the pruned batch
    must reproduce the unpruned batch's o and U at every kept node."""
    parents = [W.frontier_tree(50 + s, n, 5, 3)[0] for s, n in enumerate([9, 14, 6])]
    w = W.synthetic(parents, 2, 16, 16, seed=5, in_dtype="f32")
    trees = [(par, W.acceptance_estimates(par, 20 + s)) for s, par in enumerate(parents)]
    keeps = Bd.select_nodes(trees, 15, min_nodes=1)
    par, offs, rows = Bd.pack(parents, keeps)
    ws = w.subset(par, offs, rows)
    o_full, U_full = O.tree_verify(w)
    o_sub, U_sub = O.tree_verify(ws)
    np.testing.assert_array_equal(o_sub, o_full[rows])
    np.testing.assert_array_equal(U_sub, U_full[rows])


def test_cost_model_fit_recovers_its_coefficients():
    true = Bd.CostModel(tc=(5.0, 0.03, 0.0004), wide=(7.0, 0.02, 0.0002, 0.09))
    rng = np.random.default_rng(2)
    samples = []
    for _ in range(30):
        B = int(rng.integers(1, 200))
        hi = int(rng.choice([8, 64, 256]))
        sizes = list(rng.integers(1, hi + 1, size=B))
        samples.append((sizes, 32, true.predict_us(sizes, 32)))
    got = Bd.CostModel.fit(samples)
    np.testing.assert_allclose(got.tc, true.tc, rtol=1e-6)
    np.testing.assert_allclose(got.wide, true.wide, rtol=1e-6)
    assert Bd.CostModel.features([64, 3], 8)[0] == "tc"
    assert Bd.CostModel.features([65, 3], 8)[0] == "wide"
    assert list(Bd.CostModel.features([65, 3], 8)[1]) == [1, 16, 544, 24]


def _scan(trees, H, model, fixed, layers, min_nodes):
    """Every (value, µs) of the greedy allocations for every node budget, capped and not."""
    out = []
    total = sum(len(par) for par, _ in trees)
    for cap in (Bd.TC_MAX_NODES, None):
        for n in range(sum(min(min_nodes, len(par)) for par, _ in trees), total + 1):
            keeps = Bd.select_nodes(trees, n, cap=cap, min_nodes=min_nodes)
            sizes = [len(k) for k in keeps]
            out.append((Bd.expected_tokens(trees, keeps),
                        fixed + layers * model.predict_us(sizes, H)))
    return out


def test_time_budget_and_chosen_budget_match_an_exhaustive_scan():
    model = Bd.CostModel(tc=(6.0, 0.03, 0.0008), wide=(6.0, 0.05, 0.0008, 0.1))
    rng = np.random.default_rng(5)
    parents = [W.frontier_tree(300 + s, int(n), 8, 4)[0]
               for s, n in enumerate(rng.integers(20, 120, size=6))]
    trees = [(par, W.acceptance_estimates(par, s)) for s, par in enumerate(parents)]
    scan = _scan(trees, 32, model, 0.0, 1, 1)
    for budget_us in (8.0, 10.0, 14.0, 30.0):
        fits = [v for v, us in scan if us <= budget_us]
        if not fits:
            with pytest.raises(ValueError):
                Bd.allocate_time(trees, 32, budget_us, model)
            continue
        keeps, us, value = Bd.allocate_time(trees, 32, budget_us, model)
        assert us <= budget_us
        assert value == pytest.approx(max(fits), rel=1e-12)
        assert value == pytest.approx(Bd.expected_tokens(trees, keeps), rel=1e-12)
        assert all(_closed(par, k) for (par, _), k in zip(trees, keeps))
    for fixed, layers in ((0.0, 1), (40.0, 1), (400.0, 24)):
        scan = _scan(trees, 32, model, fixed, layers, 1)
        best = max(v / us for v, us in scan)
        got = Bd.choose_budget(trees, 32, model, fixed_us=fixed, layers=layers)
        assert got["tokens_per_us"] == pytest.approx(best, rel=1e-12)
        assert got["budget"] == sum(len(k) for k in got["keeps"])
    # A costlier rest of the step buys a larger verification budget.
    small = Bd.choose_budget(trees, 32, model, fixed_us=0.0)["budget"]
    large = Bd.choose_budget(trees, 32, model, fixed_us=2000.0)["budget"]
    assert large >= small


def test_edge_cases():
    assert Bd.select_nodes([], 5) == []
    assert [len(k) for k in Bd.select_nodes([([], [])], 5)] == [0]
    # equal (zero) probabilities: the shallower node first, then the next tree
    keeps = Bd.select_nodes([([-1, 0], [0.0, 0.0]), ([-1], [1.0])], 2)
    assert [list(k) for k in keeps] == [[0], [0]]
    assert [len(k) for k in Bd.select_nodes([([-1, 0, 0], [0.5] * 3)], 3, cap=0)] == [0]
    # a reserve larger than a tree keeps the whole tree
    assert [list(k) for k in Bd.select_nodes([([-1, 0], [0.5, 0.5])], 2, min_nodes=5)] == [[0, 1]]
    assert list(Bd.cap_largest([], 3)) == [] and list(Bd.cap_largest([3, 3], 0)) == [0, 0]
    par, offs, rows = Bd.pack([], [])
    assert len(par) == 0 and list(offs) == [0] and len(rows) == 0
    assert Bd.B200_DEFAULT.predict_us([], 32) == pytest.approx(Bd.B200_DEFAULT.tc[0])
    with pytest.raises(ValueError):
        Bd.allocate_time([([-1, 0], [0.5, 0.5])], 32, 1.0)
    with pytest.raises(ValueError):
        Bd.select_nodes([([-1], [0.5])], -1)
