"""The batch-wide budget on the GPU: a cost model calibrated on this GPU predicts the verify
time of batches it was not fitted on, and a pruned batch verifies to the oracle's outputs and
to the unpruned batch's outputs at every kept node."""
import numpy as np
import pytest

from linear_attention_tree_b200 import budget as Bd
from linear_attention_tree_b200 import workloads as W
from oracle import oracle as O
from tests._gpu_util import TOL, assert_close, run

pytestmark = pytest.mark.gpu


def test_calibrated_model_predicts_unseen_batches():
    model, samples = Bd.calibrate(launches=8)
    for sizes, H, us in samples:                       # the fit itself
        assert model.predict_us(sizes, H) == pytest.approx(us, rel=0.25)
    held_out = [W.config(3, 1), W.config(4, 1), W.config(5, 1),
                Bd.calibration_workload(48, 20, 60, seed=9),
                Bd.calibration_workload(6, 90, 220, 9, 6, seed=9)]
    for w in held_out:
        sizes = [int(x) for x in np.diff(w.node_offsets)]
        us = Bd.measure_us(w, launches=8)
        pred = model.predict_us(sizes, w.H)
        assert pred == pytest.approx(us, rel=0.25), (w.name, pred, us)


@pytest.mark.parametrize("budget", [160, 300])
def test_pruned_batch_verifies_like_the_full_batch(budget):
    counts = [90, 40, 64, 120, 8, 30]
    parents = [W.frontier_tree(700 + s, n, 8, 4)[0] for s, n in enumerate(counts)]
    w = W.synthetic(parents, 4, 128, 128, seed=71)
    trees = [(par, W.acceptance_estimates(par, 80 + s)) for s, par in enumerate(parents)]
    keeps = Bd.select_nodes(trees, budget, min_nodes=1)
    par, offs, rows = Bd.pack(parents, keeps)
    ws = w.subset(par, offs, rows)
    assert ws.T == budget
    got, _ = run(ws)
    o, U = O.tree_verify(ws)
    assert_close(got["o"], o, TOL["bf16"], "o")
    assert_close(got["U"], U, TOL["bf16"], "U")
    assert_close(got["S_new"], O.tree_commit(ws), TOL["bf16"], "S_new")
    full, _ = run(w, commit=False)
    assert_close(got["o"], full["o"][rows], TOL["bf16"], "o against the full batch")
    assert_close(got["U"], full["U"][rows], TOL["bf16"], "U against the full batch")
