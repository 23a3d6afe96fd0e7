"""Pins for the oracle's top-k router (CPU only): selection against numpy's
stable sort of the negated logits (ties to the lower expert id), weights
against torch's softmax / sigmoid in fp64 renormalised over the selection."""
import numpy as np
import pytest
import torch

import oracle as O


@pytest.mark.parametrize("T,E,k,scoring", [(64, 8, 2, "softmax"), (64, 48, 6, "sigmoid"), (33, 384, 6, "sigmoid"),
                                           (5, 4, 4, "softmax"), (7, 1024, 32, "softmax")])
def test_topk_matches_sort_and_library(T, E, k, scoring):
    rng = np.random.default_rng(E + k)
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    logits[0, :] = 0.25                       # all tied: ids 0..k-1
    logits[1, 1] = logits[1, 3] = 9.0         # a tie at the top: 1 before 3
    ids, w = O.topk(logits, k, scoring)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    np.testing.assert_array_equal(ids, order)
    assert ids[0].tolist() == list(range(k))
    if k >= 2:
        assert ids[1, :2].tolist() == [1, 3]
    sel = torch.from_numpy(np.take_along_axis(logits, order, axis=1)).double()
    ref = torch.softmax(sel, dim=1) if scoring == "softmax" else torch.sigmoid(sel) / torch.sigmoid(sel).sum(1, keepdim=True)
    np.testing.assert_allclose(w, ref.numpy(), rtol=1e-6, atol=0)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-6)


def test_topk_equals_topk_of_scores():
    """Selecting on logits equals selecting on softmax or sigmoid scores."""
    rng = np.random.default_rng(3)
    logits = rng.normal(0, 2, (50, 48)).astype(np.float32)
    for scoring, f in [("softmax", lambda x: torch.softmax(x.double(), 1)), ("sigmoid", lambda x: torch.sigmoid(x.double()))]:
        ids, _ = O.topk(logits, 6, scoring)
        _, ref = torch.topk(f(torch.from_numpy(logits)), 6, dim=1)
        np.testing.assert_array_equal(ids, ref.numpy())


def test_shared_slots_follow_the_routed_ones():
    """Shared-expert slots (reading R13): the routed slots are unchanged, then
    slot k + i holds expert E + i with weight exactly 1."""
    rng = np.random.default_rng(9)
    logits = rng.normal(0, 1, (40, 48)).astype(np.float32)
    for scoring in ("softmax", "sigmoid"):
        ids, w = O.topk(logits, 6, scoring)
        ids2, w2 = O.topk(logits, 6, scoring, num_shared=2)
        assert ids2.shape == (40, 8) and w2.shape == (40, 8)
        np.testing.assert_array_equal(ids2[:, :6], ids)
        np.testing.assert_array_equal(w2[:, :6], w)
        assert (ids2[:, 6] == 48).all() and (ids2[:, 7] == 49).all()
        assert (w2[:, 6:] == 1.0).all()
