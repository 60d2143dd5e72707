"""Host logic of the parity rules (CPU)."""
import numpy as np

from parity_utils import hq_close, rel_l2, routing_mismatches


def test_routing_rule_accepts_exact_and_near_ties_only():
    sel = np.array([[0.9, 0.5, 0.5 + 1e-8, 0.1], [0.9, 0.8, 0.7, 0.1]])
    orc = np.array([[0, 2], [0, 1]])
    assert routing_mismatches(orc, orc, sel) == ([], [])
    allowed, bad = routing_mismatches(np.array([[0, 1], [0, 1]]), orc, sel)
    assert allowed == [0] and bad == []
    allowed, bad = routing_mismatches(np.array([[0, 2], [0, 2]]), orc, sel)
    assert allowed == [] and bad == [1]
    allowed, bad = routing_mismatches(np.array([[0, 0], [0, 1]]), orc, sel)
    assert bad == [0]  # duplicate expert


def test_rel_l2_and_hq():
    assert rel_l2([1.0, 2.0], [1.0, 2.0]) == 0.0
    assert abs(rel_l2([1.0, 0.0], [0.0, 1.0]) - np.sqrt(2)) < 1e-12
    assert hq_close([1, 2, 3], [1, 3, 3]) == (1, 1 / 3)
