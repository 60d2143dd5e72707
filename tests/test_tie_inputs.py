"""The tying router inputs of the GPU tie-break tests can fail a wrong rule.

The GPU tests in test_gpu_ties.py compare routing indices exactly with the
oracle on inputs built to tie.  This CPU test checks that those inputs would
expose a top-k that broke ties the other way: on every case, choosing the
HIGHER index among equal selection values (computed here from the oracle's
own fp32 selection values by a plain sort) gives a different expert list from
the oracle's, and choosing the lower index gives the oracle's list.
"""
import numpy as np
import pytest

import test_gpu_ties as TT


def topk_by_sort(sel_row, k, prefer_low):
    E = sel_row.shape[0]
    order = sorted(range(E), key=lambda e: (-float(sel_row[e]), e if prefer_low else -e))
    return np.array(order[:k], np.int32)


@pytest.mark.parametrize("kind,E,k,T", TT.ROUTE_CASES)
def test_tie_inputs_expose_the_tie_rule(kind, E, k, T):
    wr, bias = TT.tie_router(E, 256, k, kind)
    x = TT.tie_tokens(T, 256)
    idx, _, sel = TT.oracle_route(x, wr, bias, k)
    for t in range(T):
        np.testing.assert_array_equal(topk_by_sort(sel[t], k, True), idx[t])
        assert not np.array_equal(topk_by_sort(sel[t], k, False), idx[t])
