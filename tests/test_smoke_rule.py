"""The routing rule of __graft_entry__.smoke(): the GPU's index equals the oracle's except at
near-ties (within 1e-5 of the dot product's term magnitudes). Checked here on the CPU with
indices made from the oracle's own: the exact index passes, the closest pair of consecutive
ranks swapped passes, a region outside the top-k fails."""
import math

import numpy as np

import __graft_entry__ as entry
import oracle
from bi_level_routing_b200.workloads import WORKLOADS, make_inputs


def _case():
    w = WORKLOADS["stage2"].with_(B=2)
    inp = make_inputs(w)
    ref, A = oracle.route(inp["q"], inp["k"], w.n_win, w.topk, want_affinity=True)
    qm, km = oracle.region_means(inp["q"], w.n_win), oracle.region_means(inp["k"], w.n_win)
    return w, ref, A, qm, km


def test_smoke_routing_rule():
    w, ref, A, qm, km = _case()
    assert entry._routing_mismatches(ref, ref, A, qm, km) == []
    # the closest pair of consecutive ranks inside the top-k, swapped: a near-tie
    best = None
    for b in range(w.B):
        mag = np.abs(qm[b]) @ np.abs(km[b]).T / math.sqrt(qm.shape[-1])
        for r in range(w.R):
            o = np.argsort(-A[b, r], kind="stable")
            for j in range(w.topk - 1):
                gap = abs(A[b, r, o[j]] - A[b, r, o[j + 1]]) / max(mag[r, o[j]], mag[r, o[j + 1]])
                if best is None or gap < best[0]:
                    best = (gap, b, r, j)
    gap, b, r, j = best
    assert gap < entry.ROUTE_REL_TOL
    swapped = ref.copy()
    swapped[b, r, j], swapped[b, r, j + 1] = ref[b, r, j + 1], ref[b, r, j]
    assert entry._routing_mismatches(swapped, ref, A, qm, km) == []
    # a region outside the row's top-k in place of its last one
    wrong = ref.copy()
    wrong[0, 0, -1] = next(s for s in range(w.R) if s not in ref[0, 0])
    assert entry._routing_mismatches(wrong, ref, A, qm, km) == [(0, 0)]
    # a repeated region
    rep = ref.copy()
    rep[1, 3, 1] = rep[1, 3, 0]
    assert entry._routing_mismatches(rep, ref, A, qm, km) == [(1, 3)]
