"""The parity tests' selection check, exercised on the CPU: the oracle's own
selection passes; on a row flagged as a near tie, taking the other side of
the tie passes; any invalid selection (wrong size, duplicate, an index outside
the candidates, a clearly worse pick, or a change on an unflagged row) fails."""

import numpy as np
import pytest

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

from hga_testlib import check_selection


@pytest.fixture(scope="module")
def case():
    w = synth.custom(n_q_heads=8, n_kv_heads=2, head_dim=128, ctx_len=8192, seg_len=2048,
                     topk_blocks=4, topk_groups=16, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=3, first_seg=3)
    q_begin = w.segments()[0]
    k64 = synth.widen(synth.keys(w), w.dtype)
    q64 = synth.widen(synth.queries(w, q_begin), w.dtype)
    g, b = oracle.build_summaries(k64, 0, q_begin + w.seg_len)
    sb, sg, tie = oracle.route(q64, b, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    assert tie.any() and (~tie).any()
    return w, q_begin, q64, g, b, sb, sg, tie


def run(case, sb, sg):
    w, q_begin, q64, g, b = case[:5]
    return check_selection(sb, sg, q64, b, g, q_begin, w, w.n_kv_heads)


def other_side_of_tie(case, row):
    """The level-2 selection of a flagged row with its k-th group swapped for
    the (k+1)-th (the two are within the tie window)."""
    w, q_begin, q64, g, b, sb, sg, tie = case
    bb, h, j = row
    G = w.group_heads
    qbar = q64[bb, h * G:(h + 1) * G, 64 * j:64 * j + 64].reshape(-1, w.head_dim).mean(0)
    blocks = sb[bb, h, j][sb[bb, h, j] >= 0]
    groups = np.array([8 * c + i for c in blocks for i in range(8)])
    s = g[bb, h, groups] @ qbar
    order = np.lexsort((groups, -s))
    kg = w.topk_groups
    a, c = s[order[kg - 1]], s[order[kg]]
    if abs(a - c) > 1e-3 * max(abs(a), abs(c)):
        return None                                   # the tie was at level 1
    new = set(sg[bb, h, j].tolist())
    new.discard(int(groups[order[kg - 1]]))
    new.add(int(groups[order[kg]]))
    return sorted(new), groups[order[-1]]


def flagged_level2_row(case):
    for row in np.argwhere(case[7]):
        alt = other_side_of_tie(case, tuple(row))
        if alt is not None:
            return tuple(row), alt
    pytest.skip("no level-2 near tie in this case")


def test_oracle_selection_passes(case):
    flagged, differ = run(case, case[5], case[6])
    assert flagged == int(case[7].sum()) and differ == 0


def test_other_side_of_a_tie_passes(case):
    row, (alt, _) = flagged_level2_row(case)
    sg = case[6].copy()
    sg[row] = alt
    assert run(case, case[5], sg)[1] == 1


@pytest.mark.parametrize("how", ["duplicate", "short", "outside", "worst", "unflagged",
                                 "descending"])
def test_invalid_selections_fail(case, how):
    row, (alt, worst) = flagged_level2_row(case)
    sb, sg = case[5].copy(), case[6].copy()
    r = sg[row].copy()
    if how == "duplicate":
        r[1] = r[0]
    elif how == "short":
        r[-1] = -1
    elif how == "outside":
        r[-1] = 8 * (case[1] // 64 + 5)               # a group of a later block
    elif how == "worst":
        r = np.array(sorted(set(r.tolist()) - {int(r[-1])} | {int(worst)}))
    elif how == "descending":
        r = r[::-1].copy()
    elif how == "unflagged":
        row = tuple(np.argwhere(~case[7])[0])
        r = sg[row].copy()
        r[0], r[1] = r[1], r[0]
    sg[row] = r
    with pytest.raises(AssertionError):
        run(case, sb, sg)
