"""The tie-tolerant walk that judges GPU rows inside the gap exemption (tests/_parity.py).

A selection row whose oracle gap is under 1e-4 may come out differently on the
GPU, whose fp32 scores differ from the oracle's double ones by a few 1e-5. Such
a row is accepted only if the walk can reach it when every comparison between
two oracle scores within TIE_EPS of each other may go either way. Pinned here,
on the CPU, against the oracle itself:
  - with eps = 0 the oracle's own result is reachable (no exact ties in these inputs);
  - where every level's margin exceeds eps, no other valid row is reachable;
  - a pyramid perturbed by noise well under eps/2 per score makes the oracle pick
    other rows, and every one of them is reachable (the call the GPU tests make);
  - a perturbation ten times larger yields rows that are not (the check is not vacuous);
  - an exhausted search reports None instead of an answer.
"""
import numpy as np
import pytest

import oracle
import synth
from _parity import GAP_EXEMPT, TIE_EPS, check_exempt_rows, check_traces, validate_trace, walk_reaches

W32 = synth.BY_NAME["mha_bf16_32k"]


@pytest.fixture(scope="module")
def w32():
    w = W32
    Q, K, V, _ = synth.generate(w)
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    items = [(u, q) for u in units for q in range(oracle.num_qblocks(w))]
    idx, gap, _ = oracle.select(w, Q, pyr, units, items)
    return w, Q, pyr, units, items, idx, gap


def test_own_result_is_reachable_with_no_slack():
    w = synth.WORKLOADS[0]
    Q, K, V, _ = synth.generate(w)
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    items = [(u, q) for u in units for q in range(oracle.num_qblocks(w))]
    idx, _, _ = oracle.select(w, Q, pyr, units, items)
    for k, (u, q) in enumerate(items):
        assert walk_reaches(w, Q, pyr[u], u, q, idx[k], 0.0) is True, (u, q)


def _swapped(w, q, row, rng):
    """A valid row (ascending, before block i, same count) that differs from `row` in one block."""
    i = w.q_offset // w.b + q
    kept = [int(x) for x in row if x >= 0]
    others = [j for j in range(i) if j not in kept]
    if not kept or not others:
        return None
    out = sorted(set(kept) - {kept[rng.integers(len(kept))]} | {others[rng.integers(len(others))]})
    return np.array(out + [-1] * (w.topk - len(out)), dtype=np.int32)


def test_rows_with_clear_margins_admit_only_the_oracle_result(w32):
    w, Q, pyr, units, items, idx, gap = w32
    rng = np.random.default_rng(3)
    clear = [k for k in np.nonzero(gap > 4 * TIE_EPS)[0]]
    assert len(clear) > 1000
    tried = 0
    for k in rng.choice(clear, 150, replace=False):
        u, q = items[k]
        assert walk_reaches(w, Q, pyr[u], u, q, idx[k], TIE_EPS) is True
        alt = _swapped(w, q, idx[k], rng)
        if alt is None:
            continue
        tried += 1
        assert walk_reaches(w, Q, pyr[u], u, q, alt, TIE_EPS) is False, (u, q, idx[k], alt)
    assert tried > 100


def test_rows_from_scores_within_half_the_slack_are_all_reachable(w32):
    w, Q, pyr, units, items, idx, gap = w32
    rng = np.random.default_rng(7)
    # node means moved by N(0, 3e-5^2) per element move each score by about 3e-5, well under TIE_EPS / 2
    moved = pyr + rng.normal(0.0, 3e-5, pyr.shape)
    idx2, _, _ = oracle.select(w, Q, moved, units, items)
    differ = int((~(idx2 == idx).all(axis=1)).sum())
    assert differ >= 10
    assert (gap[~(idx2 == idx).all(axis=1)] < GAP_EXEMPT).all()
    differing, reached, undecided = check_exempt_rows(w, Q, pyr, units, items, idx2, idx, gap)
    assert (differing, reached, undecided) == (differ, differ, 0)


def test_rows_from_much_larger_score_errors_are_not_all_reachable(w32):
    w, Q, pyr, units, items, idx, gap = w32
    rng = np.random.default_rng(7)
    moved = pyr + rng.normal(0.0, 1e-3, pyr.shape)
    idx2, _, _ = oracle.select(w, Q, moved, units, items)
    rows = np.nonzero(~(idx2 == idx).all(axis=1))[0][:300]
    answers = [walk_reaches(w, Q, pyr[items[k][0]], items[k][0], items[k][1], idx2[k], TIE_EPS) for k in rows]
    assert answers.count(False) >= 20 and answers.count(None) == 0


def test_search_bound_reports_undecided(w32):
    w, Q, pyr, units, items, idx, gap = w32
    k = int(np.nonzero(gap < GAP_EXEMPT)[0][-1])
    u, q = items[k]
    assert walk_reaches(w, Q, pyr[u], u, q, idx[k], TIE_EPS, max_states=1) is None


# ---- the trace check (validate_trace / check_traces), which decides every exempt row ----------

def _traced(w, Q, pyr, units, items, opts=None):
    return oracle.select(w, Q, pyr, units, items, opts=opts, with_trace=True)


@pytest.mark.parametrize("opts", [None, oracle.SelectOpts(fcf_tau=0.5, fcf_extra=2, rcg_lambda=0.3)],
                         ids=["plain", "fcf_rcg"])
def test_oracle_trace_is_a_valid_walk_with_no_slack(opts):
    w = synth.WORKLOADS[0].scaled(topk=10, cap=16)
    Q, K, V, _ = synth.generate(w)
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    items = [(u, q) for u in units for q in range(oracle.num_qblocks(w))]
    idx, gap, _, trace = _traced(w, Q, pyr, units, items, opts)
    for k, (u, q) in enumerate(items):
        ok, msg = validate_trace(w, Q, pyr[u], u, q, trace[k], idx[k], 0.0, opts)
        assert ok, (u, q, msg)


def test_tampered_traces_fail(w32):
    w, Q, pyr, units, items, _, _ = w32
    rng = np.random.default_rng(11)
    idx, gap, _, trace = _traced(w, Q, pyr, units, items)
    clear = [k for k in np.nonzero(gap > 4 * TIE_EPS)[0] if items[k][1] > w.topk + 2]
    n_rank = n_idx = n_count = 0
    for k in rng.choice(clear, 60, replace=False):
        u, q = items[k]
        cache = {}
        # level 0: swap the worst kept block for the best dropped one (margin > 4 eps)
        t = trace[k].copy()
        lv0 = t[-1]
        kept = [int(x) for x in lv0 if x >= 0]
        lv = [n for _, n in oracle.level_offsets(w)]
        i = q
        cands = sorted(ch for m in t[-2] if m >= 0 for ch in (2 * m, 2 * m + 1) if ch < lv[0] and ch < i)
        dropped = [m for m in cands if m not in kept]
        if dropped:
            sc = {m: oracle.node_score(w, Q, pyr[u], u, q, 0, m)[0] for m in cands}
            worst = min(kept, key=lambda m: sc[m])
            best = max(dropped, key=lambda m: sc[m])
            t2 = t.copy()
            t2[-1][list(lv0).index(worst)] = best
            new = sorted(set(kept) - {worst} | {best})
            idx2 = np.array(new + [-1] * (w.topk - len(new)), dtype=np.int32)
            ok, msg = validate_trace(w, Q, pyr[u], u, q, t2, idx2, TIE_EPS, score_cache=cache)
            assert not ok and "ranks" in msg, msg
            n_rank += 1
        # idx that is not the level-0 kept set
        alt = _swapped(w, q, idx[k], rng)
        if alt is not None:
            ok, msg = validate_trace(w, Q, pyr[u], u, q, trace[k], alt, TIE_EPS, score_cache=cache)
            assert not ok and "idx" in msg, msg
            n_idx += 1
        # one node too few at the start level
        t3 = trace[k].copy()
        first_row = t3[0]
        if (first_row >= 0).sum() > 1:
            first_row[(first_row >= 0).sum() - 1] = -1
            ok, msg = validate_trace(w, Q, pyr[u], u, q, t3, idx[k], TIE_EPS, score_cache=cache)
            assert not ok, msg
            n_count += 1
    assert n_rank > 20 and n_idx > 20 and n_count > 20


def test_walks_from_scores_within_half_the_slack_all_validate(w32):
    """The GPU's situation: fp32 scores a few 1e-5 off the oracle's. Every differing row is decided."""
    w, Q, pyr, units, items, _, _ = w32
    rng = np.random.default_rng(7)
    idx, gap, _, trace = _traced(w, Q, pyr, units, items)
    moved = pyr + rng.normal(0.0, 3e-5, pyr.shape)
    idx2, _, _, trace2 = _traced(w, Q, moved, units, items)
    counts = check_traces(w, Q, pyr, units, items, idx2, trace2, idx, gap, trace)
    assert counts["differing"] >= 10 and counts["validated"] >= counts["differing"]


def test_walks_from_much_larger_score_errors_fail_the_trace_check(w32):
    w, Q, pyr, units, items, _, _ = w32
    rng = np.random.default_rng(7)
    idx, gap, _, trace = _traced(w, Q, pyr, units, items)
    moved = pyr + rng.normal(0.0, 1e-3, pyr.shape)
    idx2, _, _, trace2 = _traced(w, Q, moved, units, items)
    rows = np.nonzero(~(idx2 == idx).all(axis=1))[0][:300]
    bad = sum(not validate_trace(w, Q, pyr[items[k][0]], items[k][0], items[k][1], trace2[k], idx2[k], TIE_EPS)[0]
              for k in rows)
    assert bad >= 20
