"""Pins of the oracle's PHAROS selection variants and of its selection trace.

PHAROS page ("Four mechanisms powering PHAROS"): depth-sounding budget
allocation (DBA) gives heads different token budgets, fog-gate confidence
fallback (FCF) expands the budget when confidence is low, range-light
cross-level guidance (RCG) lets coarse-level information guide finer-level
selection. The readings (tests/golden/walk_variants.txt states them in full):
  DBA  a per-(batch, kv head) level-0 budget;
  FCF  confidence = the walk's smallest margin above level 0 and at the level-0
       budget boundary; below tau, level 0 keeps `extra` more blocks;
  RCG  candidates rank by R = S + lambda R(parent).

Pinned by: hand-derived walks (golden file); reductions to the plain walk that
fix every variant's end points (lambda = 0; tau = -inf and +inf; budget = topk
for every unit; a unit's budget k equals the plain walk with topk = k); and the
trace's structure (every kept node is a child of a node kept one level up, each
level keeps the right count, level 0 is idx).
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import F32, Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def W(**kw):
    base = dict(name="t", B=1, Hq=1, Hkv=1, N=256, Nq=256, q_offset=0, d=8, b=16, topk=2, cap=4, dtype=F32, seed=0,
                n_needle=0, needle_mode=0)
    base.update(kw)
    return Workload(**base)


def rand_qk(w, seed, k_scale=1.2):
    Q = synth.normal(seed, 10, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    K = synth.normal(seed, 11, (w.B, w.Hkv, w.N, w.d), w.torch_dtype, scale=k_scale)
    return Q, K


def _read_variants():
    cases = []
    with open(os.path.join(GOLDEN, "walk_variants.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, keys, i, cap, topk, budget, tau, extra, lam, idx, gap = line.split()
            cases.append(dict(name=name, keys=[float(x) for x in keys.split(",")], i=int(i), cap=int(cap),
                              topk=int(topk), budget=None if budget == "-" else int(budget), tau=float(tau),
                              extra=int(extra), lam=float(lam), idx=[int(x) for x in idx.split(",")],
                              gap=float(gap)))
    return cases


@pytest.mark.parametrize("c", _read_variants(), ids=lambda c: c["name"])
def test_variant_hand_derived_examples(c):
    w = W(N=9, Nq=9, d=1, b=1, topk=c["topk"], cap=c["cap"])
    Q = torch.ones((1, 1, 9, 1), dtype=torch.float32)
    K = torch.tensor(c["keys"], dtype=torch.float32).reshape(1, 1, 9, 1)
    pyr = oracle.pyramid(w, K, [0])
    opts = oracle.SelectOpts(budget=None if c["budget"] is None else [c["budget"]], fcf_tau=c["tau"],
                             fcf_extra=c["extra"], rcg_lambda=c["lam"])
    idx, gap, _ = oracle.select(w, Q, pyr, [0], [(0, c["i"])], opts=opts)
    assert idx[0].tolist() == c["idx"]
    assert abs(gap[0] - c["gap"]) < 1e-5, gap[0]


SHAPES = [
    W(B=2, Hq=4, Hkv=2, N=1024, Nq=1024, b=16, d=16, topk=6, cap=8),   # nb = 64, GQA
    W(B=1, Hq=2, Hkv=2, N=1000, Nq=1000, b=16, d=8, topk=5, cap=10),   # ragged
    W(B=2, Hq=4, Hkv=1, N=2048, Nq=1, q_offset=2047, b=32, d=16, topk=6, cap=8),  # decode
]


def _all(w, Q, K, opts=None, with_trace=False):
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    nqb = oracle.num_qblocks(w)
    items = [(u, q) for u in units for q in range(nqb)]
    return oracle.select(w, Q, pyr, units, items, opts=opts, with_trace=with_trace)


def _pad(idx, width):
    out = -np.ones((idx.shape[0], width), dtype=np.int32)
    out[:, :idx.shape[1]] = idx
    return out


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_rcg_with_zero_lambda_is_the_plain_walk(w):
    Q, K = rand_qk(w, 3)
    i0, g0, _ = _all(w, Q, K)
    i1, g1, _ = _all(w, Q, K, oracle.SelectOpts(rcg_lambda=0.0))
    assert np.array_equal(i0, i1) and np.array_equal(g0, g1)


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_rcg_changes_routes_when_guided(w):
    """Guidance is not a no-op: with lambda = 1 some rows change (inputs with varied node means)."""
    Q, K = rand_qk(w, 3)
    i0, _, _ = _all(w, Q, K)
    i1, _, _ = _all(w, Q, K, oracle.SelectOpts(rcg_lambda=1.0))
    assert (i0 != i1).any(axis=1).sum() > 0


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_fcf_end_points_are_plain_walks(w):
    """tau = -inf never expands (plain walk with topk = budget); tau = +inf always expands (plain walk
    with topk = budget + extra); idx and gap both match."""
    Q, K = rand_qk(w, 4)
    extra = 2
    base_w, wide_w = w.scaled(topk=w.topk - extra), w
    ib, gb, _ = _all(base_w, Q, K)
    iw, gw, _ = _all(wide_w, Q, K)
    lo, glo, _ = _all(w, Q, K, oracle.SelectOpts(fcf_tau=-np.inf, fcf_extra=extra))
    hi, ghi, _ = _all(w, Q, K, oracle.SelectOpts(fcf_tau=np.inf, fcf_extra=extra))
    assert np.array_equal(lo, _pad(ib, w.topk)) and np.array_equal(glo, gb)
    assert np.array_equal(hi, iw) and np.array_equal(ghi, gw)


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_fcf_expands_exactly_the_rows_below_tau(w):
    """Between the end points each row is the narrow or the wide plain walk, according to its confidence."""
    Q, K = rand_qk(w, 5)
    extra = 2
    ib, gb, _ = _all(w.scaled(topk=w.topk - extra), Q, K)
    iw, _, _ = _all(w, Q, K)
    tau = float(np.median(gb[np.isfinite(gb)]))
    got, _, _ = _all(w, Q, K, oracle.SelectOpts(fcf_tau=tau, fcf_extra=extra))
    # the confidence of a row is the plain narrow walk's gap (its margins above level 0 and at the budget)
    narrow = _pad(ib, w.topk)
    n_wide = 0
    for r in range(len(got)):
        want = iw[r] if gb[r] < tau else narrow[r]
        n_wide += int(gb[r] < tau and not np.array_equal(iw[r], narrow[r]))
        assert np.array_equal(got[r], want), (r, got[r], want, gb[r], tau)
    assert n_wide > 0


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_dba_budget_per_unit_is_the_plain_walk_at_that_topk(w):
    Q, K = rand_qk(w, 6)
    U = w.B * w.Hkv
    budget = [(u % w.topk) + 1 for u in range(U)]
    budget[0] = 0
    got, _, _ = _all(w, Q, K, oracle.SelectOpts(budget=budget))
    nqb = oracle.num_qblocks(w)
    got = got.reshape(U, nqb, w.topk)
    for u in range(U):
        k = budget[u]
        if k == 0:
            assert (got[u] == -1).all()
            continue
        ref, _, _ = oracle.select_all(w.scaled(topk=k), Q, K, units=[u])
        assert np.array_equal(got[u], _pad(ref[0], w.topk))
    full, _, _ = _all(w, Q, K, oracle.SelectOpts(budget=[w.topk] * U))
    plain, _, _ = _all(w, Q, K)
    assert np.array_equal(full, plain)


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
@pytest.mark.parametrize("opts", [None, oracle.SelectOpts(fcf_tau=0.3, fcf_extra=2, rcg_lambda=0.5)],
                         ids=["plain", "fcf_rcg"])
def test_trace_structure(w, opts):
    Q, K = rand_qk(w, 7)
    idx, _, ncand, trace = _all(w, Q, K, opts, with_trace=True)
    nb = w.nb
    lv = [n for _, n in oracle.level_offsets(w)]
    s0 = oracle.trace_levels(w) - 1
    assert lv[s0] <= w.cap and (s0 == 0 or lv[s0 - 1] > w.cap)
    first = w.q_offset // w.b
    nqb = oracle.num_qblocks(w)
    for r in range(len(idx)):
        i = first + r % nqb
        cands = [m for m in range(lv[s0]) if (m << s0) < i]
        for k, l in enumerate(range(s0, -1, -1)):
            row = trace[r, k]
            kept = [int(x) for x in row if x >= 0]
            assert (row[len(kept):] == -1).all()
            assert len(set(kept)) == len(kept) and set(kept) <= set(cands)
            assert len(cands) == ncand[r, l]
            if l > 0:
                assert len(kept) == min(w.cap // 2, len(cands))
                cands = sorted(ch for m in kept for ch in (2 * m, 2 * m + 1) if ch < lv[l - 1] and (ch << (l - 1)) < i)
            else:
                assert sorted(kept) == [int(x) for x in idx[r] if x >= 0]
    assert nb == lv[0]
