"""Helpers shared by the GPU parity tests: run the CUDA path, compare with the oracle.

Acceptance (per the selection/attention contract):
  idx   bit-exact for every (batch, kv head, query block) whose oracle gap is
        >= GAP_EXEMPT; a row under it may differ, but then the walk must be able
        to end in the GPU's result when every comparison of two oracle scores
        within TIE_EPS of each other may go either way (`walk_reaches`);
  O     bf16: max-abs <= 2e-2 and relative L2 <= 1e-2; fp32: max-abs <= 1e-4;
  lse   bf16: max-abs <= 2e-3; fp32: max-abs <= 1e-4;
  pyr   fp32 accumulation against the double oracle: max-abs <= 2e-5 * (1 + |x|).
"""
from __future__ import annotations

import itertools
import math

import numpy as np
import torch

import hierarchical_block_sparse_pyr_b200 as P
import oracle
import synth

GAP_EXEMPT = 1e-4
# comparisons the walk may take either way when a GPU row differs inside the exemption: twice the
# exemption, i.e. per-score differences up to GAP_EXEMPT between the GPU's fp32 scores and the oracle's
TIE_EPS = 2 * GAP_EXEMPT
TOL = {synth.F32: dict(o_abs=1e-4, o_rel=1e-4, lse=1e-4), synth.BF16: dict(o_abs=2e-2, o_rel=1e-2, lse=2e-3)}


def to_dev(*ts):
    return [t.cuda() for t in ts]


def run_gpu(w, Q, K, V, idx=None, dense=False, opts=None, with_trace=False):
    """Run the CUDA path on CPU inputs. Returns a dict of CPU tensors.

    opts: an oracle.SelectOpts-like object (budget, fcf_tau, fcf_extra, rcg_lambda) whose values are
    passed to pyr_select_ex; with_trace adds the selection trace ("trace", [U, nqb, levels, width])."""
    s = P.shape_of(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    buf = P.Buffers(s)
    P.pyr_build(s, Kd, buf.pyr, buf.status)
    trace = P.new_trace(s) if with_trace else None
    if opts is None and trace is None:
        P.pyr_select(s, Qd, buf.pyr, buf.idx, buf.gap, buf.status)
    else:
        kw = {}
        if opts is not None:
            budget = None if opts.budget is None else torch.as_tensor(np.asarray(opts.budget, dtype=np.int32)).cuda()
            kw = dict(budget=budget, fcf_tau=opts.fcf_tau, fcf_extra=opts.fcf_extra, rcg_lambda=opts.rcg_lambda)
        P.pyr_select_ex(s, Qd, buf.pyr, buf.idx, buf.gap, trace=trace, status=buf.status, **kw)
    if dense:
        P.dense_forward(s, Qd, Kd, Vd, buf.O, buf.lse, buf.status)
    else:
        use = buf.idx if idx is None else torch.as_tensor(np.ascontiguousarray(idx), dtype=torch.int32).cuda()
        P.bsa_forward(s, Qd, Kd, Vd, use, buf.O, buf.lse, buf.status)
    torch.cuda.synchronize()
    out = dict(pyr=P.pyramid_means(s, buf.pyr).cpu(), idx=buf.idx.cpu(), gap=buf.gap.cpu(), O=buf.O.float().cpu(),
               lse=buf.lse.cpu(), status=int(buf.status.item()))
    if trace is not None:
        out["trace"] = trace.reshape(w.B * w.Hkv, trace.shape[2], trace.shape[3], trace.shape[4]).cpu()
    del buf, Qd, Kd, Vd
    return out


def check_pyramid(pyr_gpu_units: np.ndarray, pyr_ora: np.ndarray):
    err = np.abs(pyr_gpu_units - pyr_ora)
    bound = 2e-5 * (1.0 + np.abs(pyr_ora))
    assert (err <= bound).all(), f"pyramid max err {err.max():.3e}"


def check_select(idx_gpu: np.ndarray, idx_ora: np.ndarray, gap_ora: np.ndarray):
    """Returns (checked, exempt, exempt_differing)."""
    idx_gpu = idx_gpu.reshape(-1, idx_gpu.shape[-1])
    idx_ora = idx_ora.reshape(-1, idx_ora.shape[-1])
    gap_ora = gap_ora.reshape(-1)
    same = (idx_gpu == idx_ora).all(axis=1)
    exempt = gap_ora < GAP_EXEMPT
    bad = np.nonzero(~same & ~exempt)[0]
    assert len(bad) == 0, (f"{len(bad)} non-exempt rows differ; first: gpu {idx_gpu[bad[0]]} oracle "
                           f"{idx_ora[bad[0]]} gap {gap_ora[bad[0]]}")
    return int((~exempt).sum()), int(exempt.sum()), int((~same & exempt).sum())


def check_valid_idx(w, idx_gpu: np.ndarray):
    first = w.q_offset // w.b
    nqb = idx_gpu.shape[-2]
    for qb in range(nqb):
        i = first + qb
        sel = idx_gpu[..., qb, :].reshape(-1, w.topk)
        k = min(w.topk, i)
        assert (sel[:, :k] >= 0).all() and (sel[:, k:] == -1).all()
        assert (sel[:, :k] < i).all()
        if k > 1:
            assert (np.diff(sel[:, :k], axis=1) > 0).all()


def check_out(w, O_gpu: np.ndarray, lse_gpu: np.ndarray, O_ora: np.ndarray, lse_ora: np.ndarray):
    t = TOL[w.dtype]
    err = np.abs(O_gpu - O_ora)
    rel = np.linalg.norm(O_gpu - O_ora) / max(np.linalg.norm(O_ora), 1e-30)
    assert err.max() <= t["o_abs"], f"O max-abs {err.max():.3e} > {t['o_abs']}"
    assert rel <= t["o_rel"], f"O rel-L2 {rel:.3e} > {t['o_rel']}"
    lerr = np.abs(lse_gpu - lse_ora).max()
    assert lerr <= t["lse"], f"lse max-abs {lerr:.3e}"
    return float(err.max()), float(rel)


def flat_rows(w, bi, hq, ts):
    return [((bi * w.Hq + hq) * w.Nq + t) for t in ts]


def sample_items(w, rng, n_units=2, n_qb=12):
    """(unit list, per-unit query blocks) to sample at full size."""
    U = w.B * w.Hkv
    units = sorted(set([0, U - 1] + list(rng.choice(U, size=min(n_units, U), replace=False))))[:max(n_units, 2)]
    nqb = oracle.num_qblocks(w)
    base = {0, 1, 2, nqb - 1, nqb // 2} if nqb > 3 else set(range(nqb))
    extra = set(rng.choice(nqb, size=min(n_qb, nqb), replace=False).tolist())
    qbs = sorted(q for q in base | extra if 0 <= q < nqb)
    return units, qbs


def rows_of_qblock(w, bi, hk, qb, rng, per_head=4):
    """Sampled flat query rows of query block qb for every head of kv head hk."""
    first = w.q_offset // w.b
    i = first + qb
    p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
    ts = np.arange(p0, p1) - w.q_offset
    pick = ts if len(ts) <= per_head else np.unique(np.concatenate([[ts[0], ts[-1]], rng.choice(ts, per_head - 2)]))
    rows = []
    for g in range(w.G):
        rows += flat_rows(w, bi, hk * w.G + g, pick)
    return rows


def fmt(w):
    return f"{w.name}[B{w.B} Hq{w.Hq} Hkv{w.Hkv} N{w.N} Nq{w.Nq} d{w.d} b{w.b} K{w.topk} C{w.cap}]"


def sqrt_d(w):
    return math.sqrt(w.d)


# ---- tie-tolerant walk: which results can the coarse-to-fine walk reach when near-ties go either way --

def walk_reaches(w, Q, pyr_unit: np.ndarray, unit: int, qb: int, target, eps: float, max_states: int = 20000):
    """Can the walk of (unit, query block qb) end in `target` (one idx row) if each comparison between
    two oracle node scores that differ by at most `eps` may be decided either way?

    The walk (PISA abstract: coarse-to-fine, a bounded candidate set per level) starts at the finest
    level s0 with at most `cap` nodes, with every node that begins before query block i; a level
    above 0 keeps min(cap/2, #candidates) nodes and hands on their children that exist and begin
    before i; level 0 keeps min(topk, #candidates). A kept set S of candidates C is reachable when
    min score over S >= max score over C minus S, minus eps. With eps = 0 and no exact ties only the
    oracle's own result is reachable; when every level's margin exceeds eps it is still the only one.
    Scores are the oracle's (`oracle.node_score`). Returns True, False, or None when the search
    visited more than max_states (level, candidate set) states.
    """
    first = w.q_offset // w.b
    i = first + qb
    lv = [n for _, n in oracle.level_offsets(w)]
    s0 = 0
    while lv[s0] > w.cap:
        s0 += 1
    T = sorted(int(x) for x in np.asarray(target).reshape(-1) if x >= 0)
    if len(set(T)) != len(T):
        return False
    cache = {}

    def score(l, m):
        if (l, m) not in cache:
            cache[(l, m)] = oracle.node_score(w, Q, pyr_unit, unit, qb, l, m)[0]
        return cache[(l, m)]

    def reachable_sets(cands, sc, keep, required):
        """Every kept set of size `keep` that holds `required` and meets the eps rule."""
        if keep == 0:
            return [frozenset()] if not required else []
        out = []
        seen = set()
        for z in cands:  # z: the lowest-scoring member of the kept set
            t = sc[z]
            must = {x for x in cands if sc[x] > t + eps} | set(required) | {z}
            if any(sc[x] < t for x in must) or len(must) > keep:
                continue
            opt = sorted((x for x in cands if x not in must and t <= sc[x] <= t + eps), key=lambda x: (-sc[x], x))
            need = keep - len(must)
            if need > len(opt):
                continue
            if math.comb(len(opt), need) > 2000:
                return None
            for extra in itertools.combinations(opt, need):
                S = frozenset(must | set(extra))
                if S in seen:
                    continue
                seen.add(S)
                rest = [sc[x] for x in cands if x not in S]
                if not rest or min(sc[x] for x in S) >= max(rest) - eps:
                    out.append(S)
        # the oracle's own choice (best scores, lower index on ties) first
        out.sort(key=lambda S: sorted((-sc[x], x) for x in S))
        return out

    states = [0]
    visited = {}

    def dfs(l, cands):
        key = (l, frozenset(cands))
        if key in visited:
            return visited[key]
        states[0] += 1
        if states[0] > max_states:
            raise _SearchBound
        sc = {m: score(l, m) for m in cands}
        want = w.cap // 2 if l > 0 else w.topk
        keep = min(want, len(cands))
        required = sorted({t >> l for t in T})
        if any(r not in sc for r in required):
            visited[key] = False
            return False
        if l == 0:
            if len(T) != keep:
                res = False
            else:
                rest = [sc[x] for x in cands if x not in set(T)]
                res = not rest or min(sc[x] for x in T) >= max(rest) - eps
            visited[key] = res
            return res
        sets = reachable_sets(cands, sc, keep, required)
        if sets is None:
            raise _SearchBound
        res = False
        for S in sets:
            nxt = sorted(ch for m in S for ch in (2 * m, 2 * m + 1) if ch < lv[l - 1] and (ch << (l - 1)) < i)
            if dfs(l - 1, nxt):
                res = True
                break
        visited[key] = res
        return res

    start = [m for m in range(lv[s0]) if (m << s0) < i]
    try:
        return dfs(s0, start)
    except _SearchBound:
        return None


class _SearchBound(Exception):
    pass


# ---- selection trace: check the GPU's own walk level by level ----------------------------------

def validate_trace(w, Q, pyr_unit: np.ndarray, unit: int, qb: int, trace_rows, idx_row, eps: float,
                   opts=None, score_cache=None):
    """Is the GPU's walk of (unit, query block qb), as its trace records it, a valid walk?

    trace_rows [s0 + 1][width]: row s0 - l lists the nodes the GPU kept at level l (any order, -1
    padded). Following the GPU's own chain of kept sets, with the oracle's scores (oracle.node_score):
      - level s0's candidates are the nodes that begin before block i; level l - 1's are the children
        of the nodes kept at level l that exist and begin before block i;
      - each level keeps the right number of distinct candidates: min(cap/2, #candidates) above level
        0; at level 0 the budget (opts: DBA budget, FCF expansion), where a confidence within eps of
        fcf_tau allows either count;
      - every kept candidate ranks within eps of every dropped one: min R over kept >= max R over
        dropped - eps (R = S + rcg_lambda * R(parent), R = S without RCG);
      - idx lists the level-0 kept set, ascending, then -1.
    With eps = 0 and no exact ties only the oracle's own walk passes. Returns (ok, message).
    """
    first = w.q_offset // w.b
    i = first + qb
    lv = [n for _, n in oracle.level_offsets(w)]
    s0 = 0
    while lv[s0] > w.cap:
        s0 += 1
    trace_rows = np.asarray(trace_rows).reshape(s0 + 1, -1)
    lam = opts.rcg_lambda if opts is not None else 0.0
    extra = opts.fcf_extra if opts is not None else 0
    tau = opts.fcf_tau if opts is not None else 0.0
    if opts is not None and opts.budget is not None:
        base = int(opts.budget[unit])
    else:
        base = w.topk - extra
    base = min(max(base, 0), w.topk)
    cache = {} if score_cache is None else score_cache

    def S(l, m):
        if (l, m) not in cache:
            cache[(l, m)] = oracle.node_score(w, Q, pyr_unit, unit, qb, l, m)[0]
        return cache[(l, m)]

    cands = {m: 0.0 for m in range(lv[s0]) if (m << s0) < i}  # node -> parent's R
    conf = math.inf
    for k, l in enumerate(range(s0, -1, -1)):
        kept = [int(x) for x in trace_rows[k] if x >= 0]
        if len(set(kept)) != len(kept):
            return False, f"level {l}: a node is kept twice: {kept}"
        if not set(kept) <= set(cands):
            return False, f"level {l}: kept {sorted(set(kept) - set(cands))} are not candidates"
        R = {m: S(l, m) + lam * p for m, p in cands.items()}
        order = sorted(R, key=lambda m: (-R[m], m))
        if l > 0:
            allowed = {min(w.cap // 2, len(R))}
        else:
            kb = min(base, len(R))
            allowed = {kb}
            if extra > 0:
                c0 = conf
                if 0 < kb < len(R):
                    c0 = min(c0, R[order[kb - 1]] - R[order[kb]])
                wide = min(base + extra, w.topk, len(R))
                if c0 < tau + eps:
                    allowed.add(wide)
                if c0 < tau - eps:
                    allowed.discard(kb)
        if len(kept) not in allowed:
            return False, f"level {l}: kept {len(kept)} nodes, allowed {sorted(allowed)}"
        dropped = [m for m in R if m not in set(kept)]
        if kept and dropped:
            margin = min(R[m] for m in kept) - max(R[m] for m in dropped)
            if margin < -eps:
                return False, (f"level {l}: kept node ranks {-margin:.3e} below a dropped one "
                               f"(kept {sorted(kept)}, best dropped {max(dropped, key=lambda m: R[m])})")
            if l > 0:
                conf = min(conf, margin)
        if l == 0:
            want = sorted(kept) + [-1] * (w.topk - len(kept))
            got = [int(x) for x in np.asarray(idx_row).reshape(-1)]
            if got != want:
                return False, f"idx {got} is not the level-0 kept set {want}"
            return True, ""
        cands = {ch: R[m] for m in kept for ch in (2 * m, 2 * m + 1) if ch < lv[l - 1] and (ch << (l - 1)) < i}
    return False, "unreachable"


def check_traces(w, Q, pyr_units: np.ndarray, units, items, idx_gpu, trace_gpu, idx_ora, gap_ora, trace_ora,
                 opts=None, eps: float = TIE_EPS):
    """Selection acceptance with the GPU's trace: rows with oracle gap >= GAP_EXEMPT must match the
    oracle bit for bit, trace included (as sets per level); every other row whose idx or trace
    differs from the oracle's must be a valid walk (validate_trace). Nothing is left undecided.
    Returns dict(checked, exempt, differing, validated)."""
    n = len(items)
    idx_gpu = np.asarray(idx_gpu).reshape(n, -1)
    idx_ora = np.asarray(idx_ora).reshape(n, -1)
    trace_gpu = np.asarray(trace_gpu).reshape(n, trace_ora.shape[1], -1)
    gap_ora = np.asarray(gap_ora).reshape(-1)
    checked = exempt = differing = validated = 0
    for k, (slot, qb) in enumerate(items):
        same_idx = (idx_gpu[k] == idx_ora[k]).all()
        same_trace = all(set(trace_gpu[k, l][trace_gpu[k, l] >= 0].tolist()) ==
                         set(trace_ora[k, l][trace_ora[k, l] >= 0].tolist()) for l in range(trace_ora.shape[1]))
        if gap_ora[k] >= GAP_EXEMPT:
            checked += 1
            assert same_idx, (f"unit {units[slot]} query block {qb}: gpu {idx_gpu[k]} oracle {idx_ora[k]} "
                              f"gap {gap_ora[k]:.3e}")
            assert same_trace, f"unit {units[slot]} query block {qb}: trace differs with gap {gap_ora[k]:.3e}"
            continue
        exempt += 1
        if same_idx and same_trace:
            continue
        differing += int(not same_idx)
        ok, msg = validate_trace(w, Q, pyr_units[slot], units[slot], qb, trace_gpu[k], idx_gpu[k], eps, opts)
        assert ok, (f"unit {units[slot]} query block {qb} (oracle gap {gap_ora[k]:.2e}, gpu idx {idx_gpu[k]}, "
                    f"oracle idx {idx_ora[k]}): {msg}")
        validated += 1
    return dict(checked=checked, exempt=exempt, differing=differing, validated=validated)


def check_exempt_rows(w, Q, pyr_units: np.ndarray, units, items, idx_gpu: np.ndarray, idx_ora: np.ndarray,
                      gap_ora: np.ndarray, eps: float = TIE_EPS):
    """Every row inside the gap exemption whose GPU idx differs from the oracle's must be reachable by
    the tie-tolerant walk. items[k] = (slot, qb): slot indexes units and pyr_units ([len(units), P, d]).
    Returns (differing, reached, undecided); undecided rows (search bound) are reported, not failed."""
    idx_gpu = idx_gpu.reshape(len(items), -1)
    idx_ora = idx_ora.reshape(len(items), -1)
    gap_ora = gap_ora.reshape(-1)
    differing = reached = undecided = 0
    for k, (slot, qb) in enumerate(items):
        if gap_ora[k] >= GAP_EXEMPT or (idx_gpu[k] == idx_ora[k]).all():
            continue
        differing += 1
        r = walk_reaches(w, Q, pyr_units[slot], units[slot], qb, idx_gpu[k], eps)
        if r is None:
            undecided += 1
            continue
        assert r, (f"unit {units[slot]} query block {qb}: GPU idx {idx_gpu[k]} is not reachable by the walk with "
                   f"near-ties within {eps} (oracle {idx_ora[k]}, gap {gap_ora[k]:.2e})")
        reached += 1
    return differing, reached, undecided
