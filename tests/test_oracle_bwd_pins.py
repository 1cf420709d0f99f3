"""Pins of the oracle's backward pass (block-major route metadata, sparse gradients).

The gradients are pinned to central finite differences of the oracle's own
forward pass (which is pinned to torch SDPA elsewhere), in float64, and to two
identities that hold for any routes:
  - sum over every key of dK is zero (softmax is invariant to a shift of the
    scores, so each row's dS sums to zero);
  - sum over every key of dV equals the sum of dO over the rows that attend
    (each row's probabilities sum to one).
The route inversion is pinned to a worked example (tests/golden/route_invert.txt)
and to a brute-force reading of its definition on random tables.
Sources: PHBA summary, A.1.2 (block-major metadata) and A.1.4 (sparse backward).
"""
import os
from types import SimpleNamespace

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "route_invert.txt")


def _shape(**kw):
    base = dict(B=1, Hq=2, Hkv=1, N=80, Nq=80, q_offset=0, d=8, b=16, topk=2, cap=4, dtype=oracle.F64)
    base.update(kw)
    return SimpleNamespace(**base)


def _random_routes(w, rng, full=False):
    nqb = oracle.num_qblocks(w)
    first = w.q_offset // w.b
    idx = np.full((w.B, w.Hkv, nqb, w.topk), -1, dtype=np.int32)
    for u in range(w.B * w.Hkv):
        for q in range(nqb):
            i = first + q
            n = min(w.topk, i)
            if n:
                pick = np.arange(i) if full else rng.choice(i, size=n, replace=False)
                idx[u // w.Hkv, u % w.Hkv, q, :n] = np.sort(pick[:n])
    return idx


def _tensors(w, rng):
    Q = np.ascontiguousarray(rng.standard_normal((w.B, w.Hq, w.Nq, w.d)))
    K = np.ascontiguousarray(rng.standard_normal((w.B, w.Hkv, w.N, w.d)) * 1.5)
    V = np.ascontiguousarray(rng.standard_normal((w.B, w.Hkv, w.N, w.d)))
    dO = np.ascontiguousarray(rng.standard_normal((w.B, w.Hq, w.Nq, w.d)))
    return Q, K, V, dO


def _loss(w, Q, K, V, dO, idx, dense=False):
    rows = np.arange(w.B * w.Hq * w.Nq)
    O, _ = oracle.attend(w, Q, K, V, idx, rows, dense=dense)
    return float((O * dO.reshape(-1, w.d)).sum())


def _all_grads(w, Q, K, V, dO, idx, dense=False):
    rows = np.arange(w.B * w.Hq * w.Nq)
    dQ = oracle.attend_bwd_q(w, Q, K, V, dO, idx, rows, dense=dense).reshape(Q.shape)
    nb = (w.N + w.b - 1) // w.b
    blocks = [(u, j) for u in range(w.B * w.Hkv) for j in range(nb)]
    dKb, dVb = oracle.attend_bwd_kv(w, Q, K, V, dO, idx, blocks, dense=dense)
    dK = dKb.reshape(w.B, w.Hkv, nb * w.b, w.d)[:, :, :w.N]
    dV = dVb.reshape(w.B, w.Hkv, nb * w.b, w.d)[:, :, :w.N]
    return dQ, np.ascontiguousarray(dK), np.ascontiguousarray(dV)


@pytest.mark.parametrize("case", [
    dict(),                                                # GQA (G = 2), ragged last block
    dict(q_offset=32, Nq=48),                              # a prefill chunk starting at block 2
    dict(Hq=2, Hkv=2, N=64, Nq=64, topk=1),                # MHA, one route per block
])
def test_gradients_match_central_differences(case):
    w = _shape(**case)
    rng = np.random.default_rng(7)
    Q, K, V, dO = _tensors(w, rng)
    idx = _random_routes(w, rng)
    dQ, dK, dV = _all_grads(w, Q, K, V, dO, idx)
    h = 1e-5
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        flat = X.reshape(-1)
        for e in rng.choice(flat.size, size=10, replace=False):
            keep = flat[e]
            flat[e] = keep + h
            lp = _loss(w, Q, K, V, dO, idx)
            flat[e] = keep - h
            lm = _loss(w, Q, K, V, dO, idx)
            flat[e] = keep
            fd = (lp - lm) / (2 * h)
            an = G.reshape(-1)[e]
            assert abs(fd - an) <= 1e-6 * (1 + abs(fd)), (name, e, fd, an)


@pytest.mark.parametrize("dense", [False, True])
def test_shift_and_normalisation_identities(dense):
    w = _shape(B=2, Hq=4, Hkv=2, N=112, Nq=112, d=16, b=16, topk=3, dtype=0)
    rng = np.random.default_rng(3)
    Q, K, V, dO = [x.astype(np.float32) for x in _tensors(w, rng)]
    idx = _random_routes(w, rng)
    dQ, dK, dV = _all_grads(w, Q, K, V, dO, idx, dense=dense)
    G = w.Hq // w.Hkv
    for bi in range(w.B):
        for hk in range(w.Hkv):
            assert np.abs(dK[bi, hk].sum(axis=0)).max() < 1e-9
            rows_dO = dO[bi, hk * G:(hk + 1) * G].astype(np.float64).reshape(-1, w.d).sum(axis=0)
            assert np.abs(dV[bi, hk].sum(axis=0) - rows_dO).max() < 1e-9


def test_every_block_routed_equals_dense():
    w = _shape(N=96, Nq=96, topk=6, cap=12)
    rng = np.random.default_rng(11)
    Q, K, V, dO = _tensors(w, rng)
    idx = _random_routes(w, rng, full=True)
    a = _all_grads(w, Q, K, V, dO, idx)
    b = _all_grads(w, Q, K, V, dO, None, dense=True)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() < 1e-12


def _read_golden():
    idx, offset, rho = [], None, None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = line.split(":", 1)
        vals = [int(v) for v in val.split()]
        if key.startswith("idx"):
            idx.append(vals)
        elif key == "offset":
            offset = vals
        elif key == "rho":
            rho = vals
    return np.array(idx, dtype=np.int32), np.array(offset), np.array(rho)


def test_route_inversion_worked_example():
    idx, offset, rho = _read_golden()
    w = _shape(Hq=1, Hkv=1, N=96, Nq=96, topk=2)
    off, r = oracle.route_invert(w, idx.reshape(1, 1, 6, 2))
    assert off[0].tolist() == offset.tolist()
    assert r[0, :offset[-1]].tolist() == rho.tolist()
    assert (r[0, offset[-1]:] == -1).all()


def test_route_inversion_brute_force():
    w = _shape(B=2, Hq=4, Hkv=2, N=400, Nq=400, b=16, topk=5)
    rng = np.random.default_rng(5)
    idx = _random_routes(w, rng)
    off, rho = oracle.route_invert(w, idx)
    nb = (w.N + w.b - 1) // w.b
    for u in range(w.B * w.Hkv):
        table = idx[u // w.Hkv, u % w.Hkv]
        for j in range(nb):
            want = [q for q in range(table.shape[0]) if j in set(table[q].tolist())]
            assert rho[u, off[u, j]:off[u, j + 1]].tolist() == want


def test_route_inversion_rejects_bad_routes():
    w = _shape(Hq=1, Hkv=1, N=96, Nq=96, topk=2)
    idx = np.full((1, 1, 6, 2), -1, dtype=np.int32)
    idx[0, 0, 3] = [3, -1]  # not strictly before its query block
    with pytest.raises(ValueError):
        oracle.route_invert(w, idx)
    idx[0, 0, 3] = [1, 1]  # repeated
    with pytest.raises(ValueError):
        oracle.route_invert(w, idx)
