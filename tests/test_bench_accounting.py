"""The roofline numerators of bench.py against counts taken from the method itself.

`bench.work_counts` computes the algorithmic work of one step in closed form. Here
it is checked against the oracle's own routes and walk on small workloads:
  - attention pairs: every (query row, key) pair the routes and the causal own
    block admit, counted one by one, must equal the closed form exactly;
  - selection FLOPs: the closed form counts, per level, every node that could be
    a candidate; the oracle reports how many were actually scored, which can only
    be fewer (a straddling node's second child, or the end of a level), so the
    closed form is an upper bound within a few percent.
"""
import pytest

import bench
import oracle
import synth
from synth import BF16, F32

W0 = synth.WORKLOADS[0]
CASES = [
    W0.scaled(name="acc_mha_ragged", B=1, Hq=2, Hkv=2, N=3000, Nq=3000, d=64, b=64, topk=4, cap=8, dtype=F32, seed=61),
    W0.scaled(name="acc_gqa", B=2, Hq=4, Hkv=2, N=2048, Nq=2048, d=64, b=64, topk=6, cap=12, dtype=F32, seed=62),
    W0.scaled(name="acc_b128", B=1, Hq=2, Hkv=1, N=4096 + 100, Nq=4096 + 100, d=64, b=128, topk=4, cap=8, dtype=BF16,
              seed=63),
    W0.scaled(name="acc_decode", B=3, Hq=4, Hkv=2, N=5000, Nq=1, q_offset=4999, d=64, b=64, topk=8, cap=16,
              dtype=F32, seed=64, needle_mode=synth.NEEDLE_DECODE),
]


def _pairs_from_routes(w, idx):
    first = w.q_offset // w.b
    total = 0
    for u in range(w.B * w.Hkv):
        for q in range(idx.shape[1]):
            i = first + q
            p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
            keys_routed = sum(min((j + 1) * w.b, w.N) - j * w.b for j in idx[u, q] if j >= 0)
            for p in range(p0, p1):
                total += w.G * (keys_routed + (p - i * w.b + 1))
    return total


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_attention_pairs_equal_the_routes(w):
    Q, K, V, _ = synth.generate(w)
    idx, _, _ = oracle.select_all(w, Q, K)
    assert bench.work_counts(w)["att_pairs"] == _pairs_from_routes(w, idx)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_selection_flops_bound_the_scored_candidates(w):
    Q, K, V, _ = synth.generate(w)
    _, _, ncand = oracle.select_all(w, Q, K)
    first = w.q_offset // w.b
    exact = 0
    for q in range(ncand.shape[1]):
        i = first + q
        p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
        rows = w.G * (p1 - p0)
        exact += 2 * rows * w.d * int(ncand[:, q, :].sum())
    closed = bench.work_counts(w)["sel_flops"]
    assert exact <= closed <= 1.05 * exact, (exact, closed)
