"""PHAROS selection variants on the GPU against the oracle (pyr_select_ex).

PHAROS page ("Four mechanisms powering PHAROS"): per-head budgets (DBA), a
budget that grows when confidence is low (FCF), coarse levels guiding finer
ones (RCG). Each case runs the three selection kernels' paths (tensor-core
prefill, CUDA-core prefill, decode) with the variants on and checks them like
the plain walk: rows whose oracle gap is >= 1e-4 bit-exact with their trace,
every other differing row valid level by level along the GPU's own walk. With
guidance the ranking score carries each ancestor's score, so the slack of a
comparison grows with sum_k lambda^k; the slack used is TIE_EPS times that
sum. Attention then runs end to end on the variant's routes (rows of varying
length).
"""
import numpy as np
import pytest

import oracle
import synth
from _parity import TIE_EPS, check_out, check_traces, check_valid_idx, fmt, run_gpu
from synth import BF16, F32

pytestmark = pytest.mark.gpu

W0 = synth.WORKLOADS[0]


def _budget(w, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(1, w.topk + 1, size=w.B * w.Hkv).tolist()


CASES = [
    # tensor-core walk (bf16, d=128, b=64, M=64 stacked): budgets per head + fallback
    (W0.scaled(name="tc_dba_fcf", B=1, Hq=4, Hkv=4, N=8192, Nq=8192, d=128, b=64, topk=12, cap=16, dtype=BF16,
               seed=61, n_needle=4), dict(budget=0, fcf_tau=0.05, fcf_extra=4, rcg_lambda=0.0)),
    # tensor-core walk, GQA, M=128 stacked: guidance
    (W0.scaled(name="tc_rcg_gqa", B=1, Hq=8, Hkv=2, N=16384, Nq=16384, d=128, b=64, topk=24, cap=48, dtype=BF16,
               seed=62, n_needle=6), dict(budget=None, fcf_tau=0.0, fcf_extra=0, rcg_lambda=0.5)),
    # tensor-core walk, separate hi/lo operands (cap > 64): all three
    (W0.scaled(name="tc_all_cap100", B=1, Hq=2, Hkv=2, N=16384, Nq=16384, d=128, b=64, topk=50, cap=100,
               dtype=BF16, seed=63, n_needle=6), dict(budget=1, fcf_tau=0.02, fcf_extra=10, rcg_lambda=0.25)),
    # CUDA-core walk (fp32): all three
    (W0.scaled(name="simt_all_f32", B=2, Hq=4, Hkv=2, N=3000, Nq=3000, d=64, b=32, topk=8, cap=12, dtype=F32,
               seed=64), dict(budget=2, fcf_tau=0.1, fcf_extra=3, rcg_lambda=0.3)),
    # decode walk: budgets + fallback + guidance
    (W0.scaled(name="decode_all", B=6, Hq=16, Hkv=4, N=20000, Nq=1, q_offset=19999, d=128, b=64, topk=20, cap=32,
               dtype=BF16, seed=65, n_needle=4, needle_mode=synth.NEEDLE_DECODE),
     dict(budget=3, fcf_tau=0.05, fcf_extra=6, rcg_lambda=0.2)),
]


def _opts(w, spec):
    budget = None if spec["budget"] is None else _budget(w, spec["budget"])
    return oracle.SelectOpts(budget=budget, fcf_tau=spec["fcf_tau"], fcf_extra=spec["fcf_extra"],
                             rcg_lambda=spec["rcg_lambda"])


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_variant_parity(case):
    w, spec = case
    opts = _opts(w, spec)
    Q, K, V, _ = synth.generate(w)
    units = list(range(w.B * w.Hkv))
    g = run_gpu(w, Q, K, V, opts=opts, with_trace=True)
    assert g["status"] == 0
    pyr_o = oracle.pyramid(w, K, units)
    nqb = oracle.num_qblocks(w)
    items = [(u, q) for u in units for q in range(nqb)]
    idx_o, gap_o, _, trace_o = oracle.select(w, Q, pyr_o, units, items, opts=opts, with_trace=True)
    lam = abs(spec["rcg_lambda"])
    eps = TIE_EPS * sum(lam ** k for k in range(oracle.trace_levels(w)))
    counts = check_traces(w, Q, pyr_o, units, items, g["idx"].numpy(), g["trace"].numpy(), idx_o, gap_o, trace_o,
                          opts=opts, eps=eps)
    # each row keeps its own count (budget, fallback): ascending, before the query block, -1 after
    idx_g = g["idx"].numpy().reshape(len(items), w.topk)
    first = w.q_offset // w.b
    n_kept = []
    for k, (u, q) in enumerate(items):
        row = idx_g[k]
        kept = row[row >= 0]
        n_kept.append(len(kept))
        assert (row[len(kept):] == -1).all() and (kept < first + q).all() and (np.diff(kept) > 0).all()
    gap_g = g["gap"].double().numpy().reshape(-1)
    fin = np.isfinite(gap_o)
    assert (np.isfinite(gap_g) == fin).all()
    np.testing.assert_allclose(gap_g[fin], gap_o[fin], atol=1e-3 * (1 + 10 * lam), rtol=1e-3)
    # attention end to end on the GPU's variable-length routes
    rng = np.random.default_rng(w.seed)
    total = w.B * w.Hq * w.Nq
    rows = np.unique(np.concatenate([rng.choice(total, min(total, 500), replace=False), [0, total - 1]]))
    O_o, lse_o = oracle.attend(w, Q, K, V, g["idx"].numpy(), rows)
    e, r = check_out(w, g["O"].double().numpy().reshape(-1, w.d)[rows], g["lse"].double().numpy().reshape(-1)[rows],
                     O_o, lse_o)
    print(f"\n{fmt(w)} {spec}: {counts['checked']} rows bit-exact with their trace, {counts['exempt']} exempt "
          f"({counts['differing']} differ, {counts['validated']} validated); blocks kept per row "
          f"{min(n_kept)}..{max(n_kept)}; attention max-abs {e:.2e}")


def test_plain_options_equal_pyr_select():
    """A zeroed option struct is the plain walk, bit for bit (idx and gap)."""
    w = W0.scaled(name="plain_ex", B=1, Hq=4, Hkv=2, N=8192, Nq=8192, d=128, b=64, topk=8, cap=16, dtype=BF16,
                  seed=66)
    Q, K, V, _ = synth.generate(w)
    a = run_gpu(w, Q, K, V)
    b = run_gpu(w, Q, K, V, opts=oracle.SelectOpts(), with_trace=True)
    assert np.array_equal(a["idx"].numpy(), b["idx"].numpy())
    assert np.array_equal(a["gap"].numpy(), b["gap"].numpy())
    check_valid_idx(w, b["idx"].numpy())
