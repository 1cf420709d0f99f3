"""The five synthetic workloads at full size, through the same C-ABI calls the benchmark times.

The GPU runs the whole path on the full workload; the oracle then computes a
seeded sample one item at a time:
  - the pyramids of 8 (batch, kv head) units (all of them when there are fewer);
  - the selection of 64 query blocks of each sampled unit (all when fewer). Rows
    whose oracle gap is >= 1e-4 must match bit for bit, with the GPU's trace of
    kept nodes per level; every other row whose result differs is checked level
    by level along the GPU's own walk (validate_trace), so no row is left
    undecided;
  - attention for every row of 2 query blocks per sampled unit (all G heads) and
    4 rows per head of every sampled block, given the oracle's indices and, end
    to end, given the GPU's.
Properties that hold at any size (index validity, status) are checked on every
row. The counts are printed (pytest -s) for the design notes.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _parity import (check_out, check_pyramid, check_traces, check_valid_idx, flat_rows, fmt, rows_of_qblock,
                     run_gpu)

pytestmark = pytest.mark.gpu

N_UNITS, N_QB = 8, 64


def sample(w, rng):
    """(units, query blocks per unit, fully checked blocks per unit)."""
    U = w.B * w.Hkv
    units = sorted(set([0, U - 1]) | set(rng.choice(U, size=min(N_UNITS, U), replace=False).tolist()))[:N_UNITS]
    nqb = oracle.num_qblocks(w)
    if nqb <= N_QB:
        qbs = list(range(nqb))
    else:
        base = {0, 1, 2, nqb // 2, nqb - 1}
        qbs = sorted(base | set(rng.choice(nqb, size=N_QB - len(base), replace=False).tolist()))
    full = sorted({qbs[-1], qbs[len(qbs) // 2]})
    return units, qbs, full


@pytest.mark.parametrize("w", synth.WORKLOADS, ids=lambda w: w.name)
def test_workload_full_size(w):
    rng = np.random.default_rng(w.seed + 100)
    Q, K, V, owner = synth.generate(w)
    g = run_gpu(w, Q, K, V, with_trace=True)
    assert g["status"] == 0
    idx_all = g["idx"].numpy()
    check_valid_idx(w, idx_all)

    units, qbs, full = sample(w, rng)
    pyr_o = oracle.pyramid(w, K, units)
    pyr_g = g["pyr"].double().numpy().reshape(w.B * w.Hkv, -1, w.d)[units]
    check_pyramid(pyr_g, pyr_o)

    items = [(s, q) for s in range(len(units)) for q in qbs]
    idx_o, gap_o, _, trace_o = oracle.select(w, Q, pyr_o, units, items, with_trace=True)
    U = w.B * w.Hkv
    idx_g = np.stack([idx_all.reshape(U, -1, w.topk)[units[s], q] for s, q in items])
    trace_g = np.stack([g["trace"].numpy()[units[s], q] for s, q in items])
    counts = check_traces(w, Q, pyr_o, units, items, idx_g, trace_g, idx_o, gap_o, trace_o)

    # attention for sampled rows, given the oracle's idx: patch those rows into a copy of the GPU idx
    idx_patch = idx_all.copy().reshape(U, -1, w.topk)
    for k, (s, q) in enumerate(items):
        idx_patch[units[s], q] = idx_o[k]
    idx_patch = idx_patch.reshape(idx_all.shape)
    g2 = run_gpu(w, Q, K, V, idx=idx_patch)
    assert g2["status"] == 0
    rows = []
    first = w.q_offset // w.b
    for s, q in items:
        bi, hk = divmod(units[s], w.Hkv)
        rows += rows_of_qblock(w, bi, hk, q, rng)
    n_full = 0
    for s in range(len(units)):
        bi, hk = divmod(units[s], w.Hkv)
        for q in full:
            i = first + q
            p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
            for gg in range(w.G):
                block_rows = flat_rows(w, bi, hk * w.G + gg, range(p0 - w.q_offset, p1 - w.q_offset))
                rows += block_rows
                n_full += len(block_rows)
    rows = np.array(sorted(set(rows)), dtype=np.int64)
    O_o, lse_o = oracle.attend(w, Q, K, V, idx_patch, rows)
    e, r = check_out(w, g2["O"].double().numpy().reshape(-1, w.d)[rows],
                     g2["lse"].double().numpy().reshape(-1)[rows], O_o, lse_o)
    # end to end with the GPU's own idx
    O_o2, lse_o2 = oracle.attend(w, Q, K, V, idx_all, rows)
    check_out(w, g["O"].double().numpy().reshape(-1, w.d)[rows], g["lse"].double().numpy().reshape(-1)[rows],
              O_o2, lse_o2)

    # needle recall of the GPU selection (owned needles), reported
    own = owner.numpy().reshape(U, -1)
    hit = tot = 0
    sel = idx_all.reshape(U, -1, w.topk)
    for u in range(own.shape[0]):
        for j in np.nonzero(own[u] >= 0)[0]:
            i = own[u, j]
            if 0 <= i - first < sel.shape[1]:
                tot += 1
                hit += int(j in sel[u, i - first])
    print(f"\n{fmt(w)}: {len(units)} units x {len(qbs)} query blocks; select {counts['checked']} rows bit-exact "
          f"with their trace, {counts['exempt']} exempt ({counts['differing']} differ, {counts['validated']} "
          f"validated level by level, 0 undecided); attention on {len(rows)} rows ({n_full} in whole blocks) "
          f"max-abs {e:.2e} rel-L2 {r:.2e}; needle recall {hit}/{tot}")
    del g, g2
    torch.cuda.empty_cache()
