"""The five synthetic workloads at full size, through the same C-ABI calls the benchmark times.

The GPU runs the whole path on the full workload; the oracle then computes a
seeded sample one item at a time: the pyramids of a few (batch, kv head)
units, the selection of a few query blocks of those units, and attention for
a few rows of each sampled block (given the oracle's indices and, end to end,
given the GPU's). Properties that hold at any size (index validity, status)
are checked on every row.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _parity import (check_exempt_rows, check_out, check_pyramid, check_select, check_valid_idx, fmt,
                     rows_of_qblock, run_gpu, sample_items)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", synth.WORKLOADS, ids=lambda w: w.name)
def test_workload_full_size(w):
    rng = np.random.default_rng(w.seed + 100)
    Q, K, V, owner = synth.generate(w)
    g = run_gpu(w, Q, K, V)
    assert g["status"] == 0
    idx_all = g["idx"].numpy()
    check_valid_idx(w, idx_all)

    units, qbs = sample_items(w, rng)
    pyr_o = oracle.pyramid(w, K, units)
    pyr_g = g["pyr"].double().numpy().reshape(w.B * w.Hkv, -1, w.d)[units]
    check_pyramid(pyr_g, pyr_o)

    items = [(s, q) for s in range(len(units)) for q in qbs]
    idx_o, gap_o, _ = oracle.select(w, Q, pyr_o, units, items)
    idx_g = np.stack([idx_all.reshape(w.B * w.Hkv, -1, w.topk)[units[s], q] for s, q in items])
    checked, exempt, exempt_diff = check_select(idx_g, idx_o, gap_o)
    _, reached, undecided = check_exempt_rows(w, Q, pyr_o, units, items, idx_g, idx_o, gap_o)

    # attention for sampled rows, given the oracle's idx: patch those rows into a copy of the GPU idx
    idx_patch = idx_all.copy().reshape(w.B * w.Hkv, -1, w.topk)
    for k, (s, q) in enumerate(items):
        idx_patch[units[s], q] = idx_o[k]
    idx_patch = idx_patch.reshape(idx_all.shape)
    g2 = run_gpu(w, Q, K, V, idx=idx_patch)
    assert g2["status"] == 0
    rows = []
    for s, q in items:
        bi, hk = divmod(units[s], w.Hkv)
        rows += rows_of_qblock(w, bi, hk, q, rng)
    rows = np.array(sorted(set(rows)), dtype=np.int64)
    O_o, lse_o = oracle.attend(w, Q, K, V, idx_patch, rows)
    e, r = check_out(w, g2["O"].double().numpy().reshape(-1, w.d)[rows],
                     g2["lse"].double().numpy().reshape(-1)[rows], O_o, lse_o)
    # end to end with the GPU's own idx
    O_o2, lse_o2 = oracle.attend(w, Q, K, V, idx_all, rows)
    check_out(w, g["O"].double().numpy().reshape(-1, w.d)[rows], g["lse"].double().numpy().reshape(-1)[rows],
              O_o2, lse_o2)

    # needle recall of the GPU selection (owned needles), reported
    own = owner.numpy().reshape(w.B * w.Hkv, -1)
    first = w.q_offset // w.b
    hit = tot = 0
    sel = idx_all.reshape(w.B * w.Hkv, -1, w.topk)
    for u in range(own.shape[0]):
        for j in np.nonzero(own[u] >= 0)[0]:
            i = own[u, j]
            if 0 <= i - first < sel.shape[1]:
                tot += 1
                hit += int(j in sel[u, i - first])
    print(f"\n{fmt(w)}: select {checked} rows bit-exact, {exempt} exempt ({exempt_diff} differ, {reached} reachable "
          f"with near-ties either way, {undecided} undecided); "
          f"attention on {len(rows)} rows max-abs {e:.2e} rel-L2 {r:.2e}; needle recall {hit}/{tot}")
    del g, g2
    torch.cuda.empty_cache()
