"""Helpers shared by the GPU parity tests: run the CUDA path, compare with the oracle.

Acceptance (per the selection/attention contract):
  idx   bit-exact for every (batch, kv head, query block) whose oracle gap is
        >= GAP_EXEMPT; rows under it may differ and are counted;
  O     bf16: max-abs <= 2e-2 and relative L2 <= 1e-2; fp32: max-abs <= 1e-4;
  lse   bf16: max-abs <= 2e-3; fp32: max-abs <= 1e-4;
  pyr   fp32 accumulation against the double oracle: max-abs <= 2e-5 * (1 + |x|).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import hierarchical_block_sparse_pyr_b200 as P
import oracle
import synth

GAP_EXEMPT = 1e-4
TOL = {synth.F32: dict(o_abs=1e-4, o_rel=1e-4, lse=1e-4), synth.BF16: dict(o_abs=2e-2, o_rel=1e-2, lse=2e-3)}


def to_dev(*ts):
    return [t.cuda() for t in ts]


def run_gpu(w, Q, K, V, idx=None, dense=False):
    """Run the CUDA path on CPU inputs. Returns a dict of CPU tensors."""
    s = P.shape_of(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    buf = P.Buffers(s)
    P.pyr_build(s, Kd, buf.pyr, buf.status)
    P.pyr_select(s, Qd, buf.pyr, buf.idx, buf.gap, buf.status)
    if dense:
        P.dense_forward(s, Qd, Kd, Vd, buf.O, buf.lse, buf.status)
    else:
        use = buf.idx if idx is None else torch.as_tensor(np.ascontiguousarray(idx), dtype=torch.int32).cuda()
        P.bsa_forward(s, Qd, Kd, Vd, use, buf.O, buf.lse, buf.status)
    torch.cuda.synchronize()
    out = dict(pyr=P.pyramid_means(buf.pyr).cpu(), idx=buf.idx.cpu(), gap=buf.gap.cpu(), O=buf.O.float().cpu(), lse=buf.lse.cpu(),
               status=int(buf.status.item()))
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
