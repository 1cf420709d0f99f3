"""Backward pass (route inversion + gradients) on the GPU vs the CPU oracle.

Route inversion is integer work: offset and rho must equal the oracle's bit
for bit, on the GPU's own routes. Gradients are compared with the oracle's
float64 gradients of sum(dO * O) for the same routes:
  fp32: max-abs error <= 1e-4 * max(1, max |reference|) per tensor;
  bf16: relative L2 error <= 2e-2 and max-abs error <= 3e-2 * max |reference|.
The bf16 bound: inputs are the same bf16 values on both sides; the GPU rounds
each gradient to bf16 (2^-9 relative), and its D_t = dO_t . O_t uses the bf16
forward output O (2^-9 relative), which enters dS_tk = P_tk (dP_tk - D_t) as an
absolute error of at most P_tk |dO_t| |O_t| 2^-9.
Small cases compare every element; the full 32K workload compares sampled
rows and key blocks and checks two identities on every unit: the dK of all
keys sums to zero and the dV of all keys sums to the dO of all rows.
"""
import numpy as np
import pytest
import torch

import hierarchical_block_sparse_pyr_b200 as P
import oracle
import synth
from synth import BF16, F32

pytestmark = pytest.mark.gpu

W0 = synth.WORKLOADS[0]
CASES = [
    W0.scaled(name="f32_gqa_ragged", B=1, Hq=4, Hkv=2, N=1000, Nq=1000, d=64, b=64, topk=4, cap=8, dtype=F32, seed=41),
    W0.scaled(name="bf16_mha_d128", B=1, Hq=2, Hkv=2, N=1536, Nq=1536, d=128, b=64, topk=4, cap=8, dtype=BF16, seed=42),
    W0.scaled(name="bf16_gqa_ragged", B=2, Hq=4, Hkv=1, N=1100, Nq=1100, d=128, b=64, topk=3, cap=6, dtype=BF16,
              seed=43),
    W0.scaled(name="bf16_b128", B=1, Hq=2, Hkv=2, N=2048 + 40, Nq=2048 + 40, d=128, b=128, topk=4, cap=8, dtype=BF16,
              seed=44),
    # 64-row MHA blocks (the paired-list kernels): ragged tail, odd and even list lengths, two batches
    W0.scaled(name="bf16_mha_ragged", B=2, Hq=2, Hkv=2, N=2000, Nq=2000, d=128, b=64, topk=7, cap=14, dtype=BF16,
              seed=46),
    # key blocks that more than 64 query blocks attend (needles): the dK/dV work order puts them first
    W0.scaled(name="bf16_mha_long_lists", B=1, Hq=2, Hkv=2, N=8192, Nq=8192, d=128, b=64, topk=24, cap=48,
              dtype=BF16, seed=47, n_needle=4),
    # one key block: a single step whose second half is padding
    W0.scaled(name="bf16_mha_one_block", B=1, Hq=2, Hkv=2, N=64, Nq=64, d=128, b=64, topk=4, cap=8, dtype=BF16,
              seed=48),
    W0.scaled(name="f32_b16_d128", B=1, Hq=2, Hkv=1, N=333, Nq=333, d=128, b=16, topk=5, cap=10, dtype=F32, seed=45),
]


def _forward_backward(w):
    s = P.shape_of(w)
    Q, K, V, _ = synth.generate(w)
    dO = synth.grad_output(w)
    Qd, Kd, Vd, dOd = (t.cuda() for t in (Q, K, V, dO))
    fwd = P.Buffers(s)
    bwd = P.BackwardBuffers(s)
    P.run(s, Qd, Kd, Vd, fwd)
    P.run_backward(s, Qd, Kd, Vd, dOd, fwd, bwd)
    torch.cuda.synchronize()
    assert int(fwd.status.item()) == 0
    host = {k: getattr(bwd, k).float().cpu().numpy() for k in ("dQ", "dK", "dV")}
    host.update(offset=bwd.offset.cpu().numpy(), rho=bwd.rho.cpu().numpy(), idx=fwd.idx.cpu().numpy())
    return (Q, K, V, dO), host


def _close(w, got, ref, what):
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    scale = max(1.0, float(np.abs(ref).max())) if w.dtype == F32 else float(np.abs(ref).max())
    if w.dtype == F32:
        assert err.max() <= 1e-4 * scale, f"{what}: max-abs {err.max():.3e} vs bound {1e-4 * scale:.3e}"
    else:
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert rel <= 2e-2, f"{what}: rel-L2 {rel:.3e}"
        assert err.max() <= 3e-2 * scale, f"{what}: max-abs {err.max():.3e} vs bound {3e-2 * scale:.3e}"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_small(w):
    (Q, K, V, dO), g = _forward_backward(w)
    off, rho = oracle.route_invert(w, g["idx"])
    assert (g["offset"] == off).all()
    assert (g["rho"] == rho).all()
    nb = (w.N + w.b - 1) // w.b
    dQ = oracle.attend_bwd_q(w, Q, K, V, dO, g["idx"], np.arange(w.B * w.Hq * w.Nq))
    _close(w, g["dQ"].reshape(-1, w.d), dQ, "dQ")
    blocks = [(u, j) for u in range(w.B * w.Hkv) for j in range(nb)]
    dK, dV = oracle.attend_bwd_kv(w, Q, K, V, dO, g["idx"], blocks)
    pad = nb * w.b - w.N
    gk = np.pad(g["dK"].reshape(w.B * w.Hkv, w.N, w.d), ((0, 0), (0, pad), (0, 0))).reshape(-1, w.b, w.d)
    gv = np.pad(g["dV"].reshape(w.B * w.Hkv, w.N, w.d), ((0, 0), (0, pad), (0, 0))).reshape(-1, w.b, w.d)
    _close(w, gk, dK, "dK")
    _close(w, gv, dV, "dV")


def test_long_lists_case_has_long_lists():
    # the needles of bf16_mha_long_lists are attended by more than 64 query blocks (oracle routes)
    w = [c for c in CASES if c.name == "bf16_mha_long_lists"][0]
    Q, K, V, _ = synth.generate(w)
    idx = oracle.select_all(w, Q, K)[0]
    nb = (w.N + w.b - 1) // w.b
    longest = max(np.bincount(row[row >= 0], minlength=nb).max() for row in idx.reshape(w.B * w.Hkv, -1))
    assert longest + 1 > 64


def test_route_inversion_reports_bad_routes():
    w = CASES[1]
    s = P.shape_of(w)
    nqb = P.num_qblocks(s)
    idx = torch.full((w.B, w.Hkv, nqb, w.topk), -1, dtype=torch.int32)
    idx[0, 0, 5, :2] = torch.tensor([1, 3])
    idx[0, 0, 6, :2] = torch.tensor([7, 2])   # 7 is not before block 6: skipped, reported
    idx[0, 1, 9, :3] = torch.tensor([4, 4, 8])  # the repeat is skipped, reported
    b = P.BackwardBuffers(s)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.bsa_route_invert(s, idx.cuda(), b.offset, b.rho, status)
    torch.cuda.synchronize()
    assert int(status.item()) == P.PYR_EBADIDX
    good = idx.clone()
    good[0, 0, 6, 0] = -1
    good[0, 1, 9, 1] = -1
    off, rho = oracle.route_invert(w, good.numpy())
    assert (b.offset.cpu().numpy() == off).all() and (b.rho.cpu().numpy() == rho).all()


def test_backward_full_32k_sampled():
    w = [x for x in synth.WORKLOADS if x.name == "mha_bf16_32k"][0]
    (Q, K, V, dO), g = _forward_backward(w)
    off, rho = oracle.route_invert(w, g["idx"])
    assert (g["offset"] == off).all() and (g["rho"] == rho).all()
    rng = np.random.default_rng(3)
    total = w.B * w.Hq * w.Nq
    rows = np.unique(np.concatenate([rng.choice(total, 160, replace=False), [0, total - 1]]))
    _close(w, g["dQ"].reshape(-1, w.d)[rows], oracle.attend_bwd_q(w, Q, K, V, dO, g["idx"], rows), "dQ")
    nb = (w.N + w.b - 1) // w.b
    blocks = [(0, 0), (0, nb - 1), (3, 1), (7, 3), (9, 100), (12, nb - 2), (15, nb // 2), (15, 257)]
    dK, dV = oracle.attend_bwd_kv(w, Q, K, V, dO, g["idx"], blocks)
    gk = g["dK"].reshape(w.B * w.Hkv, nb, w.b, w.d)
    gv = g["dV"].reshape(w.B * w.Hkv, nb, w.b, w.d)
    _close(w, np.stack([gk[u, j] for u, j in blocks]), dK, "dK")
    _close(w, np.stack([gv[u, j] for u, j in blocks]), dV, "dV")
    # identities on every unit, up to rounding that adds like a random walk over keys and rows and
    # is compared with the L2 norm over the keys:
    #   sum_k dV_k = sum_t dO_t (each row's probabilities sum to one): only the bf16 rounding of
    #     P and of the outputs enters, well under 5 %;
    #   sum_k dK_k = 0 (each row's dS sums to zero): D_t is formed from the bf16 output O, and its
    #     error (up to |dO_t| |O_t| 2^-9) enters every row's sum, so this is only a coarse check
    sk = g["dK"].reshape(w.B * w.Hkv, w.N, w.d).astype(np.float64)
    sv = g["dV"].reshape(w.B * w.Hkv, w.N, w.d).astype(np.float64)
    do = dO.float().numpy().reshape(w.B * w.Hkv, -1, w.d).astype(np.float64)
    assert (np.abs(sv.sum(1) - do.sum(1)) <= 0.05 * np.linalg.norm(sv, axis=1)).all()
    assert (np.abs(sk.sum(1)) <= 0.25 * np.linalg.norm(sk, axis=1)).all()



@pytest.mark.parametrize("name", ["gqa_bf16_64k", "mha_bf16_1m"])
def test_backward_full_size_sampled(name):
    """The larger workloads at full size: route inversion bit-exact, sampled dQ rows, and dK/dV of
    sampled key blocks (chosen among blocks routed by at most 12 query blocks, so that the oracle,
    which recomputes every attending row in double, finishes in seconds). Only the sampled pieces
    are copied back to the host."""
    w = [x for x in synth.WORKLOADS if x.name == name][0]
    s = P.shape_of(w)
    Q, K, V, _ = synth.generate(w)
    dO = synth.grad_output(w)
    Qd, Kd, Vd, dOd = (t.cuda() for t in (Q, K, V, dO))
    fwd = P.Buffers(s)
    bwd = P.BackwardBuffers(s)
    P.run(s, Qd, Kd, Vd, fwd)
    P.run_backward(s, Qd, Kd, Vd, dOd, fwd, bwd)
    torch.cuda.synchronize()
    assert int(fwd.status.item()) == 0
    idx = fwd.idx.cpu().numpy()
    off_g, rho_g = bwd.offset.cpu().numpy(), bwd.rho.cpu().numpy()
    off, rho = oracle.route_invert(w, idx)
    assert (off_g == off).all() and (rho_g == rho).all()
    rng = np.random.default_rng(11)
    total = w.B * w.Hq * w.Nq
    rows = np.unique(np.concatenate([rng.choice(total, 48, replace=False), [0, total - 1]]))
    dQ_g = bwd.dQ.reshape(-1, w.d)[torch.as_tensor(rows).cuda()].float().cpu().numpy()
    _close(w, dQ_g, oracle.attend_bwd_q(w, Q, K, V, dO, idx, rows), "dQ")
    nb = (w.N + w.b - 1) // w.b
    counts = np.diff(off, axis=1)  # query blocks routing to each key block
    U = w.B * w.Hkv
    pool = [(u, j) for u in (0, U // 2, U - 1) for j in range(nb) if counts[u, j] <= 12]
    pick = [pool[k] for k in rng.choice(len(pool), size=min(4, len(pool)), replace=False)] + [(U - 1, nb - 1)]
    dK, dV = oracle.attend_bwd_kv(w, Q, K, V, dO, idx, pick)
    gk = bwd.dK.reshape(U, nb, w.b, w.d)
    gv = bwd.dV.reshape(U, nb, w.b, w.d)
    _close(w, np.stack([gk[u, j].float().cpu().numpy() for u, j in pick]), dK, "dK")
    _close(w, np.stack([gv[u, j].float().cpu().numpy() for u, j in pick]), dV, "dV")
    del fwd, bwd, Qd, Kd, Vd, dOd
    torch.cuda.empty_cache()
