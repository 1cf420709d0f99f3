"""PHBA prefix-state branch on the GPU against the oracle (phba_state_build, phba_forward).

PHBA summary 2.2, 3.2, A.1.1: M-slot key and value states from one slot-wise
retention and one write gate, stored before each block; 3.3, A.1.3: one softmax
over the exact tokens and the slots of the current block's state and of each
routed block's state. The oracle builds its own states from the same inputs (a
plain sequential recurrence in double) and attends with its own selection, so
nothing the GPU computes feeds it.

Tolerances: states fp32: max-abs <= 1e-4 * (1 + |x|) (chunkwise fp32 against
a sequential double recurrence); bf16 states are rounded to bf16 when stored
(2^-9 relative): max-abs <= 4e-3 |x| + 1e-3 max |x|. Attention: the
bsa_forward tolerances (bf16 max-abs 2e-2, rel-L2 1e-2; fp32 1e-4) for O. For
lse with bf16 states, the rounding of a stored state key moves its slot's score
by at most 2^-9 sum_e |qs_e| |PK_e| / sqrt(d), and lse by at most the largest
such move over the row's slots: the bound is the token path's 2e-3 plus twice
that largest move, computed per row from the oracle's states.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _parity import check_out, fmt
from synth import BF16, F32

pytestmark = pytest.mark.gpu

W0 = synth.WORKLOADS[0]
CASES = [
    # tcgen05 path: bf16, d=128, Qs = Q, M a multiple of 64
    (W0.scaled(name="phba_tc_mha", B=1, Hq=4, Hkv=4, N=4096 + 64, Nq=4096 + 64, d=128, b=64, topk=6, cap=12,
               dtype=BF16, seed=71), 64, False),
    (W0.scaled(name="phba_tc_gqa_ragged", B=2, Hq=8, Hkv=2, N=3000, Nq=3000, d=128, b=64, topk=6, cap=12,
               dtype=BF16, seed=72), 128, False),
    (W0.scaled(name="phba_tc_b128", B=1, Hq=2, Hkv=2, N=4173, Nq=4173, d=128, b=128, topk=4, cap=8, dtype=BF16,
               seed=73), 64, False),
    # the largest state: eight 32-slot tiles in the one-pass build, four state tiles per block in attention
    (W0.scaled(name="phba_tc_mha_m256", B=1, Hq=2, Hkv=2, N=2048 + 64 + 17, Nq=2048 + 64 + 17, d=128, b=64, topk=5,
               cap=10, dtype=BF16, seed=77), 256, False),
    # CUDA-core path: fp32, a separate state query, M not a multiple of 64
    (W0.scaled(name="phba_simt_f32", B=1, Hq=4, Hkv=2, N=1000, Nq=1000, d=64, b=32, topk=5, cap=10, dtype=F32,
               seed=74), 5, True),
    (W0.scaled(name="phba_simt_bf16_m96", B=1, Hq=2, Hkv=2, N=2048, Nq=2048, d=128, b=64, topk=4, cap=8,
               dtype=BF16, seed=75), 96, True),
    # decode (CUDA cores)
    (W0.scaled(name="phba_decode", B=3, Hq=8, Hkv=2, N=5000, Nq=1, q_offset=4999, d=128, b=64, topk=8, cap=16,
               dtype=BF16, seed=76, n_needle=4, needle_mode=synth.NEEDLE_DECODE), 64, False),
]


def _close_states(w, got, ref):
    got = got.float().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(got - ref)
    if w.dtype == F32:
        bound = 1e-4 * (1 + np.abs(ref))
    else:
        bound = 4e-3 * np.abs(ref) + 1e-3 * np.abs(ref).max()
    assert (err <= bound).all(), f"states: max err {err.max():.3e} (at |ref| {np.abs(ref).flat[err.argmax()]:.3e})"
    return float(err.max())


def _lse_bound(w, Q, Qs, idx, rows, PK):
    """Per-row lse tolerance (see the module docstring)."""
    base = 1e-4 if w.dtype == F32 else 2e-3
    if w.dtype == F32:
        return np.full(len(rows), base)
    q = (Qs if Qs is not None else Q).double().numpy().reshape(w.B, w.Hq, w.Nq, w.d)
    first = w.q_offset // w.b
    out = np.empty(len(rows))
    for k, r in enumerate(rows):
        t, bh = r % w.Nq, r // w.Nq
        bi, hq = divmod(bh, w.Hq)
        hk = hq // w.G
        i = (w.q_offset + t) // w.b
        blocks = [j for j in idx[bi, hk, i - first] if j >= 1] + ([i] if i >= 1 else [])
        u = bi * w.Hkv + hk
        worst = max((np.abs(PK[u, j]) @ np.abs(q[bi, hq, t])).max() for j in blocks) if blocks else 0.0
        out[k] = base + 2 * 2.0 ** -9 * worst / np.sqrt(w.d)
    return out


def _check_states_attention(w, O_g, lse, O_o, lse_o, bound):
    e, r = check_out(w, O_g, np.asarray(lse_o), O_o, lse_o)  # O only: lse checked against its own bound below
    lerr = np.abs(np.asarray(lse) - lse_o)
    assert (lerr <= bound).all(), f"lse err {lerr.max():.3e} over bound {bound[lerr.argmax()]:.3e}"
    return e, r, float(lerr.max())


def _run(w, M, separate_qs):
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(w)
    Q, K, V, _ = synth.generate(w)
    A, Wg = synth.phba_gates(w, M)
    Qs = synth.state_query(w) if separate_qs else None
    idx_o, _, _ = oracle.select_all(w, Q, K)
    idx_o = idx_o.reshape(w.B, w.Hkv, -1, w.topk)
    dev = [t.cuda() for t in (Q, K, V, A, Wg)]
    Qd, Kd, Vd, Ad, Wd = dev
    st = P.PhbaStates(s, M)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.phba_state_build(s, M, Kd, Vd, Ad, Wd, st.PK, st.PV, st.workspace, status)
    O = torch.empty(Q.shape, dtype=Q.dtype, device="cuda")
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device="cuda")
    idx_d = torch.as_tensor(np.ascontiguousarray(idx_o)).cuda()
    P.phba_forward(s, Qd, Kd, Vd, idx_d, O, lse, Qs=None if Qs is None else Qs.cuda(), M=M, PK=st.PK, PV=st.PV,
                   status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return Q, K, V, A, Wg, Qs, idx_o, st, O, lse


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_phba_states_and_attention_match_the_oracle(case):
    w, M, separate_qs = case
    Q, K, V, A, Wg, Qs, idx_o, st, O, lse = _run(w, M, separate_qs)
    PK_o, PV_o = oracle.prefix_states(w, M, K, V, A, Wg)
    ek = _close_states(w, st.PK, PK_o)
    ev = _close_states(w, st.PV, PV_o)
    total = w.B * w.Hq * w.Nq
    rng = np.random.default_rng(w.seed)
    rows = np.arange(total) if total <= 12000 else np.unique(np.concatenate(
        [rng.choice(total, 3000, replace=False), [0, total - 1]]))
    O_o, lse_o = oracle.attend_states(w, Q, K, V, idx_o, rows, PK_o, PV_o, Qs=Qs)
    bound = _lse_bound(w, Q, Qs, idx_o, rows, PK_o)
    e, r, le = _check_states_attention(w, O.float().cpu().double().numpy().reshape(-1, w.d)[rows],
                                       lse.cpu().double().numpy().reshape(-1)[rows], O_o, lse_o, bound)
    # the states matter: attention without them differs from attention with them
    O_t, _ = oracle.attend(w, Q, K, V, idx_o, rows)
    assert np.abs(O_t - O_o).max() > 10 * max(e, 1e-6)
    print(f"\n{fmt(w)} M={M}: states max err {ek:.2e} / {ev:.2e}; attention on {len(rows)} rows max-abs {e:.2e} "
          f"rel-L2 {r:.2e}, lse {le:.2e} (bound {bound.min():.1e}..{bound.max():.1e})")


def test_phba_forward_without_states_is_bsa_forward():
    import hierarchical_block_sparse_pyr_b200 as P

    w = CASES[0][0]
    s = P.shape_of(w)
    Q, K, V, _ = (t.cuda() if isinstance(t, torch.Tensor) else t for t in synth.generate(w))
    buf = P.Buffers(s)
    P.run(s, Q, K, V, buf)
    O2 = torch.empty_like(buf.O)
    lse2 = torch.empty_like(buf.lse)
    P.phba_forward(s, Q, K, V, buf.idx, O2, lse2, M=0, status=buf.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    assert torch.equal(O2, buf.O) and torch.equal(lse2, buf.lse)


def test_phba_full_size_32k_with_128_slots():
    """The 32K bf16 MHA workload with 128-slot states: states on two sampled units, attention on sampled
    rows of every sampled block, through the tcgen05 path."""
    import hierarchical_block_sparse_pyr_b200 as P

    w = synth.BY_NAME["mha_bf16_32k"]
    M = 128
    s = P.shape_of(w)
    Q, K, V, _ = synth.generate(w)
    A, Wg = synth.phba_gates(w, M)
    Qd, Kd, Vd, Ad, Wd = (t.cuda() for t in (Q, K, V, A, Wg))
    st = P.PhbaStates(s, M)
    buf = P.Buffers(s)
    P.pyr_build(s, Kd, buf.pyr, buf.status)
    P.pyr_select(s, Qd, buf.pyr, buf.idx, None, buf.status)
    P.phba_state_build(s, M, Kd, Vd, Ad, Wd, st.PK, st.PV, st.workspace, buf.status)
    P.phba_forward(s, Qd, Kd, Vd, buf.idx, buf.O, buf.lse, M=M, PK=st.PK, PV=st.PV, status=buf.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    units = [0, w.B * w.Hkv - 1]
    PK_o, PV_o = oracle.prefix_states(w, M, K, V, A, Wg, units)
    PKg = st.PK.reshape(w.B * w.Hkv, *st.PK.shape[2:])
    PVg = st.PV.reshape(w.B * w.Hkv, *st.PV.shape[2:])
    for k, u in enumerate(units):
        _close_states(w, PKg[u], PK_o[k])
        _close_states(w, PVg[u], PV_o[k])
    # attention: the oracle needs every unit's states for the rows it checks; build them for the
    # sampled units only and check rows of those units (their routes only reach their own states)
    full_PK = np.zeros((w.B * w.Hkv, w.nb, M, w.d))
    full_PV = np.zeros_like(full_PK)
    for k, u in enumerate(units):
        full_PK[u], full_PV[u] = PK_o[k], PV_o[k]
    rng = np.random.default_rng(5)
    rows = []
    for u in units:
        for qb in sorted(set([0, 1, w.nb - 1] + rng.choice(w.nb, 6, replace=False).tolist())):
            ts = rng.choice(np.arange(qb * w.b, (qb + 1) * w.b), 4, replace=False)
            rows += [u * w.Nq + int(t) for t in ts]
    rows = np.array(sorted(rows), dtype=np.int64)
    idx_g = buf.idx.cpu().numpy()
    O_o, lse_o = oracle.attend_states(w, Q, K, V, idx_g, rows, full_PK, full_PV)
    bound = _lse_bound(w, Q, None, idx_g, rows, full_PK)
    e, r, le = _check_states_attention(w, buf.O.float().cpu().double().numpy().reshape(-1, w.d)[rows],
                                       buf.lse.cpu().double().numpy().reshape(-1)[rows], O_o, lse_o, bound)
    print(f"\n{fmt(w)} M={M}: attention on {len(rows)} rows max-abs {e:.2e} rel-L2 {r:.2e}, lse {le:.2e}")
