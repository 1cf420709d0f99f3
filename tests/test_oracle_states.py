"""Pins of the oracle's PHBA prefix-state branch (oracle.prefix_states, oracle.attend_states).

PHBA summary, 2.2 and 3.2: a gated recurrence with one slot-wise retention and
one write gate shared by the key and the value state builds M-slot prefix
states, stored before each block and summarising the causal context before it;
A.1.1: computed chunkwise with log-A prefix sums, resetting at a sequence
start. 3.3 and A.1.3: one softmax over exact tokens and prefix-state slots (the
current block's state and the states aligned with the routed blocks).
Reading of the write form: S[s] <- a_t[s] S[s] + w_t[s] x_t.

Pinned by:
  - closed forms: retention 1 and write 1 give running sums; retention 0 keeps the
    last token before the boundary; a constant retention gives a geometric sum;
  - an independent restatement of the chunkwise form (per block: log-A prefix
    sums, a decay-weighted matrix product, then the carry from block to block);
  - attention: torch's float64 softmax over key sets assembled from idx and the
    states; zero states give the token-only result renormalised by the slot count
    (closed form); no states give ora_attend bit for bit; future tokens change
    nothing.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import BF16, F32, Workload


def W(**kw):
    base = dict(name="st", B=1, Hq=2, Hkv=1, N=200, Nq=200, q_offset=0, d=8, b=16, topk=3, cap=6, dtype=F32, seed=0,
                n_needle=0, needle_mode=0)
    base.update(kw)
    return Workload(**base)


def gates(w, M, seed):
    a = torch.sigmoid(synth.normal(seed, 20, (w.B, w.Hkv, w.N, M)) + 1.5).contiguous()
    wr = torch.sigmoid(synth.normal(seed, 21, (w.B, w.Hkv, w.N, M))).contiguous()
    return a, wr


def kv(w, seed):
    K = synth.normal(seed, 11, (w.B, w.Hkv, w.N, w.d), w.torch_dtype)
    V = synth.normal(seed, 12, (w.B, w.Hkv, w.N, w.d), w.torch_dtype)
    return K, V


def chunkwise(X, A, Wr, b):
    """Chunkwise form: within block j, log-A prefix sums give each token's decay to the block end;
    the block's contribution is one matrix product; the state carries from block to block."""
    N, d = X.shape
    M = A.shape[1]
    nb = -(-N // b)
    S = np.zeros((M, d))
    out = np.zeros((nb, M, d))
    for j in range(nb):
        out[j] = S
        t0, t1 = j * b, min((j + 1) * b, N)
        la = np.cumsum(np.log(A[t0:t1]), axis=0)
        decay = np.exp(la[-1][None, :] - la) * Wr[t0:t1]  # [n, M]
        S = np.exp(la[-1])[:, None] * S + decay.T @ X[t0:t1]
    return out


@pytest.mark.parametrize("dtype", [F32, BF16])
def test_unit_gates_give_running_sums(dtype):
    w = W(dtype=dtype, N=203, Nq=203)
    M = 4
    K, V = kv(w, 1)
    one = torch.ones((w.B, w.Hkv, w.N, M))
    PK, PV = oracle.prefix_states(w, M, K, V, one, one)
    k, v = K.double().numpy()[0, 0], V.double().numpy()[0, 0]
    for j in range(w.nb):
        for m in range(M):
            np.testing.assert_allclose(PK[0, j, m], k[:j * w.b].sum(0), atol=1e-12)
            np.testing.assert_allclose(PV[0, j, m], v[:j * w.b].sum(0), atol=1e-12)


def test_zero_retention_keeps_the_last_token():
    w = W()
    M = 3
    K, V = kv(w, 2)
    zero, one = torch.zeros((w.B, w.Hkv, w.N, M)), torch.ones((w.B, w.Hkv, w.N, M))
    PK, PV = oracle.prefix_states(w, M, K, V, zero, one)
    k, v = K.double().numpy()[0, 0], V.double().numpy()[0, 0]
    assert (PK[0, 0] == 0).all() and (PV[0, 0] == 0).all()
    for j in range(1, w.nb):
        for m in range(M):
            np.testing.assert_array_equal(PK[0, j, m], k[j * w.b - 1])
            np.testing.assert_array_equal(PV[0, j, m], v[j * w.b - 1])


def test_constant_retention_gives_a_geometric_sum():
    w = W()
    M = 2
    K, V = kv(w, 3)
    A = torch.empty((w.B, w.Hkv, w.N, M))
    A[..., 0], A[..., 1] = 0.5, 0.9
    Wr = torch.full((w.B, w.Hkv, w.N, M), 0.25)
    PK, _ = oracle.prefix_states(w, M, K, V, A, Wr)
    k = K.double().numpy()[0, 0]
    for j in range(w.nb):
        T = j * w.b
        for m, a in enumerate((0.5, float(np.float32(0.9)))):  # the gates are float32 inputs
            want = sum(0.25 * a ** (T - 1 - t) * k[t] for t in range(T)) if T else np.zeros(w.d)
            np.testing.assert_allclose(PK[0, j, m], want, atol=1e-12)


@pytest.mark.parametrize("w", [W(B=2, Hq=4, Hkv=2, N=1000, Nq=1000, d=16, b=32),
                               W(N=777, Nq=777, d=8, b=16, dtype=BF16)], ids=["gqa", "ragged_bf16"])
def test_sequential_recurrence_equals_the_chunkwise_form(w):
    M = 6
    K, V = kv(w, 4)
    A, Wr = gates(w, M, 4)
    PK, PV = oracle.prefix_states(w, M, K, V, A, Wr)
    for u in range(w.B * w.Hkv):
        bi, hk = divmod(u, w.Hkv)
        a, wr = A[bi, hk].double().numpy(), Wr[bi, hk].double().numpy()
        np.testing.assert_allclose(PK[u], chunkwise(K[bi, hk].double().numpy(), a, wr, w.b), rtol=1e-10, atol=1e-10)
        np.testing.assert_allclose(PV[u], chunkwise(V[bi, hk].double().numpy(), a, wr, w.b), rtol=1e-10, atol=1e-10)


def test_states_ignore_later_tokens():
    w = W(N=320, Nq=320)
    M = 3
    K, V = kv(w, 5)
    A, Wr = gates(w, M, 5)
    PK, PV = oracle.prefix_states(w, M, K, V, A, Wr)
    cut = 7 * w.b
    K2, V2, A2, W2 = K.clone(), V.clone(), A.clone(), Wr.clone()
    K2[..., cut:, :] *= -3
    V2[..., cut:, :] += 1
    A2[..., cut:, :] = 0.1
    W2[..., cut:, :] = 0.9
    PK2, PV2 = oracle.prefix_states(w, M, K2, V2, A2, W2)
    assert np.array_equal(PK[:, :8], PK2[:, :8]) and np.array_equal(PV[:, :8], PV2[:, :8])
    assert not np.array_equal(PK[:, 8:], PK2[:, 8:])


# ---- attention over tokens and state slots ----

def _routes(w, Q, K, seed):
    idx, _, _ = oracle.select_all(w, Q, K)
    nqb = oracle.num_qblocks(w)
    return idx.reshape(w.B, w.Hkv, nqb, w.topk)


def _reference_row(w, Q, K, V, Qs, idx, PK, PV, row):
    """One row by torch's float64 softmax over the key set assembled from idx and the states."""
    t, bh = row % w.Nq, row // w.Nq
    bi, hq = divmod(bh, w.Hq)
    hk = hq // w.G
    p = w.q_offset + t
    i = p // w.b
    first = w.q_offset // w.b
    u = bi * w.Hkv + hk
    blocks = [int(j) for j in idx[bi, hk, i - first] if j >= 0]
    pos = [x for j in blocks for x in range(j * w.b, min((j + 1) * w.b, w.N))] + list(range(i * w.b, p + 1))
    k = K[bi, hk, pos].double()
    v = V[bi, hk, pos].double()
    q = Q[bi, hq, t].double()
    scores = [k @ q / np.sqrt(w.d)]
    vals = [v]
    if PK is not None:
        qs = (Qs if Qs is not None else Q)[bi, hq, t].double()
        for j in blocks + [i]:
            if j >= 1:
                scores.append(torch.from_numpy(PK[u, j]) @ qs / np.sqrt(w.d))
                vals.append(torch.from_numpy(PV[u, j]))
    sc = torch.cat(scores)
    pr = torch.softmax(sc, 0)
    return (pr[:, None] * torch.cat(vals)).sum(0).numpy(), float(torch.logsumexp(sc, 0))


@pytest.mark.parametrize("w", [W(B=1, Hq=4, Hkv=2, N=500, Nq=500, d=16, b=32, topk=4, cap=8),
                               W(B=2, Hq=2, Hkv=1, N=300, Nq=1, q_offset=299, d=8, b=16, topk=3, cap=6),
                               W(N=256, Nq=128, q_offset=128, d=8, b=16, topk=3, cap=6, dtype=BF16)],
                         ids=["prefill_gqa", "decode", "chunk_bf16"])
def test_attention_over_tokens_and_states_equals_one_softmax(w):
    M = 5
    Q = synth.normal(6, 10, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    Qs = synth.normal(6, 13, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    K, V = kv(w, 6)
    A, Wr = gates(w, M, 6)
    PK, PV = oracle.prefix_states(w, M, K, V, A, Wr)
    idx = _routes(w, Q, K, 6)
    rows = np.arange(w.B * w.Hq * w.Nq)
    for qs in (None, Qs):
        O, lse = oracle.attend_states(w, Q, K, V, idx, rows, PK, PV, Qs=qs)
        for r in rows[:: max(1, len(rows) // 40)]:
            o_ref, l_ref = _reference_row(w, Q, K, V, qs, idx, PK, PV, int(r))
            np.testing.assert_allclose(O[r], o_ref, atol=1e-12)
            assert abs(lse[r] - l_ref) < 1e-12


def test_zero_states_renormalise_the_token_result():
    """Write gates of 0 leave every state at zero: each of the M slots of every attended state then
    scores 0, so O = O_tok * exp(lse_tok - lse) and exp(lse) = exp(lse_tok) + (number of slots)."""
    w = W(B=1, Hq=2, Hkv=1, N=400, Nq=400, d=8, b=16, topk=3, cap=6)
    M = 4
    Q = synth.normal(7, 10, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    K, V = kv(w, 7)
    A, _ = gates(w, M, 7)
    PK, PV = oracle.prefix_states(w, M, K, V, A, torch.zeros_like(A))
    assert not PK.any() and not PV.any()
    idx = _routes(w, Q, K, 7)
    rows = np.arange(w.B * w.Hq * w.Nq)
    O_t, l_t = oracle.attend(w, Q, K, V, idx, rows)
    O_s, l_s = oracle.attend_states(w, Q, K, V, idx, rows, PK, PV)
    for r in rows:
        i = (r % w.Nq) // w.b
        n_states = sum(1 for j in idx[0, 0, i] if j >= 1) + (1 if i >= 1 else 0)
        assert abs(np.exp(l_s[r]) - (np.exp(l_t[r]) + M * n_states)) <= 1e-9 * np.exp(l_s[r])
        np.testing.assert_allclose(O_s[r], O_t[r] * np.exp(l_t[r] - l_s[r]), atol=1e-12)


def test_no_states_is_the_token_branch_bit_for_bit():
    w = W(B=1, Hq=2, Hkv=2, N=300, Nq=300, d=8, b=16, topk=3, cap=6)
    Q = synth.normal(8, 10, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    K, V = kv(w, 8)
    idx = _routes(w, Q, K, 8)
    rows = np.arange(w.B * w.Hq * w.Nq)
    O_t, l_t = oracle.attend(w, Q, K, V, idx, rows)
    O_s, l_s = oracle.attend_states(w, Q, K, V, idx, rows, None, None)
    assert np.array_equal(O_t, O_s) and np.array_equal(l_t, l_s)


def test_attention_with_states_ignores_future_tokens():
    w = W(B=1, Hq=2, Hkv=1, N=320, Nq=320, d=8, b=16, topk=3, cap=6)
    M = 3
    Q = synth.normal(9, 10, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    K, V = kv(w, 9)
    A, Wr = gates(w, M, 9)
    idx = _routes(w, Q, K, 9)
    PK, PV = oracle.prefix_states(w, M, K, V, A, Wr)
    cut = 150
    rows = np.array([h * w.Nq + t for h in range(w.Hq) for t in range(cut)])
    O1, l1 = oracle.attend_states(w, Q, K, V, idx, rows, PK, PV)
    K2, V2, A2 = K.clone(), V.clone(), A.clone()
    K2[..., cut:, :] += 2
    V2[..., cut:, :] *= -1
    A2[..., cut:, :] = 0.3
    PK2, PV2 = oracle.prefix_states(w, M, K2, V2, A2, Wr)
    O2, l2 = oracle.attend_states(w, Q, K2, V2, idx, rows, PK2, PV2)
    assert np.array_equal(O1, O2) and np.array_equal(l1, l2)
