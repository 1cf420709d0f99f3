"""Pins of the CPU oracle against things other than itself.

Each test ties one step of the oracle to a closed form, a library routine,
brute force, a hand-derived worked example or an invariant of the method, so
that a dropped term, a wrong sign or index, or a transposed operand fails at
least one of them:

  pyramid   node means == numpy means of the raw key rows (closed form)
  score     == brute-force per-key LogSumExp when all keys under the node are
            equal (Jensen equality case); <= it otherwise (Jensen bound)
  walk      hand-derived examples (tests/golden/walk_trap.txt); survivor and
            completeness invariants; start-at-root == start-at-s0; flat top-K
            when cap >= nb; causality; ties to the lower index
  attention == torch SDPA in float64 with the block mask built from idx;
            dense identity when every causal block is selected; local causal
            attention when none is; causality
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
import synth
from synth import BF16, F32, Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def W(**kw):
    base = dict(name="t", B=1, Hq=1, Hkv=1, N=256, Nq=256, q_offset=0, d=8, b=16, topk=2, cap=4, dtype=F32, seed=0,
                n_needle=0, needle_mode=0)
    base.update(kw)
    return Workload(**base)


def rand_qkv(w, seed, k_scale=1.0):
    dt = w.torch_dtype
    Q = synth.normal(seed, 10, (w.B, w.Hq, w.Nq, w.d), dt)
    K = synth.normal(seed, 11, (w.B, w.Hkv, w.N, w.d), dt, scale=k_scale)
    V = synth.normal(seed, 12, (w.B, w.Hkv, w.N, w.d), dt)
    return Q, K, V


def query_rows(w, Q, bi, hk, i):
    """All query rows (over the kv group's heads) whose position is in block i."""
    G = w.Hq // w.Hkv
    p0, p1 = max(i * w.b, w.q_offset), min((i + 1) * w.b, w.q_offset + w.Nq)
    Qd = Q.double().numpy()
    return np.concatenate([Qd[bi, hk * G + g, p0 - w.q_offset:p1 - w.q_offset] for g in range(G)], axis=0)


# ---------------------------------------------------------------- pyramid --

@pytest.mark.parametrize("N,b,dtype", [(256, 16, F32), (250, 16, F32), (1000, 64, BF16), (64 * 37 + 5, 64, BF16),
                                       (64, 64, F32)])
def test_pyramid_node_means_closed_form(N, b, dtype):
    w = W(B=2, Hq=2, Hkv=2, N=N, Nq=N, b=b, dtype=dtype)
    _, K, _ = rand_qkv(w, 1)
    pyr = oracle.pyramid(w, K, [0, 1, 2, 3])
    Kd = K.double().numpy().reshape(4, N, w.d)
    levels = oracle.level_offsets(w)
    nb = -(-N // b)
    assert len(levels) == (math.ceil(math.log2(nb)) if nb > 1 else 0) + 1
    assert pyr.shape[1] == sum(n for _, n in levels)
    for l, (off, n) in enumerate(levels):
        assert n == -(-nb // (1 << l))
        for m in range(n):
            t0, t1 = m * (1 << l) * b, min((m + 1) * (1 << l) * b, N)
            np.testing.assert_allclose(pyr[:, off + m], Kd[:, t0:t1].mean(axis=1), rtol=0, atol=1e-12)
    np.testing.assert_allclose(pyr[:, -1], Kd.mean(axis=1), rtol=0, atol=1e-12)


def test_pyramid_level_counts_of_the_workloads():
    # "64 blocks, 6 pyramid levels" and "8192 blocks, 13 levels": pooling steps L = ceil(log2 nb)
    assert len(oracle.level_offsets(synth.WORKLOADS[0])) - 1 == 6
    assert len(oracle.level_offsets(synth.WORKLOADS[4])) - 1 == 13


# ------------------------------------------------------------------ score --

def _const_node_case(w, seed, level, m, i):
    """Random inputs where every key under node (level, m) equals one vector."""
    Q, K, V = rand_qkv(w, seed)
    t0, t1 = m * (1 << level) * w.b, min((m + 1) * (1 << level) * w.b, w.N)
    vec = synth.normal(seed, 20, (w.d,), w.torch_dtype) * 1.5
    K[:, :, t0:t1] = vec
    return Q, K


@pytest.mark.parametrize("case", [
    dict(w=dict(), level=0, m=3, i=9),  # full level-0 node
    dict(w=dict(), level=2, m=1, i=10),  # full level-2 node
    dict(w=dict(), level=2, m=2, i=10),  # straddles block 10: valid part [8, 10)
    dict(w=dict(Hq=4, Hkv=2, B=2), level=3, m=0, i=15),  # GQA: rows of both heads
    dict(w=dict(Hq=4, Hkv=1, N=250, Nq=1, q_offset=249), level=3, m=1, i=15),  # decode, ragged tail
    dict(w=dict(d=64, b=32, N=640, Nq=640, dtype=BF16), level=1, m=4, i=9),  # straddling, bf16
])
def test_score_equals_bruteforce_lse_for_constant_keys(case):
    """Jensen equality: with equal keys, ln sum_r sum_k exp(q_r.k/sqrt d) == LSE_r(q_r.kbar/sqrt d) + ln n."""
    w = W(**case["w"])
    level, m, i = case["level"], case["m"], case["i"]
    Q, K = _const_node_case(w, 3, level, m, i)
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    first = w.q_offset // w.b
    for unit in units:
        bi, hk = divmod(unit, w.Hkv)
        s, n = oracle.node_score(w, Q, pyr[unit], unit, i - first, level, m)
        j0 = m << level
        j1 = min((m + 1) << level, i)
        keys = K.double().numpy()[bi, hk, j0 * w.b:min(j1 * w.b, w.N)]
        rows = query_rows(w, Q, bi, hk, i)
        exact = logsumexp((rows @ keys.T).ravel() / math.sqrt(w.d))
        assert n == keys.shape[0]
        assert abs(s - exact) < 1e-10, (s, exact)


def test_score_jensen_bound_on_random_keys():
    w = W(Hq=2, Hkv=1, N=512, Nq=512, b=16, d=16)
    Q, K, _ = rand_qkv(w, 5, k_scale=1.3)
    pyr = oracle.pyramid(w, K, [0])
    Kd = K.double().numpy()[0, 0]
    checked = 0
    for i in (5, 17, 31):
        rows = query_rows(w, Q, 0, 0, i)
        for level in range(0, 5):
            for m in range(0, (32 >> level) + 1):
                s, n = oracle.node_score(w, Q, pyr[0], 0, i, level, m)
                j0, j1 = m << level, min((m + 1) << level, i)
                if j0 >= i:
                    assert s == -math.inf
                    continue
                keys = Kd[j0 * w.b:j1 * w.b]
                exact = logsumexp((rows @ keys.T).ravel() / math.sqrt(w.d))
                assert s < exact + 1e-12
                checked += 1
    assert checked > 40


# ------------------------------------------------------------------- walk --

def _read_trap():
    cases = []
    with open(os.path.join(GOLDEN, "walk_trap.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, keys, i, cap, topk, idx, gap = line.split()
            cases.append((name, [float(x) for x in keys.split(",")], int(i), int(cap), int(topk),
                          [int(x) for x in idx.split(",")], float(gap)))
    return cases


@pytest.mark.parametrize("case", _read_trap(), ids=lambda c: c[0])
def test_walk_hand_derived_examples(case):
    name, keys, i, cap, topk, want_idx, want_gap = case
    w = W(N=9, Nq=9, d=1, b=1, topk=topk, cap=cap)
    Q = torch.ones((1, 1, 9, 1), dtype=torch.float32)
    K = torch.tensor(keys, dtype=torch.float32).reshape(1, 1, 9, 1)
    pyr = oracle.pyramid(w, K, [0])
    idx, gap, _ = oracle.select(w, Q, pyr, [0], [(0, i)])
    assert idx[0].tolist() == want_idx
    assert abs(gap[0] - want_gap) < 1e-5


def _walk_shapes():
    return [
        W(B=1, Hq=2, Hkv=2, N=1024, Nq=1024, b=16, d=16, topk=4, cap=8),  # nb=64, s0=3
        W(B=2, Hq=4, Hkv=2, N=1000, Nq=1000, b=16, d=8, topk=3, cap=6),  # ragged, GQA
        W(B=2, Hq=4, Hkv=1, N=2048, Nq=1, q_offset=2047, b=32, d=16, topk=4, cap=8),  # decode
        W(B=1, Hq=1, Hkv=1, N=4096, Nq=4096, b=32, d=8, topk=8, cap=16),  # nb=128
    ]


@pytest.mark.parametrize("w", _walk_shapes(), ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_walk_output_invariants(w):
    Q, K, _ = rand_qkv(w, 7, k_scale=1.2)
    idx, gap, ncand = oracle.select_all(w, Q, K)
    first = w.q_offset // w.b
    for u in range(idx.shape[0]):
        for qb in range(idx.shape[1]):
            i = first + qb
            sel = idx[u, qb]
            k = min(w.topk, i)
            assert (sel[:k] >= 0).all() and (sel[k:] == -1).all()
            assert (np.diff(sel[:k]) > 0).all() and (sel[:k] < i).all()
            assert (ncand[u, qb] <= w.cap).all()
            if i <= w.topk and i <= w.cap // 2:
                assert gap[u, qb] == math.inf


def _top_set(scores, keep):
    order = sorted(scores, key=lambda t: (-t[1], t[0]))
    return {m for m, _ in order[:keep]}


@pytest.mark.parametrize("w", _walk_shapes(), ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_walk_survivors_and_completeness(w):
    """Survivors at s0 are the top cap/2 of all valid s0 nodes; globally dominant paths are found."""
    Q, K, _ = rand_qkv(w, 8, k_scale=1.2)
    units = list(range(w.B * w.Hkv))
    pyr = oracle.pyramid(w, K, units)
    nb = w.nb
    s0 = 0
    while -(-nb // (1 << s0)) > w.cap:
        s0 += 1
    first = w.q_offset // w.b
    nqb = oracle.num_qblocks(w)
    qbs = sorted(set([nqb - 1, nqb // 2, nqb // 3, max(nqb - 7, 0)]))
    pruned_somewhere = 0
    for unit in units[:2]:
        for qb in qbs:
            i = first + qb
            idx, _, _ = oracle.select(w, Q, pyr, units, [(unit, qb)])
            sel = set(int(j) for j in idx[0] if j >= 0)
            lvl_scores = {}
            for l in range(0, s0 + 1):
                n_l = -(-nb // (1 << l))
                lvl_scores[l] = [(m, oracle.node_score(w, Q, pyr[unit], unit, qb, l, m)[0]) for m in range(n_l)
                                 if (m << l) < i]
            top_s0 = _top_set(lvl_scores[s0], w.cap // 2)
            for j in sel:
                assert (j >> s0) in top_s0
            if len(lvl_scores[s0]) > w.cap // 2:
                pruned_somewhere += 1
            flat_top = _top_set(lvl_scores[0], w.topk)
            for j in flat_top:
                if all((j >> l) in _top_set(lvl_scores[l], w.cap // 2) for l in range(1, s0 + 1)):
                    assert j in sel
            assert len(sel) == min(w.topk, i)
    assert pruned_somewhere > 0


@pytest.mark.parametrize("w", _walk_shapes(), ids=lambda w: f"N{w.N}_Nq{w.Nq}_G{w.G}")
def test_walk_start_at_root_equals_start_at_s0(w):
    Q, K, _ = rand_qkv(w, 9, k_scale=1.2)
    a, ga, _ = oracle.select_all(w, Q, K)
    b, gb, _ = oracle.select_all(w, Q, K, start_level=64)
    assert np.array_equal(a, b)
    assert np.array_equal(ga, gb)


def test_walk_is_flat_topk_when_cap_covers_all_blocks():
    w = W(Hq=2, Hkv=1, N=512, Nq=512, b=16, d=8, topk=5, cap=32)  # nb = 32 <= cap
    Q, K, _ = rand_qkv(w, 10, k_scale=1.2)
    pyr = oracle.pyramid(w, K, [0])
    idx, _, ncand = oracle.select_all(w, Q, K)
    for qb in range(32):
        scores = [(j, oracle.node_score(w, Q, pyr[0], 0, qb, 0, j)[0]) for j in range(qb)]
        want = sorted(_top_set(scores, w.topk))
        got = [int(j) for j in idx[0, qb] if j >= 0]
        assert got == want
        assert (ncand[0, qb, 1:] == 0).all()


def test_walk_ties_go_to_the_lower_index():
    """Duplicate a key block bit-exactly: equal scores at every level; the lower index must win."""
    w = W(N=512, Nq=512, b=16, d=8, topk=1, cap=2)
    Q, K, _ = rand_qkv(w, 11)
    # make blocks 4..7 a bit-exact copy of blocks 0..3, scaled up so they win
    K[:, :, 0:64] *= 3
    K[:, :, 64:128] = K[:, :, 0:64]
    pyr = oracle.pyramid(w, K, [0])
    # query block 9: at level 2 nodes 0 ([0..3]) and 1 ([4..7]) tie exactly
    s_a = oracle.node_score(w, Q, pyr[0], 0, 9, 2, 0)[0]
    s_b = oracle.node_score(w, Q, pyr[0], 0, 9, 2, 1)[0]
    assert s_a == s_b
    idx, gap, _ = oracle.select(w, Q, pyr, [0], [(0, 9)])
    assert idx[0, 0] < 4
    assert gap[0] == 0.0


@pytest.mark.parametrize("w", _walk_shapes()[:2], ids=["mha", "gqa_ragged"])
def test_walk_ignores_keys_at_or_after_the_query_block(w):
    Q, K, _ = rand_qkv(w, 12)
    units = list(range(w.B * w.Hkv))
    for qb in (3, 11, w.nb - 2):
        pyr = oracle.pyramid(w, K, units)
        a, ga, _ = oracle.select(w, Q, pyr, units, [(u, qb) for u in units])
        K2 = K.clone()
        K2[:, :, qb * w.b:] = synth.normal(99, 13, K2[:, :, qb * w.b:].shape, K.dtype) * 5
        pyr2 = oracle.pyramid(w, K2, units)
        b, gb, _ = oracle.select(w, Q, pyr2, units, [(u, qb) for u in units])
        assert np.array_equal(a, b) and np.array_equal(ga, gb)


def test_needle_recall_on_the_tiny_workload():
    w = synth.WORKLOADS[0]
    Q, K, V, owner = synth.generate(w)
    idx, _, _ = oracle.select_all(w, Q, K)
    own = owner.numpy().reshape(w.B * w.Hkv, -1)
    hit = tot = 0
    for u in range(own.shape[0]):
        for j, i in enumerate(own[u]):
            if i > 0:
                tot += 1
                hit += int(j in idx[u, i])
    assert tot > 50 and hit / tot >= 0.95, (hit, tot)


def test_needle_recall_on_a_decode_shaped_workload():
    w = synth.WORKLOADS[3].scaled(B=4, N=16384, q_offset=16383, seed=30)
    Q, K, V, owner = synth.generate(w)
    idx, _, _ = oracle.select_all(w, Q, K)
    own = owner.numpy().reshape(w.B * w.Hkv, -1)
    hit = tot = 0
    for u in range(own.shape[0]):
        for j in np.nonzero(own[u] >= 0)[0]:
            tot += 1
            hit += int(j in idx[u, 0])
    assert tot == w.B * w.Hkv * w.n_needle and hit == tot


# -------------------------------------------------------------- attention --

def _expand(t, G):
    return t.repeat_interleave(G, dim=1)


def _block_mask(w, idx):
    """[B, Hq, Nq, N] boolean mask built directly from idx (+ the causal diagonal block)."""
    G = w.G
    first = w.q_offset // w.b
    mask = torch.zeros((w.B, w.Hq, w.Nq, w.N), dtype=torch.bool)
    for bi in range(w.B):
        for hq in range(w.Hq):
            for t in range(w.Nq):
                p = w.q_offset + t
                i = p // w.b
                mask[bi, hq, t, i * w.b:p + 1] = True
                for j in idx[bi, hq // G, i - first]:
                    if j >= 0:
                        mask[bi, hq, t, j * w.b:min((j + 1) * w.b, w.N)] = True
    return mask


def _sdpa(w, Q, K, V, mask):
    G = w.G
    q, k, v = Q.double(), _expand(K.double(), G), _expand(V.double(), G)
    O = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(w.d)
    lse = torch.logsumexp(s.masked_fill(~mask, -math.inf), dim=-1)
    return O.numpy().reshape(-1, w.d), lse.numpy().reshape(-1)


def _random_valid_idx(w, seed):
    rng = np.random.default_rng(seed)
    nqb = oracle.num_qblocks(w)
    first = w.q_offset // w.b
    idx = -np.ones((w.B, w.Hkv, nqb, w.topk), dtype=np.int32)
    for bi in range(w.B):
        for hk in range(w.Hkv):
            for qb in range(nqb):
                i = first + qb
                k = min(w.topk, i)
                idx[bi, hk, qb, :k] = np.sort(rng.choice(i, size=k, replace=False))
    return idx


ATT_SHAPES = [
    W(B=1, Hq=2, Hkv=2, N=256, Nq=256, b=32, d=16, topk=3, cap=6),
    W(B=2, Hq=4, Hkv=2, N=200, Nq=200, b=32, d=8, topk=2, cap=4, dtype=BF16),  # ragged GQA bf16
    W(B=2, Hq=4, Hkv=1, N=300, Nq=1, q_offset=299, b=32, d=16, topk=3, cap=6),  # decode
]


@pytest.mark.parametrize("w", ATT_SHAPES, ids=["mha", "gqa_ragged_bf16", "decode"])
def test_attend_dense_equals_causal_sdpa(w):
    Q, K, V = rand_qkv(w, 21)
    rows = np.arange(w.B * w.Hq * w.Nq)
    O, lse = oracle.attend(w, Q, K, V, None, rows, dense=True)
    pos = w.q_offset + torch.arange(w.Nq)
    mask = (torch.arange(w.N)[None, :] <= pos[:, None]).expand(w.B, w.Hq, w.Nq, w.N)
    Oref, lref = _sdpa(w, Q, K, V, mask)
    np.testing.assert_allclose(O, Oref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("w", ATT_SHAPES, ids=["mha", "gqa_ragged_bf16", "decode"])
def test_attend_block_sparse_equals_masked_sdpa(w):
    Q, K, V = rand_qkv(w, 22)
    idx = _random_valid_idx(w, 5)
    rows = np.arange(w.B * w.Hq * w.Nq)
    O, lse = oracle.attend(w, Q, K, V, idx, rows)
    Oref, lref = _sdpa(w, Q, K, V, _block_mask(w, idx))
    np.testing.assert_allclose(O, Oref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lref, atol=1e-12, rtol=0)


def test_attend_all_blocks_selected_equals_dense():
    w = W(B=1, Hq=2, Hkv=1, N=320, Nq=320, b=32, d=16, topk=10, cap=20)
    Q, K, V = rand_qkv(w, 23)
    idx = -np.ones((1, 1, 10, 10), dtype=np.int32)
    for i in range(10):
        idx[0, 0, i, :i] = np.arange(i)
    rows = np.arange(2 * 320)
    O, lse = oracle.attend(w, Q, K, V, idx, rows)
    Od, ld = oracle.attend(w, Q, K, V, None, rows, dense=True)
    np.testing.assert_allclose(O, Od, atol=1e-13)
    np.testing.assert_allclose(lse, ld, atol=1e-13)


def test_attend_no_blocks_is_local_causal_attention():
    w = W(B=1, Hq=1, Hkv=1, N=256, Nq=256, b=32, d=16, topk=4, cap=8)
    Q, K, V = rand_qkv(w, 24)
    idx = -np.ones((1, 1, 8, 4), dtype=np.int32)
    O, lse = oracle.attend(w, Q, K, V, idx, np.arange(256))
    t = torch.arange(256)
    mask = ((t[None, :] <= t[:, None]) & (t[None, :] // 32 == t[:, None] // 32)).expand(1, 1, 256, 256)
    Oref, lref = _sdpa(w, Q, K, V, mask)
    np.testing.assert_allclose(O, Oref, atol=1e-12)
    np.testing.assert_allclose(lse, lref, atol=1e-12)


def test_attend_ignores_future_keys_and_values():
    w = W(B=1, Hq=2, Hkv=1, N=256, Nq=256, b=32, d=16, topk=3, cap=6)
    Q, K, V = rand_qkv(w, 25)
    idx = _random_valid_idx(w, 6)
    p = 150
    rows = np.array([p, 256 + p])
    O, lse = oracle.attend(w, Q, K, V, idx, rows)
    K2, V2 = K.clone(), V.clone()
    K2[:, :, p + 1:] = 7.0
    V2[:, :, p + 1:] = -3.0
    O2, lse2 = oracle.attend(w, Q, K2, V2, idx, rows)
    assert np.array_equal(O, O2) and np.array_equal(lse, lse2)


def test_attend_rejects_non_causal_or_repeated_blocks():
    w = W(B=1, Hq=1, Hkv=1, N=128, Nq=128, b=32, d=8, topk=2, cap=4)
    Q, K, V = rand_qkv(w, 26)
    idx = -np.ones((1, 1, 4, 2), dtype=np.int32)
    idx[0, 0, 2] = [0, 2]
    with pytest.raises(ValueError):
        oracle.attend(w, Q, K, V, idx, np.array([70]))
    idx[0, 0, 2] = [1, 1]
    with pytest.raises(ValueError):
        oracle.attend(w, Q, K, V, idx, np.array([70]))


def _recall(w):
    Q, K, V, owner = synth.generate(w)
    idx, _, _ = oracle.select_all(w, Q, K)
    own = owner.numpy().reshape(w.B * w.Hkv, -1)
    first = w.q_offset // w.b
    hit = tot = 0
    for u in range(own.shape[0]):
        for j in np.nonzero(own[u] >= 0)[0]:
            i = own[u, j]
            if 0 <= i - first < idx.shape[1]:
                tot += 1
                hit += int(j in idx[u, i - first])
    return hit, tot


@pytest.mark.parametrize("name,expect", [("mha_bf16_32k", (6411, 6588)), ("gqa_bf16_64k", (9036, 14591))])
def test_needle_recall_is_frozen_at_full_size(name, expect):
    """Regression pins: the oracle's needle recall on the full workloads, as measured on this generator
    (a property of the method and the data, not a target)."""
    assert _recall(synth.BY_NAME[name]) == expect
