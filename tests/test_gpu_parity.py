"""CUDA path vs the CPU oracle on small shapes that span several tiles and ragged tails.

Every case runs the three C-ABI calls on the GPU and compares, element by
element, with the oracle on the same seeded inputs: the pyramid, the selected
indices (bit-exact outside the gap exemption), attention given the oracle's
indices, attention given the GPU's own indices, and dense causal attention.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _parity import check_out, check_pyramid, check_traces, check_valid_idx, fmt, run_gpu
from synth import BF16, F32

pytestmark = pytest.mark.gpu

W0 = synth.WORKLOADS[0]
CASES = [
    W0,  # the tiny fp32 workload at full size
    W0.scaled(name="mha_bf16_ragged", B=1, Hq=4, Hkv=4, N=2000, Nq=2000, d=128, b=64, topk=4, cap=8, dtype=BF16,
              seed=11),
    W0.scaled(name="gqa_bf16_ragged", B=2, Hq=8, Hkv=2, N=3000, Nq=3000, d=128, b=64, topk=6, cap=12, dtype=BF16,
              seed=12, n_needle=3),
    W0.scaled(name="mha_bf16_b128", B=1, Hq=2, Hkv=2, N=4096 + 77, Nq=4096 + 77, d=128, b=128, topk=4, cap=8,
              dtype=BF16, seed=13, needle_mode=synth.NEEDLE_LOGUNIFORM),
    W0.scaled(name="decode_gqa_ragged", B=3, Hq=8, Hkv=2, N=5000, Nq=1, q_offset=4999, d=128, b=64, topk=8, cap=16,
              dtype=BF16, seed=14, n_needle=4, needle_mode=synth.NEEDLE_DECODE),
    W0.scaled(name="f32_d128_b32", B=1, Hq=2, Hkv=2, N=1000, Nq=1000, d=128, b=32, topk=5, cap=10, dtype=F32, seed=15),
    W0.scaled(name="bf16_d64_b16", B=1, Hq=2, Hkv=1, N=777, Nq=777, d=64, b=16, topk=3, cap=6, dtype=BF16, seed=16),
    W0.scaled(name="topk_eq_cap", B=1, Hq=2, Hkv=2, N=2048, Nq=2048, d=64, b=64, topk=8, cap=8, dtype=BF16, seed=17),
    W0.scaled(name="single_partial_block", B=2, Hq=2, Hkv=2, N=50, Nq=50, d=64, b=64, topk=2, cap=4, dtype=F32,
              seed=18),
    W0.scaled(name="decode_first_block", B=2, Hq=4, Hkv=1, N=40, Nq=1, q_offset=39, d=128, b=64, topk=2, cap=4,
              dtype=BF16, seed=19, n_needle=0),
    W0.scaled(name="chunked_prefill", B=1, Hq=4, Hkv=2, N=2048, Nq=1024, q_offset=1024, d=128, b=64, topk=4, cap=8,
              dtype=BF16, seed=20),
    # MHA chunked prefill: 64-row query blocks paired from block 16 on, an odd count (the last CTA has one)
    W0.scaled(name="chunked_prefill_mha", B=1, Hq=3, Hkv=3, N=2100, Nq=1076, q_offset=1024, d=128, b=64, topk=5,
              cap=10, dtype=BF16, seed=33),
    W0.scaled(name="mha_bf16_odd_qblocks", B=1, Hq=2, Hkv=2, N=2100, Nq=2100, d=128, b=64, topk=5, cap=10,
              dtype=BF16, seed=25),
    W0.scaled(name="gqa2_bf16_b128", B=1, Hq=4, Hkv=2, N=3000, Nq=3000, d=128, b=128, topk=4, cap=8, dtype=BF16,
              seed=26, needle_mode=synth.NEEDLE_LOGUNIFORM),
    W0.scaled(name="decode_mha_b128", B=2, Hq=2, Hkv=2, N=9000, Nq=1, q_offset=8999, d=128, b=128, topk=6, cap=12,
              dtype=BF16, seed=28, n_needle=3, needle_mode=synth.NEEDLE_DECODE),
    W0.scaled(name="decode_gqa8", B=2, Hq=16, Hkv=2, N=4096, Nq=1, q_offset=4095, d=128, b=64, topk=20, cap=40,
              dtype=BF16, seed=29, n_needle=4, needle_mode=synth.NEEDLE_DECODE),
    W0.scaled(name="cap_covers_all", B=1, Hq=2, Hkv=2, N=1024, Nq=1024, d=64, b=64, topk=4, cap=16, dtype=F32,
              seed=21),
    # tensor-core selection layouts: candidates stacked in M=128 rows (32 < cap <= 64), and separate
    # hi / lo operands (cap > 64)
    W0.scaled(name="cap48_stacked_m128", B=1, Hq=2, Hkv=2, N=8192 + 30, Nq=8192 + 30, d=128, b=64, topk=20, cap=48,
              dtype=BF16, seed=31, n_needle=6),
    W0.scaled(name="cap100_separate", B=1, Hq=4, Hkv=2, N=16384, Nq=16384, d=128, b=64, topk=40, cap=100,
              dtype=BF16, seed=32, n_needle=6),
    # long route lists for the paired-block MHA attention (up to 101 entries per query block) and the
    # separate hi / lo selection layout
    W0.scaled(name="mha_topk100", B=1, Hq=2, Hkv=2, N=12288 + 40, Nq=12288 + 40, d=128, b=64, topk=100, cap=128,
              dtype=BF16, seed=34, n_needle=6),
]


def _rows_all(w):
    return np.arange(w.B * w.Hq * w.Nq)


def _rows_sample(w, n=600, seed=0):
    rng = np.random.default_rng(seed)
    total = w.B * w.Hq * w.Nq
    if total <= n:
        return np.arange(total)
    return np.unique(np.concatenate([rng.choice(total, n, replace=False), [0, total - 1]]))


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_parity_small(w):
    Q, K, V, _ = synth.generate(w)
    units = list(range(w.B * w.Hkv))
    g = run_gpu(w, Q, K, V, with_trace=True)
    assert g["status"] == 0

    pyr_o = oracle.pyramid(w, K, units)
    check_pyramid(g["pyr"].double().numpy().reshape(pyr_o.shape), pyr_o)

    nqb = oracle.num_qblocks(w)
    items = [(u, q) for u in units for q in range(nqb)]
    idx_o, gap_o, _, trace_o = oracle.select(w, Q, pyr_o, units, items, with_trace=True)
    counts = check_traces(w, Q, pyr_o, units, items, g["idx"].numpy(), g["trace"].numpy(), idx_o, gap_o, trace_o)
    check_valid_idx(w, g["idx"].numpy())
    gap_g = g["gap"].double().numpy().reshape(-1)
    fin = np.isfinite(gap_o)
    assert (np.isfinite(gap_g) == fin).all()
    np.testing.assert_allclose(gap_g[fin], gap_o[fin], atol=1e-3, rtol=1e-3)
    print(f"\n{fmt(w)} select: {counts['checked']} rows bit-exact with their trace, {counts['exempt']} exempt "
          f"({counts['differing']} differ, {counts['validated']} validated level by level, 0 undecided)")
    idx_o = idx_o.reshape(len(units), nqb, w.topk)

    rows = _rows_all(w) if w.B * w.Hq * w.Nq <= 16384 else _rows_sample(w)
    # attention given the oracle's idx
    g2 = run_gpu(w, Q, K, V, idx=idx_o.reshape(g["idx"].shape))
    O_o, lse_o = oracle.attend(w, Q, K, V, idx_o.reshape(g["idx"].shape), rows)
    O_g = g2["O"].double().numpy().reshape(-1, w.d)[rows]
    lse_g = g2["lse"].double().numpy().reshape(-1)[rows]
    e, r = check_out(w, O_g, lse_g, O_o, lse_o)
    print(f"  attention (oracle idx): max-abs {e:.2e} rel-L2 {r:.2e}")
    # end to end: the GPU's own idx
    O_o2, lse_o2 = oracle.attend(w, Q, K, V, g["idx"].numpy(), rows)
    check_out(w, g["O"].double().numpy().reshape(-1, w.d)[rows], g["lse"].double().numpy().reshape(-1)[rows],
              O_o2, lse_o2)


@pytest.mark.parametrize("w", [CASES[0], CASES[1], CASES[2], CASES[4], CASES[8], CASES[13], CASES[14]],
                         ids=lambda w: w.name)
def test_dense_parity(w):
    Q, K, V, _ = synth.generate(w)
    g = run_gpu(w, Q, K, V, dense=True)
    assert g["status"] == 0
    rows = _rows_sample(w, 300, seed=1)
    O_o, lse_o = oracle.attend(w, Q, K, V, None, rows, dense=True)
    check_out(w, g["O"].double().numpy().reshape(-1, w.d)[rows], g["lse"].double().numpy().reshape(-1)[rows],
              O_o, lse_o)


@pytest.mark.parametrize("case", [
    dict(w=W0.scaled(name="upd_decode", B=2, Hq=4, Hkv=2, N=8192, Nq=8192, d=128, b=64, topk=4, cap=8, dtype=BF16,
                     seed=30), from_pos=8191),
    dict(w=W0.scaled(name="upd_ragged_f32", B=1, Hq=2, Hkv=2, N=3000, Nq=3000, d=64, b=32, topk=4, cap=8, dtype=F32,
                     seed=31), from_pos=2500),
    dict(w=W0.scaled(name="upd_rebuild", B=1, Hq=2, Hkv=2, N=8192, Nq=8192, d=128, b=64, topk=4, cap=8,
                     dtype=BF16, seed=32), from_pos=100),
], ids=lambda c: c["w"].name)
def test_pyr_update_matches_a_rebuild_and_the_oracle(case):
    """Rewrite the keys at positions >= from_pos, update the pyramid in place, compare."""
    import hierarchical_block_sparse_pyr_b200 as P
    w, from_pos = case["w"], case["from_pos"]
    Q, K, V, _ = synth.generate(w)
    s = P.shape_of(w)
    Kd = K.cuda()
    buf = P.Buffers(s)
    P.pyr_build(s, Kd, buf.pyr, buf.status)
    K2 = K.clone()
    K2[:, :, from_pos:] = synth.normal(77, 14, K2[:, :, from_pos:].shape, K.dtype) * 2
    Kd.copy_(K2)
    P.pyr_update(s, Kd, buf.pyr, from_pos, buf.status)
    fresh = P.Buffers(s)
    P.pyr_build(s, Kd, fresh.pyr, fresh.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    upd = P.pyramid_means(s, buf.pyr).cpu().double().numpy()
    reb = P.pyramid_means(s, fresh.pyr).cpu().double().numpy()
    pyr_o = oracle.pyramid(w, K2, list(range(w.B * w.Hkv)))
    check_pyramid(upd.reshape(pyr_o.shape), pyr_o)
    assert np.abs(upd - reb).max() <= 2e-5 * (1 + np.abs(reb).max())


def test_all_blocks_selected_equals_dense_on_gpu():
    w = W0.scaled(name="all_blocks", B=1, Hq=2, Hkv=1, N=1024, Nq=1024, d=128, b=64, topk=16, cap=32, dtype=BF16,
                  seed=22)
    Q, K, V, _ = synth.generate(w)
    nqb = 16
    idx = -np.ones((1, 1, nqb, 16), dtype=np.int32)
    for i in range(nqb):
        idx[0, 0, i, :i] = np.arange(i)
    a = run_gpu(w, Q, K, V, idx=idx)
    b = run_gpu(w, Q, K, V, dense=True)
    assert (a["O"] - b["O"]).abs().max().item() <= 2e-2
    assert (a["lse"] - b["lse"]).abs().max().item() <= 2e-3


def test_bad_idx_is_reported_and_skipped():
    w = W0.scaled(name="bad_idx", B=1, Hq=1, Hkv=1, N=512, Nq=512, d=64, b=64, topk=2, cap=4, dtype=F32, seed=23)
    Q, K, V, _ = synth.generate(w)
    idx = -np.ones((1, 1, 8, 2), dtype=np.int32)
    idx[0, 0, 5] = [1, 6]  # 6 is not before block 5
    g = run_gpu(w, Q, K, V, idx=idx)
    assert g["status"] == 5
    ok = idx.copy()
    ok[0, 0, 5] = [1, -1]
    O_o, _ = oracle.attend(w, Q, K, V, ok, np.arange(512))
    assert np.abs(g["O"].double().numpy().reshape(-1, 64) - O_o).max() <= 1e-4


def test_bad_idx_is_reported_and_skipped_on_the_tensor_core_path():
    w = W0.scaled(name="bad_idx_tc", B=1, Hq=2, Hkv=1, N=640, Nq=640, d=128, b=64, topk=3, cap=6, dtype=BF16,
                  seed=27)
    Q, K, V, _ = synth.generate(w)
    idx = -np.ones((1, 1, 10, 3), dtype=np.int32)
    idx[0, 0, 6] = [4, 2, 5]  # 2 breaks the ascending order
    idx[0, 0, 7] = [1, 7, -1]  # 7 is the diagonal block, not an earlier one
    g = run_gpu(w, Q, K, V, idx=idx)
    assert g["status"] == 5
    ok = idx.copy()
    ok[0, 0, 6] = [4, 5, -1]
    ok[0, 0, 7] = [1, -1, -1]
    O_o, lse_o = oracle.attend(w, Q, K, V, ok, np.arange(2 * 640))
    check_out(w, g["O"].double().numpy().reshape(-1, 128), g["lse"].double().numpy().reshape(-1), O_o, lse_o)


def test_future_keys_do_not_change_selection_or_output():
    w = W0.scaled(name="causal", B=1, Hq=2, Hkv=2, N=2048, Nq=2048, d=128, b=64, topk=4, cap=8, dtype=BF16, seed=24)
    Q, K, V, _ = synth.generate(w)
    a = run_gpu(w, Q, K, V)
    K2, V2 = K.clone(), V.clone()
    cut = 20 * 64
    K2[:, :, cut:] = (K2[:, :, cut:].float() * -3 + 1).to(K.dtype)
    V2[:, :, cut:] = (V2[:, :, cut:].float() * 5).to(V.dtype)
    b = run_gpu(w, Q, K2, V2)
    assert torch.equal(a["idx"][:, :, :20], b["idx"][:, :, :20])
    assert torch.equal(a["O"][:, :, :cut], b["O"][:, :, :cut])
    assert torch.equal(a["lse"][:, :, :cut], b["lse"][:, :, :cut])
