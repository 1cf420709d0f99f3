"""The seeded generator: determinism, rounding, distribution and planted structure."""
import numpy as np
import torch

import synth


def test_draws_are_deterministic_and_seed_dependent():
    a = synth.normal(5, 1, (4096,))
    b = synth.normal(5, 1, (4096,))
    c = synth.normal(6, 1, (4096,))
    d = synth.normal(5, 2, (4096,))
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)


def test_normals_have_unit_moments():
    x = synth.normal(1, 0, (1 << 20,)).double()
    assert abs(x.mean().item()) < 5e-3
    assert abs(x.std().item() - 1.0) < 5e-3
    # Box-Muller pairs are independent: no lag-1 correlation
    assert abs(torch.corrcoef(torch.stack([x[0::2], x[1::2]]))[0, 1].item()) < 5e-3


def test_bf16_storage_is_round_to_nearest_even_of_the_fp32_draw():
    f = synth.normal(3, 7, (1 << 16,), torch.float32)
    h = synth.normal(3, 7, (1 << 16,), torch.bfloat16)
    assert torch.equal(f.to(torch.bfloat16), h)


def test_workload_shapes_and_needles():
    w = synth.WORKLOADS[0]
    Q, K, V, owner = synth.generate(w)
    assert Q.shape == (1, 2, 4096, 64) and K.shape == (1, 2, 4096, 64) and Q.dtype == torch.float32
    own = owner.numpy()
    assert ((own == -1) | (own > np.arange(w.nb)[None, None, :])).all()  # the owner comes after its needle
    Qd, Kd = Q.double().numpy(), K.double().numpy()
    # an owned needle block holds 2 * mean(query rows of its owner) + N(0, 0.1^2)
    for hk in range(2):
        for j in np.nonzero(own[0, hk] > 0)[0][:10]:
            i = own[0, hk, j]
            target = 2.0 * Qd[0, hk, i * 64:(i + 1) * 64].mean(axis=0)
            resid = Kd[0, hk, j * 64:(j + 1) * 64] - target[None, :]
            assert abs(resid.std() - 0.1) < 0.01


def test_gqa_needles_use_all_heads_of_the_group():
    w = synth.WORKLOADS[2].scaled(B=1, N=4096, Nq=4096, seed=9)
    Q, K, V, owner = synth.generate(w)
    Qd, Kd, own = Q.float().double().numpy(), K.float().double().numpy(), owner.numpy()
    G = w.G
    j = int(np.nonzero(own[0, 1] > 0)[0][0])
    i = own[0, 1, j]
    target = 2.0 * Qd[0, G:2 * G, i * 64:(i + 1) * 64].reshape(-1, w.d).mean(axis=0)
    resid = Kd[0, 1, j * 64:(j + 1) * 64] - target[None, :]
    assert resid.std() < 0.12


def test_decode_workload_plants_needles_for_the_single_query():
    w = synth.WORKLOADS[3].scaled(B=2, N=8192, q_offset=8191, seed=4)
    Q, K, V, owner = synth.generate(w)
    own = owner.numpy()
    assert Q.shape == (2, 32, 1, 128)
    last = w.nb - 1
    for bi in range(2):
        for hk in range(w.Hkv):
            planted = np.nonzero(own[bi, hk] >= 0)[0]
            assert len(planted) == w.n_needle and (own[bi, hk, planted] == last).all()
