"""bsa_forward_host: the forward path from host buffers, streamed through the device by chunks of units.

Each (batch, kv head) unit is computed by the same kernels whatever else shares
its launch, so the host entry point must give bit-identical O and lse to
pyr_build + pyr_select + bsa_forward over the whole batch on device buffers
(which the parity tests compare with the oracle). Covered: one unit per
chunk, a ragged last chunk, one chunk for everything, the automatic size,
pinned and pageable host memory, the CUDA-core (fp32), tensor-core (bf16)
and decode kernels, a chunked prefill, and two calls in a row that reuse one
workspace on one stream.
"""
import pytest
import torch

import synth
from synth import BF16, F32

pytestmark = pytest.mark.gpu

W0 = synth.WORKLOADS[0]
CASES = [
    W0.scaled(name="host_gqa_bf16_ragged", B=2, Hq=8, Hkv=2, N=3000, Nq=3000, d=128, b=64, topk=6, cap=12, dtype=BF16,
              seed=71),
    W0.scaled(name="host_mha_bf16_b128", B=1, Hq=3, Hkv=3, N=4096 + 77, Nq=4096 + 77, d=128, b=128, topk=4, cap=8,
              dtype=BF16, seed=72),
    W0.scaled(name="host_f32_d64", B=1, Hq=4, Hkv=4, N=1000, Nq=1000, d=64, b=64, topk=4, cap=8, dtype=F32, seed=73),
    W0.scaled(name="host_decode", B=3, Hq=8, Hkv=2, N=5000, Nq=1, q_offset=4999, d=128, b=64, topk=8, cap=16,
              dtype=BF16, seed=74, needle_mode=synth.NEEDLE_DECODE),
    W0.scaled(name="host_chunked_prefill", B=1, Hq=4, Hkv=2, N=2048, Nq=1024, q_offset=1024, d=128, b=64, topk=4,
              cap=8, dtype=BF16, seed=75),
]


def _device_reference(P, s, Q, K, V):
    buf = P.Buffers(s)
    P.run(s, Q.cuda(), K.cuda(), V.cuda(), buf, with_gap=False)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    return buf.O.cpu(), buf.lse.cpu()


def _host_run(P, s, Q, K, V, upc, pinned, with_lse=True, workspace=None):
    if pinned:
        Q, K, V = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    O = torch.full((s.B, s.Hq, s.Nq, s.d), float("nan"), dtype=Q.dtype, pin_memory=pinned)
    lse = torch.full((s.B, s.Hq, s.Nq), float("nan"), dtype=torch.float32, pin_memory=pinned) if with_lse else None
    if workspace is None:
        workspace = torch.empty(P.host_workspace_bytes(s, upc, with_lse), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    P.bsa_forward_host(s, Q, K, V, O, lse, units_per_chunk=upc, workspace=workspace, status=status)
    torch.cuda.current_stream().synchronize()
    assert int(status.item()) == 0
    return O, lse


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_host_path_is_bit_identical_to_the_device_path(w):
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(w)
    Q, K, V, _ = synth.generate(w)
    O_ref, lse_ref = _device_reference(P, s, Q, K, V)
    U = w.B * w.Hkv
    sizes = sorted({1, max(1, U - 1), U, 0})
    for k, upc in enumerate(sizes):
        O, lse = _host_run(P, s, Q, K, V, upc, pinned=(k % 2 == 0))
        assert torch.equal(O, O_ref), f"{w.name}: O differs with {upc} units per chunk"
        assert torch.equal(lse, lse_ref), f"{w.name}: lse differs with {upc} units per chunk"


def test_host_path_two_calls_reuse_one_workspace():
    import hierarchical_block_sparse_pyr_b200 as P

    w1, w2 = CASES[0], CASES[0].scaled(seed=76)
    s = P.shape_of(w1)
    ws = torch.empty(P.host_workspace_bytes(s, 1, False), dtype=torch.uint8, device="cuda")
    outs = []
    for w in (w1, w2):
        Q, K, V, _ = synth.generate(w)
        Qp, Kp, Vp = Q.pin_memory(), K.pin_memory(), V.pin_memory()
        O = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=Q.dtype, pin_memory=True)
        P.bsa_forward_host(s, Qp, Kp, Vp, O, None, units_per_chunk=1, workspace=ws)  # no sync in between
        outs.append((O, Q, K, V))
    torch.cuda.current_stream().synchronize()
    for O, Q, K, V in outs:
        O_ref, _ = _device_reference(P, s, Q, K, V)
        assert torch.equal(O, O_ref)
