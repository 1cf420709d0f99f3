"""bsa_backward_noalloc: the backward pass for callers that cannot allocate device memory.

Plugins whose host framework owns all device memory, and serving or real-time
loops that must not call cudaMalloc (it can synchronise the device), cannot hand
bsa_backward its per-row workspace. The no-allocation entry point keeps that
workspace in a fixed array inside the library. Here it is called through the C
ABI several times in a row, on different shapes and fresh inputs with nothing
cleared in between, and each result is compared with bsa_backward's on the same
inputs, within the backward tests' tolerance (fp32: max-abs <= 1e-4 * max(1,
max |ref|); bf16: relative L2 <= 2e-2 and max-abs <= 3e-2 * max |ref|). The
tensor-core path (bf16, d = 128) and the CUDA-core path (fp32) are both covered.
Host-side refusals (a malformed shape, a shape beyond the array's limit) need no
GPU and run in the CPU suite.

This file is collected last on purpose; it passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from synth import BF16, F32

W0 = synth.WORKLOADS[0]
GQA = W0.scaled(name="noalloc_bf16_gqa", B=1, Hq=4, Hkv=2, N=2048 + 40, Nq=2048 + 40, d=128, b=64, topk=4, cap=8,
                dtype=BF16, seed=51)
F32_CASE = W0.scaled(name="noalloc_f32", B=1, Hq=2, Hkv=2, N=1000, Nq=1000, d=64, b=64, topk=4, cap=8, dtype=F32,
                     seed=52)
# calls in this order, with nothing cleared in between: a stale workspace from one call would
# show up as a wrong gradient in the next, whose rows and values differ
SEQUENCE = [GQA, F32_CASE, GQA.scaled(seed=53), F32_CASE.scaled(seed=54, N=777, Nq=777)]


def _close(dtype, got, ref, what):
    got = got.float().cpu().double().numpy()
    ref = ref.float().cpu().double().numpy()
    err = np.abs(got - ref)
    if dtype == F32:
        bound = 1e-4 * max(1.0, float(np.abs(ref).max()))
        assert err.max() <= bound, f"{what}: max-abs {err.max():.3e} > {bound:.3e}"
    else:
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert rel <= 2e-2, f"{what}: rel-L2 {rel:.3e}"
        assert err.max() <= 3e-2 * float(np.abs(ref).max()), f"{what}: max-abs {err.max():.3e}"


@pytest.mark.gpu
def test_noalloc_backward_matches_bsa_backward_on_calls_in_a_row():
    import hierarchical_block_sparse_pyr_b200 as P

    lib = P._L()
    stream = torch.cuda.current_stream().cuda_stream
    for call, w in enumerate(SEQUENCE, start=1):
        s = P.shape_of(w)
        Q, K, V, _ = synth.generate(w)
        dO = synth.grad_output(w)
        Q, K, V, dO = (t.cuda() for t in (Q, K, V, dO))
        fwd = P.Buffers(s)
        P.run(s, Q, K, V, fwd)
        ref = P.BackwardBuffers(s)
        P.run_backward(s, Q, K, V, dO, fwd, ref)
        torch.cuda.synchronize()
        assert int(fwd.status.item()) == 0

        dQ, dK, dV = (torch.full_like(t, float("nan")) for t in (ref.dQ, ref.dK, ref.dV))
        rc = lib.bsa_backward_noalloc(ctypes.byref(s), Q.data_ptr(), K.data_ptr(), V.data_ptr(), fwd.O.data_ptr(),
                                      fwd.lse.data_ptr(), dO.data_ptr(), fwd.idx.data_ptr(), ref.offset.data_ptr(),
                                      ref.rho.data_ptr(), dQ.data_ptr(), dK.data_ptr(), dV.data_ptr(),
                                      fwd.status.data_ptr(), stream)
        assert rc == P.PYR_OK, P.strerror(rc)
        torch.cuda.synchronize()
        assert int(fwd.status.item()) == 0
        for got, want, name in ((dQ, ref.dQ, "dQ"), (dK, ref.dK, "dK"), (dV, ref.dV, "dV")):
            _close(w.dtype, got, want, f"call {call} ({w.name}, seed {w.seed}) {name}")


def test_noalloc_refuses_shapes_beyond_its_workspace():
    """Host validation only: returns before any CUDA call, so it runs without a GPU."""
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(GQA)
    s.B, s.Hq, s.Hkv, s.N, s.Nq = 1, 128, 64, 65536, 65536  # 8,388,608 query rows > 4,194,304
    rc = P._L().bsa_backward_noalloc(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == P.PYR_EUNSUPPORTED


def test_noalloc_reports_a_malformed_shape_as_invalid():
    """Negative B and Hq multiply to a positive row count; the shape check comes first."""
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(GQA)
    s.B, s.Hq = -1, -4
    rc = P._L().bsa_backward_noalloc(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == P.PYR_EINVAL
