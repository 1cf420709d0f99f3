"""The C ABI: the library loads, exports every declared symbol, validates on the host.

Nothing here launches a kernel: every call below returns from host-side
validation before the CUDA runtime is touched, so it runs without a GPU.
"""
import ctypes
import os
import re

import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"PYR_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    import hierarchical_block_sparse_pyr_b200 as P

    declared = _declared()
    assert {"pyr_build", "pyr_select", "bsa_forward", "dense_forward", "pyr_strerror"} <= declared
    lib = ctypes.CDLL(P.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert set(P.ABI_SYMBOLS) <= declared


def test_geometry_matches_the_oracle():
    import hierarchical_block_sparse_pyr_b200 as P

    for w in synth.WORKLOADS + [synth.WORKLOADS[0].scaled(N=4000, Nq=4000), synth.WORKLOADS[1].scaled(N=100, Nq=1,
                                                                                                       q_offset=99)]:
        s = P.shape_of(w)
        assert P.num_levels(s) == oracle.num_levels(w)
        assert P.num_nodes(s) == oracle.num_nodes(w)
        assert P.num_qblocks(s) == oracle.num_qblocks(w)
        assert P.pyramid_elems(s) == w.B * w.Hkv * oracle.num_nodes(w) * 2 * w.d
    bad = P.shape_of(synth.WORKLOADS[0])
    bad.cap = 7
    assert P.pyramid_elems(bad) == 0


@pytest.mark.parametrize("field,value,code", [
    ("Hq", 3, 1),          # Hq % Hkv != 0 with Hkv = 2
    ("N", 0, 1),
    ("topk", 0, 1),
    ("cap", 7, 1),         # odd cap
    ("topk", 40, 1),       # topk > cap
    ("d", 96, 2),
    ("b", 48, 2),
    ("dtype", 5, 2),
    ("q_offset", 10, 2),   # a prefill chunk that does not start on a block boundary
])
def test_host_validation_rejects_bad_shapes(field, value, code):
    import hierarchical_block_sparse_pyr_b200 as P

    w = synth.WORKLOADS[0]
    s = P.shape_of(w)
    s.Hkv = 2
    s.Nq = 1024
    setattr(s, field, value)
    lib = P._L()
    rc = lib.pyr_build(ctypes.byref(s), 16, 16, None, None)
    assert rc == code, P.strerror(rc)
    rc = lib.pyr_select(ctypes.byref(s), 16, 16, 16, None, None, None)
    assert rc == code


def test_host_validation_rejects_null_and_misaligned_pointers():
    import hierarchical_block_sparse_pyr_b200 as P

    s = P.shape_of(synth.WORKLOADS[1])
    lib = P._L()
    assert lib.pyr_build(ctypes.byref(s), None, 16, None, None) == P.PYR_EINVAL
    assert lib.pyr_build(ctypes.byref(s), 24, 16, None, None) == P.PYR_EINVAL
    assert lib.pyr_select(ctypes.byref(s), 16, 16, None, None, None, None) == P.PYR_EINVAL
    assert lib.bsa_forward(ctypes.byref(s), 16, 16, 16, None, 16, None, None, None) == P.PYR_EINVAL
    assert lib.dense_forward(ctypes.byref(s), 16, 16, 16, 8, None, None, None) == P.PYR_EINVAL
    assert lib.pyr_build(None, 16, 16, None, None) == P.PYR_EINVAL
    assert lib.pyr_means(ctypes.byref(s), None, 16, None, None) == P.PYR_EINVAL  # no pyramid
    assert lib.pyr_means(ctypes.byref(s), 16, 18, None, None) == P.PYR_EINVAL    # means not 4-byte aligned
    for code in range(6):
        assert isinstance(P.strerror(code), str) and P.strerror(code)


def test_python_binding_refuses_cpu_tensors():
    import torch

    import hierarchical_block_sparse_pyr_b200 as P

    w = synth.WORKLOADS[0].scaled(N=256, Nq=256)
    s = P.shape_of(w)
    K = torch.zeros((1, 2, 256, 64))
    with pytest.raises(TypeError):
        P.pyr_build(s, K, torch.zeros((1, 2, P.num_nodes(s), 64)))


def test_backward_entry_points_validate_on_the_host():
    import hierarchical_block_sparse_pyr_b200 as P

    lib = P._L()
    s = P.shape_of(synth.WORKLOADS[0].scaled(N=1024, Nq=1024))
    ok = [16] * 13
    # route inversion: idx must be 16-byte aligned, offset and rho 4-byte aligned, none null
    assert lib.bsa_route_invert(ctypes.byref(s), None, 16, 16, None, None) == P.PYR_EINVAL
    assert lib.bsa_route_invert(ctypes.byref(s), 24, 16, 16, None, None) == P.PYR_EINVAL
    assert lib.bsa_route_invert(ctypes.byref(s), 16, 18, 16, None, None) == P.PYR_EINVAL
    assert lib.bsa_route_invert(ctypes.byref(s), 16, 16, None, None, None) == P.PYR_EINVAL
    assert lib.bsa_route_invert(None, 16, 16, 16, None, None) == P.PYR_EINVAL
    # backward: every operand present; tensors 16-byte aligned, lse/delta/offset/rho 4-byte aligned
    for k in range(13):
        args = list(ok)
        args[k] = None
        assert lib.bsa_backward(ctypes.byref(s), *args, None, None) == P.PYR_EINVAL, k
    for k in range(13):
        args = list(ok)
        args[k] = 16 + 2  # misaligned for every operand
        assert lib.bsa_backward(ctypes.byref(s), *args, None, None) == P.PYR_EINVAL, k
    # shape errors come first, as in the forward entry points
    bad = P.shape_of(synth.WORKLOADS[0].scaled(N=1024, Nq=1024))
    bad.cap = 7
    assert lib.bsa_backward(ctypes.byref(bad), *ok, None, None) == P.PYR_EINVAL
    # the backward pass covers whole sequences only: a chunk or a decode step is refused
    chunk = P.shape_of(synth.WORKLOADS[0].scaled(N=1024, Nq=512, q_offset=512))
    assert lib.bsa_backward(ctypes.byref(chunk), *ok, None, None) == P.PYR_EUNSUPPORTED
    dec = P.shape_of(synth.WORKLOADS[1].scaled(N=100, Nq=1, q_offset=99))
    assert lib.bsa_backward(ctypes.byref(dec), *ok, None, None) == P.PYR_EUNSUPPORTED


def _ws_expected(w, upc, with_lse):
    """Workspace of bsa_forward_host: two slots of one chunk's Q, K, V, O (and lse), one pyramid, one idx."""
    r = lambda x: -(-x // 256) * 256  # noqa: E731
    elt = 4 if w.dtype == synth.F32 else 2
    q = r(upc * w.G * w.Nq * w.d * elt)
    kv = r(upc * w.N * w.d * elt)
    lse = r(upc * w.G * w.Nq * 4) if with_lse else 0
    pyr = r(upc * oracle.num_nodes(w) * 2 * w.d * 2)
    idx = r(upc * oracle.num_qblocks(w) * w.topk * 4)
    return 2 * (2 * q + 2 * kv + lse) + pyr + idx


def test_host_entry_point_workspace_size():
    import hierarchical_block_sparse_pyr_b200 as P

    w = synth.WORKLOADS[1]
    s = P.shape_of(w)
    U = w.B * w.Hkv
    for upc, with_lse in ((1, False), (1, True), (3, True), (U, False)):
        assert P.host_workspace_bytes(s, upc, with_lse) == _ws_expected(w, upc, with_lse), (upc, with_lse)
    # 0 shrinks the chunks towards the end of the call; the largest, which sizes the slots, is a quarter
    # of the units with at most 96 MiB of inputs (Q, K, V) per chunk: 4 of the 32K workload's 16 units
    in_unit = (w.G * w.Nq + 2 * w.N) * w.d * 2
    cap = max(1, min(U // 4, (96 << 20) // in_unit))
    assert cap == 4
    assert P.host_workspace_bytes(s, 0) == _ws_expected(w, cap, False)
    # more units per chunk than there are units means one chunk
    assert P.host_workspace_bytes(s, 10 * U) == _ws_expected(w, U, False)
    assert P.host_workspace_bytes(s, -1) == 0
    bad = P.shape_of(w)
    bad.cap = 7
    assert P.host_workspace_bytes(bad, 1) == 0


def test_host_entry_point_validates_on_the_host():
    import hierarchical_block_sparse_pyr_b200 as P

    lib = P._L()
    w = synth.WORKLOADS[1]
    s = P.shape_of(w)
    need = P.host_workspace_bytes(s, 1, False)
    call = lambda sh, q=16, k=16, v=16, o=16, upc=1, ws=256, nbytes=need: lib.bsa_forward_host(  # noqa: E731
        ctypes.byref(sh) if sh is not None else None, q, k, v, o, None, upc, ws, nbytes, None, None)
    assert call(None) == P.PYR_EINVAL
    for kw in ({"q": None}, {"k": None}, {"v": None}, {"o": None}, {"ws": None}, {"ws": 264}, {"upc": -1},
               {"nbytes": need - 1}):
        assert call(s, **kw) == P.PYR_EINVAL, kw
    # shape errors are those of the device entry points
    for field, value in (("cap", 7), ("d", 96), ("q_offset", 10)):
        bad = P.shape_of(w)
        setattr(bad, field, value)
        assert call(bad) == lib.pyr_build(ctypes.byref(bad), 16, 16, None, None), field
    with pytest.raises(TypeError):
        import torch
        P.bsa_forward_host(s, torch.zeros(4), torch.zeros(4), torch.zeros(4), torch.zeros(4),
                           workspace=torch.zeros(16, dtype=torch.uint8))


def test_device_memory_grows_linearly_with_the_context():
    """The score matrix is never formed (PISA abstract): every buffer the path needs, and the host-buffer
    workspace, grow in proportion to N, never with N^2."""
    import hierarchical_block_sparse_pyr_b200 as P

    base = synth.WORKLOADS[1]
    sizes = []
    for N in (32768, 65536, 131072, 262144, 1 << 20):
        w = base.scaled(N=N, Nq=N)
        s = P.shape_of(w)
        nqb = P.num_qblocks(s)
        tensors = 4 * w.B * w.Hq * N * w.d * 2                    # Q, K, V, O (bf16, MHA)
        routes = w.B * w.Hkv * nqb * (w.topk + 1) * 4 + w.B * w.Hq * N * 4  # idx, gap, lse
        total = tensors + routes + P.pyramid_elems(s) * 2
        sizes.append((N, total, P.host_workspace_bytes(s, 0, True)))
    for (n0, t0, h0), (n1, t1, h1) in zip(sizes, sizes[1:]):
        assert t1 / t0 <= 1.01 * n1 / n0 and h1 / h0 <= 1.01 * n1 / n0, (n0, n1)
