"""Hierarchical (pyramid) top-K key-block selection + causal block-sparse attention on B200.

Thin ctypes binding over ``lib/libpyr.so`` (the C ABI declared in
``include/pyr.h``). Functions here only marshal arguments: torch tensors give
device pointers and the current CUDA stream; every step of the computation
runs in the library's sm_100a kernels. There is no CPU fallback: the library
is loaded on first use and every call raises ImportError if it is missing;
every call needs CUDA tensors.

    pyr_build(shape, K, pyr)                  key pyramid (mean pooling)
    pyr_update(shape, K, pyr, from_pos)       refresh the nodes over rewritten key positions
    pyr_select(shape, Q, pyr, idx, gap)       coarse-to-fine LogSumExp top-K
    pyr_select_ex(shape, Q, pyr, idx, gap, opts)
                                              the same with the PHAROS variants (per-head budget,
                                              confidence fallback, cross-level guidance) and a trace
    bsa_forward(shape, Q, K, V, idx, O, lse)  causal block-sparse attention
    phba_state_build(shape, M, Ks, V, A, W, PK, PV, workspace)
                                              PHBA prefix states (gated slot recurrence, chunkwise)
    phba_forward(shape, Q, K, V, idx, O, lse, Qs, M, PK, PV)
                                              block-sparse attention over tokens and state slots
    dense_forward(shape, Q, K, V, O, lse)     dense causal attention
    bsa_route_invert(shape, idx, offset, rho) routes in block-major form (for the backward)
    bsa_backward(shape, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV)
                                              gradients of the block-sparse attention
    forward(Q, K, V, b, topk, cap)            allocate outputs and run all three
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libpyr.so")

PYR_OK, PYR_EINVAL, PYR_EUNSUPPORTED, PYR_ECUDA, PYR_ETIMEOUT, PYR_EBADIDX = range(6)
PYR_F32, PYR_BF16 = 0, 1

ABI_SYMBOLS = ("pyr_num_levels", "pyr_num_nodes", "pyr_num_qblocks", "pyr_pyramid_elems", "pyr_build", "pyr_means",
               "pyr_update",
               "pyr_select", "pyr_select_ex", "pyr_select_trace_levels", "pyr_select_trace_width", "bsa_forward",
               "dense_forward", "bsa_forward_host", "pyr_host_workspace_bytes", "bsa_route_invert", "bsa_backward",
               "bsa_backward_noalloc", "pyr_selftest_wait", "pyr_strerror", "phba_state_elems",
               "phba_state_workspace_bytes", "phba_state_build", "phba_forward")


class PyrShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "Hq", "Hkv", "N", "Nq", "q_offset", "d", "b", "topk", "cap",
                                             "dtype")]

    def __repr__(self):
        return "PyrShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class PyrSelectOpts(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_void_p), ("fcf_tau", ctypes.c_float), ("fcf_extra", ctypes.c_int),
                ("rcg_lambda", ctypes.c_float), ("trace", ctypes.c_void_p)]


class PyrError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} (status {code})")


def _load_lib():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libpyr.so is missing at {LIB_PATH}; build it with `python -m hierarchical_block_sparse_pyr_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    sp = ctypes.POINTER(PyrShape)
    vp = ctypes.c_void_p
    lib.pyr_num_levels.argtypes = [sp]
    lib.pyr_num_levels.restype = ctypes.c_int
    lib.pyr_num_nodes.argtypes = [sp]
    lib.pyr_num_nodes.restype = ctypes.c_int64
    lib.pyr_num_qblocks.argtypes = [sp]
    lib.pyr_num_qblocks.restype = ctypes.c_int64
    lib.pyr_pyramid_elems.argtypes = [sp]
    lib.pyr_pyramid_elems.restype = ctypes.c_size_t
    lib.pyr_build.argtypes = [sp, vp, vp, vp, vp]
    lib.pyr_build.restype = ctypes.c_int
    lib.pyr_means.argtypes = [sp, vp, vp, vp, vp]
    lib.pyr_means.restype = ctypes.c_int
    lib.pyr_update.argtypes = [sp, vp, vp, ctypes.c_int, vp, vp]
    lib.pyr_update.restype = ctypes.c_int
    lib.pyr_select.argtypes = [sp, vp, vp, vp, vp, vp, vp]
    lib.pyr_select.restype = ctypes.c_int
    lib.pyr_select_ex.argtypes = [sp, vp, vp, ctypes.POINTER(PyrSelectOpts), vp, vp, vp, vp]
    lib.pyr_select_ex.restype = ctypes.c_int
    lib.pyr_select_trace_levels.argtypes = [sp]
    lib.pyr_select_trace_levels.restype = ctypes.c_int
    lib.pyr_select_trace_width.argtypes = [sp]
    lib.pyr_select_trace_width.restype = ctypes.c_int
    lib.bsa_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.bsa_forward.restype = ctypes.c_int
    lib.dense_forward.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp]
    lib.dense_forward.restype = ctypes.c_int
    lib.bsa_forward_host.argtypes = [sp, vp, vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_size_t, vp, vp]
    lib.bsa_forward_host.restype = ctypes.c_int
    lib.pyr_host_workspace_bytes.argtypes = [sp, ctypes.c_int, ctypes.c_int]
    lib.pyr_host_workspace_bytes.restype = ctypes.c_size_t
    lib.bsa_route_invert.argtypes = [sp, vp, vp, vp, vp, vp]
    lib.bsa_route_invert.restype = ctypes.c_int
    lib.bsa_backward.argtypes = [sp] + [vp] * 15
    lib.bsa_backward.restype = ctypes.c_int
    lib.bsa_backward_noalloc.argtypes = [sp] + [vp] * 14
    lib.bsa_backward_noalloc.restype = ctypes.c_int
    lib.phba_state_elems.argtypes = [sp, ctypes.c_int]
    lib.phba_state_elems.restype = ctypes.c_size_t
    lib.phba_state_workspace_bytes.argtypes = [sp, ctypes.c_int]
    lib.phba_state_workspace_bytes.restype = ctypes.c_size_t
    lib.phba_state_build.argtypes = [sp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp, vp]
    lib.phba_state_build.restype = ctypes.c_int
    lib.phba_forward.argtypes = [sp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, vp]
    lib.phba_forward.restype = ctypes.c_int
    lib.pyr_selftest_wait.argtypes = [vp, vp]
    lib.pyr_selftest_wait.restype = ctypes.c_int
    lib.pyr_strerror.argtypes = [ctypes.c_int]
    lib.pyr_strerror.restype = ctypes.c_char_p
    return lib


_lib_handle = None


def _L():
    """The loaded libpyr (loaded once, on first use)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load_lib()
    return _lib_handle


def strerror(code: int) -> str:
    return _L().pyr_strerror(code).decode()


def make_shape(B, Hq, Hkv, N, Nq, q_offset, d, b, topk, cap, dtype) -> PyrShape:
    if isinstance(dtype, torch.dtype):
        dtype = {torch.float32: PYR_F32, torch.bfloat16: PYR_BF16}[dtype]
    return PyrShape(B, Hq, Hkv, N, Nq, q_offset, d, b, topk, cap, dtype)


def shape_of(w) -> PyrShape:
    """PyrShape from any object with fields B, Hq, Hkv, N, Nq, q_offset, d, b, topk, cap, dtype."""
    return make_shape(w.B, w.Hq, w.Hkv, w.N, w.Nq, w.q_offset, w.d, w.b, w.topk, w.cap, w.dtype)


def num_levels(s: PyrShape) -> int:
    return _L().pyr_num_levels(ctypes.byref(s))


def num_nodes(s: PyrShape) -> int:
    return _L().pyr_num_nodes(ctypes.byref(s))


def num_qblocks(s: PyrShape) -> int:
    return _L().pyr_num_qblocks(ctypes.byref(s))


def pyramid_elems(s: PyrShape) -> int:
    """bf16 values of the pyr buffer: B * Hkv * P * 2 * d."""
    return _L().pyr_pyramid_elems(ctypes.byref(s))


def _dev(t, name, nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _check(rc, what):
    if rc != PYR_OK:
        raise PyrError(rc, what)


def pyr_build(s: PyrShape, K, pyr, status=None, stream=None):
    _check(_L().pyr_build(ctypes.byref(s), _dev(K, "K"), _dev(pyr, "pyr"), _dev(status, "status", True),
                          _stream(stream)), "pyr_build")


def pyr_means(s: PyrShape, pyr, means, status=None, stream=None):
    """fp32 node means [B, Hkv, P, d] (means, written) from a pyramid's (hi, lo) pairs."""
    _check(_L().pyr_means(ctypes.byref(s), _dev(pyr, "pyr"), _dev(means, "means"), _dev(status, "status", True),
                          _stream(stream)), "pyr_means")


def pyr_update(s: PyrShape, K, pyr, from_pos: int, status=None, stream=None):
    _check(_L().pyr_update(ctypes.byref(s), _dev(K, "K"), _dev(pyr, "pyr"), int(from_pos), _dev(status, "status", True),
                           _stream(stream)), "pyr_update")


def pyr_select(s: PyrShape, Q, pyr, idx, gap=None, status=None, stream=None):
    _check(_L().pyr_select(ctypes.byref(s), _dev(Q, "Q"), _dev(pyr, "pyr"), _dev(idx, "idx"),
                           _dev(gap, "gap", True), _dev(status, "status", True), _stream(stream)), "pyr_select")


def select_trace_levels(s: PyrShape) -> int:
    return _L().pyr_select_trace_levels(ctypes.byref(s))


def select_trace_width(s: PyrShape) -> int:
    return _L().pyr_select_trace_width(ctypes.byref(s))


def new_trace(s: PyrShape, device="cuda"):
    """A trace buffer [B, Hkv, nqb, levels, width] int32 for pyr_select_ex."""
    return torch.empty((s.B, s.Hkv, num_qblocks(s), select_trace_levels(s), select_trace_width(s)),
                       dtype=torch.int32, device=device)


def pyr_select_ex(s: PyrShape, Q, pyr, idx, gap=None, budget=None, fcf_tau: float = 0.0, fcf_extra: int = 0,
                  rcg_lambda: float = 0.0, trace=None, status=None, stream=None):
    """pyr_select with the PHAROS variants: budget (int32 CUDA tensor [B, Hkv], DBA), fcf_tau / fcf_extra
    (FCF), rcg_lambda (RCG), and an optional trace buffer (new_trace)."""
    o = PyrSelectOpts(_dev(budget, "budget", True), float(fcf_tau), int(fcf_extra), float(rcg_lambda),
                      _dev(trace, "trace", True))
    _check(_L().pyr_select_ex(ctypes.byref(s), _dev(Q, "Q"), _dev(pyr, "pyr"), ctypes.byref(o), _dev(idx, "idx"),
                              _dev(gap, "gap", True), _dev(status, "status", True), _stream(stream)),
           "pyr_select_ex")


def bsa_forward(s: PyrShape, Q, K, V, idx, O, lse=None, status=None, stream=None):
    _check(_L().bsa_forward(ctypes.byref(s), _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(idx, "idx"), _dev(O, "O"),
                            _dev(lse, "lse", True), _dev(status, "status", True), _stream(stream)), "bsa_forward")


def phba_state_elems(s: PyrShape, M: int) -> int:
    return _L().phba_state_elems(ctypes.byref(s), int(M))


def phba_state_workspace_bytes(s: PyrShape, M: int) -> int:
    return _L().phba_state_workspace_bytes(ctypes.byref(s), int(M))


class PhbaStates:
    """Device buffers of the PHBA prefix states (PK, PV [B, Hkv, nb, M, d]) and the build workspace."""

    def __init__(self, s: PyrShape, M: int, device="cuda"):
        nb = (s.N + s.b - 1) // s.b
        dt = torch.float32 if s.dtype == PYR_F32 else torch.bfloat16
        self.M = M
        self.PK = torch.empty((s.B, s.Hkv, nb, M, s.d), dtype=dt, device=device)
        self.PV = torch.empty_like(self.PK)
        self.workspace = torch.empty(phba_state_workspace_bytes(s, M), dtype=torch.uint8, device=device)


def phba_state_build(s: PyrShape, M: int, Ks, V, A, W, PK, PV, workspace, status=None, stream=None):
    """Prefix states of every key block: A (retention), W (write) fp32 CUDA tensors [B, Hkv, N, M]."""
    _check(_L().phba_state_build(ctypes.byref(s), int(M), _dev(Ks, "Ks"), _dev(V, "V"), _dev(A, "A"), _dev(W, "W"),
                                 _dev(PK, "PK"), _dev(PV, "PV"), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _dev(status, "status", True),
                                 _stream(stream)), "phba_state_build")


def phba_forward(s: PyrShape, Q, K, V, idx, O, lse=None, Qs=None, M: int = 0, PK=None, PV=None, status=None,
                 stream=None):
    """bsa_forward over the tokens and the M slots of the prefix states (Qs: the state query, None = Q)."""
    _check(_L().phba_forward(ctypes.byref(s), _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(idx, "idx"),
                             _dev(Qs, "Qs", True), int(M), _dev(PK, "PK", M == 0), _dev(PV, "PV", M == 0),
                             _dev(O, "O"), _dev(lse, "lse", True), _dev(status, "status", True), _stream(stream)),
           "phba_forward")


def dense_forward(s: PyrShape, Q, K, V, O, lse=None, status=None, stream=None):
    _check(_L().dense_forward(ctypes.byref(s), _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), _dev(O, "O"),
                              _dev(lse, "lse", True), _dev(status, "status", True), _stream(stream)),
           "dense_forward")


def _host(t, name, nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu":
        raise TypeError(f"{name} must be a CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def host_workspace_bytes(s: PyrShape, units_per_chunk: int = 0, with_lse: bool = False) -> int:
    return _L().pyr_host_workspace_bytes(ctypes.byref(s), int(units_per_chunk), int(bool(with_lse)))


def bsa_forward_host(s: PyrShape, Q, K, V, O, lse=None, units_per_chunk: int = 0, workspace=None, status=None,
                     stream=None):
    """The whole forward path for host (CPU, ideally pinned) Q, K, V; writes host O and lse.

    workspace: a CUDA uint8 tensor of at least host_workspace_bytes(s, units_per_chunk, lse is not None)
    bytes. The results are ready once `stream` (default: the current stream) has been synchronised."""
    _check(_L().bsa_forward_host(ctypes.byref(s), _host(Q, "Q"), _host(K, "K"), _host(V, "V"), _host(O, "O"),
                                 _host(lse, "lse", True), int(units_per_chunk), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _dev(status, "status", True),
                                 _stream(stream)), "bsa_forward_host")


def bsa_route_invert(s: PyrShape, idx, offset, rho, status=None, stream=None):
    _check(_L().bsa_route_invert(ctypes.byref(s), _dev(idx, "idx"), _dev(offset, "offset"), _dev(rho, "rho"),
                                 _dev(status, "status", True), _stream(stream)), "bsa_route_invert")


def bsa_backward(s: PyrShape, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, status=None, stream=None):
    args = [_dev(t, n) for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O"), (lse, "lse"), (dO, "dO"), (idx, "idx"),
                                    (offset, "offset"), (rho, "rho"), (delta, "delta"), (dQ, "dQ"), (dK, "dK"),
                                    (dV, "dV"))]
    _check(_L().bsa_backward(ctypes.byref(s), *args, _dev(status, "status", True), _stream(stream)), "bsa_backward")


def bsa_backward_noalloc(s: PyrShape, Q, K, V, O, lse, dO, idx, offset, rho, dQ, dK, dV, status=None,
                         stream=None):
    """bsa_backward without the delta workspace: the library keeps it in a fixed device array."""
    args = [_dev(t, n) for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O"), (lse, "lse"), (dO, "dO"), (idx, "idx"),
                                    (offset, "offset"), (rho, "rho"), (dQ, "dQ"), (dK, "dK"), (dV, "dV"))]
    _check(_L().bsa_backward_noalloc(ctypes.byref(s), *args, _dev(status, "status", True), _stream(stream)),
           "bsa_backward_noalloc")


def selftest_wait(status, stream=None):
    """Launch the bounded-wait self-test; status (int32 CUDA tensor) reads PYR_ETIMEOUT afterwards."""
    _check(_L().pyr_selftest_wait(_dev(status, "status"), _stream(stream)), "pyr_selftest_wait")


class Buffers:
    """Device buffers of one forward pass (allocated by torch, owned by the caller)."""

    def __init__(self, s: PyrShape, device="cuda"):
        self.shape = s
        nqb = num_qblocks(s)
        dt = torch.float32 if s.dtype == PYR_F32 else torch.bfloat16
        # each node mean x is stored as the bf16 pair (hi, lo) = (RN(x), RN(x - hi))
        self.pyr = torch.empty((s.B, s.Hkv, num_nodes(s), 2, s.d), dtype=torch.bfloat16, device=device)
        self.idx = torch.empty((s.B, s.Hkv, nqb, s.topk), dtype=torch.int32, device=device)
        self.gap = torch.empty((s.B, s.Hkv, nqb), dtype=torch.float32, device=device)
        self.O = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=dt, device=device)
        self.lse = torch.empty((s.B, s.Hq, s.Nq), dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)


class BackwardBuffers:
    """Device buffers of one backward pass (allocated by torch, owned by the caller)."""

    def __init__(self, s: PyrShape, device="cuda"):
        self.shape = s
        nqb = num_qblocks(s)
        nb = (s.N + s.b - 1) // s.b
        dt = torch.float32 if s.dtype == PYR_F32 else torch.bfloat16
        self.offset = torch.empty((s.B * s.Hkv, nb + 1), dtype=torch.int32, device=device)
        self.rho = torch.empty((s.B * s.Hkv, nqb * s.topk), dtype=torch.int32, device=device)
        self.delta = torch.empty((s.B, s.Hq, s.Nq), dtype=torch.float32, device=device)
        self.dQ = torch.empty((s.B, s.Hq, s.Nq, s.d), dtype=dt, device=device)
        self.dK = torch.empty((s.B, s.Hkv, s.N, s.d), dtype=dt, device=device)
        self.dV = torch.empty((s.B, s.Hkv, s.N, s.d), dtype=dt, device=device)


def run_backward(s: PyrShape, Q, K, V, dO, fwd: "Buffers", bwd: BackwardBuffers, stream=None):
    """Enqueue route inversion and the gradients of the forward pass held in fwd."""
    bsa_route_invert(s, fwd.idx, bwd.offset, bwd.rho, fwd.status, stream)
    bsa_backward(s, Q, K, V, fwd.O, fwd.lse, dO, fwd.idx, bwd.offset, bwd.rho, bwd.delta, bwd.dQ, bwd.dK, bwd.dV,
                 fwd.status, stream)
    return bwd


def pyramid_means(s: PyrShape, pyr: torch.Tensor, stream=None) -> torch.Tensor:
    """Allocate and fill the fp32 node means [B, Hkv, P, d] of a pyramid (pyr_means)."""
    means = torch.empty((s.B, s.Hkv, num_nodes(s), s.d), dtype=torch.float32, device=pyr.device)
    pyr_means(s, pyr, means, stream=stream)
    return means


def run(s: PyrShape, Q, K, V, buf: Buffers, stream=None, with_gap=True):
    """Enqueue the whole path (pyramid, selection, attention) into buf."""
    pyr_build(s, K, buf.pyr, buf.status, stream)
    pyr_select(s, Q, buf.pyr, buf.idx, buf.gap if with_gap else None, buf.status, stream)
    bsa_forward(s, Q, K, V, buf.idx, buf.O, buf.lse, buf.status, stream)
    return buf


def forward(Q, K, V, b: int, topk: int, cap: int, q_offset: int = 0):
    """Allocate outputs and run pyramid + selection + block-sparse attention.

    Q: [B, Hq, Nq, d]; K, V: [B, Hkv, N, d] CUDA tensors (fp32 or bf16).
    Returns (O, lse, idx, gap); raises PyrError on a host-side error or on a
    device-side status (read after synchronising the current stream).
    """
    B, Hq, Nq, d = Q.shape
    N, Hkv = K.shape[2], K.shape[1]
    s = make_shape(B, Hq, Hkv, N, Nq, q_offset, d, b, topk, cap, Q.dtype)
    buf = run(s, Q, K, V, Buffers(s, Q.device))
    torch.cuda.current_stream().synchronize()
    code = int(buf.status.item())
    if code:
        raise PyrError(code, "device")
    return buf.O, buf.lse, buf.idx, buf.gap
