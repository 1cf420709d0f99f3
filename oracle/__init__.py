"""CPU oracle for pyramid top-K block selection + causal block-sparse attention.

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may call it; the CUDA product path never does.

The arithmetic lives in ``pyr_oracle.c`` (plain C, double accumulation, no
code shared with the CUDA library). This wrapper only compiles it with gcc
and marshals arguments. Every function follows the PISA abstract (pyramid of
pooled keys, coarse-to-fine LogSumExp scoring of a bounded candidate set) and
the PHBA summary (block centroids as mean key rows; routes to strictly
preceding blocks, -1 padding; the current block always attended causally;
output plus log-sum-exp). See the header of ``pyr_oracle.c`` for the readings
taken where the pages are silent.

Parity pins (tests/test_oracle_*.py) check this oracle against closed forms,
library routines, brute force and invariants, never against the CUDA path.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pyr_oracle.c")
_OUT = os.path.join(_HERE, "_build", "liboracle.so")


class OraShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "Hq", "Hkv", "N", "Nq", "q_offset", "d", "b", "topk", "cap",
                                             "dtype")]


class OraSelectOpts(ctypes.Structure):
    _fields_ = [("budget", ctypes.c_void_p), ("fcf_tau", ctypes.c_double), ("fcf_extra", ctypes.c_int),
                ("rcg_lambda", ctypes.c_double)]


class SelectOpts:
    """The PHAROS selection variants (PHAROS page, "Four mechanisms powering PHAROS"); defaults = plain walk.

    budget      DBA: level-0 budget of each (batch, kv head) unit ([B * Hkv] ints, clamped to [0, topk]),
                or None for topk - fcf_extra everywhere;
    fcf_tau,    FCF: when the walk's confidence (its smallest margin above level 0 and at the level-0
    fcf_extra   budget boundary) is below fcf_tau, level 0 keeps fcf_extra more blocks (at most topk);
    rcg_lambda  RCG: candidates rank by R = S + rcg_lambda * R(parent).
    """

    def __init__(self, budget=None, fcf_tau=0.0, fcf_extra=0, rcg_lambda=0.0):
        self.budget = None if budget is None else np.ascontiguousarray(np.asarray(budget, dtype=np.int32))
        self.fcf_tau, self.fcf_extra, self.rcg_lambda = float(fcf_tau), int(fcf_extra), float(rcg_lambda)

    def c_struct(self):
        return OraSelectOpts(None if self.budget is None else self.budget.ctypes.data, self.fcf_tau,
                             self.fcf_extra, self.rcg_lambda)


def build(force: bool = False) -> str:
    """Compile the oracle (gcc -O2, OpenMP over independent units)."""
    if force or not os.path.exists(_OUT) or os.path.getmtime(_OUT) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_OUT), exist_ok=True)
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", _SRC, "-o",
                               _OUT + ".tmp", "-lm"])
        os.replace(_OUT + ".tmp", _OUT)
    return _OUT


_lib = None
_P = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        sp = ctypes.POINTER(OraShape)
        lib.ora_num_levels.argtypes = [sp]
        lib.ora_num_levels.restype = ctypes.c_int
        lib.ora_num_nodes.argtypes = [sp]
        lib.ora_num_nodes.restype = ctypes.c_int64
        lib.ora_num_qblocks.argtypes = [sp]
        lib.ora_num_qblocks.restype = ctypes.c_int64
        lib.ora_first_qblock.argtypes = [sp]
        lib.ora_first_qblock.restype = ctypes.c_int64
        lib.ora_pyramid.argtypes = [sp, _P, ctypes.c_int, _P, _P]
        lib.ora_pyramid.restype = ctypes.c_int
        lib.ora_node_score.argtypes = [sp, _P, _P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
        lib.ora_node_score.restype = ctypes.c_int
        lib.ora_select.argtypes = [sp, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P, _P, _P]
        lib.ora_select.restype = ctypes.c_int
        lib.ora_select_ex.argtypes = [sp, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, _P, ctypes.c_int,
                                      ctypes.POINTER(OraSelectOpts), _P, _P, _P, _P]
        lib.ora_select_ex.restype = ctypes.c_int
        lib.ora_trace_levels.argtypes = [sp]
        lib.ora_trace_levels.restype = ctypes.c_int
        lib.ora_trace_width.argtypes = [sp]
        lib.ora_trace_width.restype = ctypes.c_int
        lib.ora_attend.argtypes = [sp, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, _P]
        lib.ora_attend.restype = ctypes.c_int
        lib.ora_prefix_states.argtypes = [sp, ctypes.c_int, _P, _P, _P, _P, ctypes.c_int, _P, _P, _P]
        lib.ora_prefix_states.restype = ctypes.c_int
        lib.ora_attend_states.argtypes = [sp, _P, _P, _P, _P, ctypes.c_int, _P, _P, ctypes.c_int, _P, _P, _P, _P]
        lib.ora_attend_states.restype = ctypes.c_int
        lib.ora_route_invert.argtypes = [sp, _P, ctypes.c_int32, _P, _P]
        lib.ora_route_invert.restype = ctypes.c_int
        lib.ora_attend_bwd_q.argtypes = [sp, _P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P]
        lib.ora_attend_bwd_q.restype = ctypes.c_int
        lib.ora_attend_bwd_kv.argtypes = [sp, _P, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P, _P]
        lib.ora_attend_bwd_kv.restype = ctypes.c_int
        _lib = lib
    return _lib


def shape_of(w) -> OraShape:
    """OraShape from any object with the workload fields (B, Hq, ..., dtype)."""
    return OraShape(w.B, w.Hq, w.Hkv, w.N, w.Nq, w.q_offset, w.d, w.b, w.topk, w.cap, w.dtype)


def _ptr(t):
    if isinstance(t, torch.Tensor):
        assert t.device.type == "cpu" and t.is_contiguous()
        return t.data_ptr()
    assert isinstance(t, np.ndarray) and t.flags["C_CONTIGUOUS"]
    return t.ctypes.data


def num_levels(w) -> int:
    return _load().ora_num_levels(ctypes.byref(shape_of(w)))


def num_nodes(w) -> int:
    return _load().ora_num_nodes(ctypes.byref(shape_of(w)))


def num_qblocks(w) -> int:
    return _load().ora_num_qblocks(ctypes.byref(shape_of(w)))


def level_offsets(w):
    """(offset, count) of each pyramid level in the level-major node list."""
    nb = (w.N + w.b - 1) // w.b
    out, off, l = [], 0, 0
    while True:
        n = (nb + (1 << l) - 1) >> l
        out.append((off, n))
        off += n
        if n == 1:
            break
        l += 1
    return out


def pyramid(w, K, units) -> np.ndarray:
    """Pyramids of the listed (batch*Hkv + kv_head) units: [len(units), P, d] float64."""
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    out = np.empty((len(units), num_nodes(w), w.d), dtype=np.float64)
    rc = _load().ora_pyramid(ctypes.byref(shape_of(w)), _ptr(K), len(units), _ptr(units), _ptr(out))
    if rc:
        raise ValueError(f"ora_pyramid rc={rc}")
    return out


def node_score(w, Q, pyr_unit: np.ndarray, unit: int, qb: int, level: int, m: int):
    """(score, n_valid) of node (level, m) for query block qb; (-inf, 0) if invalid."""
    s, n = ctypes.c_double(), ctypes.c_double()
    pyr_unit = np.ascontiguousarray(pyr_unit)
    _load().ora_node_score(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(pyr_unit), unit, qb, level, m,
                           ctypes.byref(s), ctypes.byref(n))
    return s.value, n.value


def trace_levels(w) -> int:
    """Levels of a selection trace: the start level s0 down to 0 (s0 + 1)."""
    return _load().ora_trace_levels(ctypes.byref(shape_of(w)))


def trace_width(w) -> int:
    """Entries per trace level: max(cap / 2, topk)."""
    return _load().ora_trace_width(ctypes.byref(shape_of(w)))


def select(w, Q, pyr: np.ndarray, units, items, start_level: int = -1, opts: SelectOpts = None,
           with_trace: bool = False):
    """Selection for items [(slot, qb), ...]; slot indexes ``units`` / ``pyr``.

    Returns (idx [n, topk] int32, gap [n] float64, ncand [n, L+1] int32), plus, with with_trace,
    trace [n, levels, width] int32: row s0 - l lists the nodes kept at level l, best first, then -1.
    """
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    items = np.asarray(items, dtype=np.int64).reshape(-1, 2)
    slot = np.ascontiguousarray(items[:, 0].astype(np.int32))
    qb = np.ascontiguousarray(items[:, 1].astype(np.int64))
    n = len(items)
    idx = np.empty((n, max(w.topk, 1)), dtype=np.int32)
    gap = np.empty(n, dtype=np.float64)
    ncand = np.empty((n, num_levels(w)), dtype=np.int32)
    pyr = np.ascontiguousarray(pyr)
    tl = trace_levels(w) if start_level < 0 else min(start_level, num_levels(w) - 1) + 1
    trace = np.empty((n, tl, trace_width(w)), dtype=np.int32) if with_trace else None
    if opts is not None and opts.budget is not None:
        assert len(opts.budget) == w.B * w.Hkv
    co = opts.c_struct() if opts is not None else None
    rc = _load().ora_select_ex(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(pyr), len(units), _ptr(units), n,
                               _ptr(slot), _ptr(qb), start_level, ctypes.byref(co) if co is not None else None,
                               _ptr(idx), _ptr(gap), _ptr(ncand), None if trace is None else _ptr(trace))
    if rc:
        raise ValueError(f"ora_select_ex rc={rc}")
    if with_trace:
        return idx[:, :w.topk], gap, ncand, trace
    return idx[:, :w.topk], gap, ncand


def select_all(w, Q, K, units=None, start_level: int = -1, opts: SelectOpts = None):
    """Full selection for the listed units (default: all): idx [U, nqb, topk], gap [U, nqb], ncand."""
    if units is None:
        units = list(range(w.B * w.Hkv))
    pyr = pyramid(w, K, units)
    nqb = num_qblocks(w)
    items = [(s, q) for s in range(len(units)) for q in range(nqb)]
    idx, gap, ncand = select(w, Q, pyr, units, items, start_level, opts)
    return idx.reshape(len(units), nqb, w.topk), gap.reshape(len(units), nqb), ncand.reshape(len(units), nqb, -1)


def attend(w, Q, K, V, idx, rows, dense: bool = False):
    """Attention for flat query rows ((b*Hq + hq)*Nq + t): (O [n, d], lse [n]) float64.

    idx: [B, Hkv, nqb, topk] int32 (ignored when dense).
    """
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rows)
    O = np.empty((n, w.d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    if idx is None:
        idx_arr = np.zeros(1, dtype=np.int32)
    else:
        idx_arr = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    rc = _load().ora_attend(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx_arr), n, _ptr(rows),
                            1 if dense else 0, _ptr(O), _ptr(lse))
    if rc == 2:
        raise ValueError("ora_attend: idx lists a block that is not strictly before the query block, or repeats")
    if rc:
        raise ValueError(f"ora_attend rc={rc}")
    return O, lse


# ---- PHBA prefix-state branch (PHBA summary, 2.2, 3.2, 3.3, A.1.1, A.1.3) ----

def prefix_states(w, M: int, Ks, V, A, W, units=None):
    """Prefix states of the listed units (default: all): (PK, PV) [len(units), nb, M, d] float64.

    Ks (state-branch keys) and V: [B, Hkv, N, d] in the workload dtype; A (retention) and W (write):
    [B, Hkv, N, M] float32. Slot s of the key state follows SK <- A_t[s] SK + W_t[s] k_t (the value
    state likewise, with v_t), from zero; block j's state is taken after the tokens before j * b."""
    if units is None:
        units = list(range(w.B * w.Hkv))
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    nb = (w.N + w.b - 1) // w.b
    PK = np.empty((len(units), nb, M, w.d), dtype=np.float64)
    PV = np.empty_like(PK)
    A = A.contiguous() if isinstance(A, torch.Tensor) else np.ascontiguousarray(A, dtype=np.float32)
    W = W.contiguous() if isinstance(W, torch.Tensor) else np.ascontiguousarray(W, dtype=np.float32)
    rc = _load().ora_prefix_states(ctypes.byref(shape_of(w)), M, _ptr(Ks), _ptr(V), _ptr(A), _ptr(W), len(units),
                                   _ptr(units), _ptr(PK), _ptr(PV))
    if rc:
        raise ValueError(f"ora_prefix_states rc={rc}")
    return PK, PV


def attend_states(w, Q, K, V, idx, rows, PK, PV, Qs=None):
    """Attention of flat query rows over tokens and prefix-state slots: (O [n, d], lse [n]) float64.

    PK, PV: [B * Hkv, nb, M, d] float64 (the states of every unit); Qs: the state branch's query
    (None: Q)."""
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = len(rows)
    O = np.empty((n, w.d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    M = 0 if PK is None else PK.shape[2]
    PK = None if PK is None else np.ascontiguousarray(PK, dtype=np.float64)
    PV = None if PV is None else np.ascontiguousarray(PV, dtype=np.float64)
    rc = _load().ora_attend_states(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(K), _ptr(V), _ptr(_idx_arr(idx)), n,
                                   _ptr(rows), None if Qs is None else _ptr(Qs), M,
                                   None if PK is None else _ptr(PK), None if PV is None else _ptr(PV), _ptr(O),
                                   _ptr(lse))
    if rc == 2:
        raise ValueError("ora_attend_states: idx lists a block that is not strictly before the query block, or repeats")
    if rc:
        raise ValueError(f"ora_attend_states rc={rc}")
    return O, lse


# ---- backward (PHBA summary, A.1.2 block-major route metadata; A.1.4 sparse backward) ----

F64 = 2  # oracle-only element type (float64 tensors), for finite-difference pins


def _idx_arr(idx):
    if idx is None:
        return np.zeros(1, dtype=np.int32)
    return np.ascontiguousarray(np.asarray(idx, dtype=np.int32))


def route_invert(w, idx):
    """Block-major form of the routes: (offset [U, nb+1], rho [U, nqb*topk]) int32.

    For unit u and key block j, rho[u, offset[u, j]:offset[u, j+1]] lists, ascending,
    the query blocks qb (row index of idx) whose routes contain j; the diagonal block
    is not listed. Entries of rho past offset[u, nb] are -1.
    """
    idx = _idx_arr(idx)
    U, nqb = w.B * w.Hkv, num_qblocks(w)
    nb = (w.N + w.b - 1) // w.b
    offset = np.zeros((U, nb + 1), dtype=np.int32)
    rho = np.full((U, max(nqb * w.topk, 1)), -1, dtype=np.int32)
    for u in range(U):
        off_u = np.zeros(nb + 1, dtype=np.int32)
        rho_u = np.full(max(nqb * w.topk, 1), -1, dtype=np.int32)
        rc = _load().ora_route_invert(ctypes.byref(shape_of(w)), _ptr(idx), u, _ptr(off_u), _ptr(rho_u))
        if rc == 2:
            raise ValueError("ora_route_invert: idx lists a block that is not strictly before the query block, or repeats")
        if rc:
            raise ValueError(f"ora_route_invert rc={rc}")
        offset[u], rho[u] = off_u, rho_u
    return offset, rho


def attend_bwd_q(w, Q, K, V, dO, idx, rows, dense: bool = False):
    """dQ [n, d] float64 of sum(dO * O) for flat query rows ((b*Hq + hq)*Nq + t)."""
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dQ = np.empty((len(rows), w.d), dtype=np.float64)
    rc = _load().ora_attend_bwd_q(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(_idx_arr(idx)),
                                  len(rows), _ptr(rows), 1 if dense else 0, _ptr(dQ))
    if rc:
        raise ValueError(f"ora_attend_bwd_q rc={rc}")
    return dQ


def attend_bwd_kv(w, Q, K, V, dO, idx, blocks, dense: bool = False):
    """(dK, dV) [n, b, d] float64 of sum(dO * O) for key blocks given as (unit, j) pairs."""
    nb = (w.N + w.b - 1) // w.b
    blocks = np.asarray(blocks, dtype=np.int64).reshape(-1, 2)
    flat = np.ascontiguousarray(blocks[:, 0] * nb + blocks[:, 1])
    dK = np.empty((len(flat), w.b, w.d), dtype=np.float64)
    dV = np.empty((len(flat), w.b, w.d), dtype=np.float64)
    rc = _load().ora_attend_bwd_kv(ctypes.byref(shape_of(w)), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(_idx_arr(idx)),
                                   len(flat), _ptr(flat), 1 if dense else 0, _ptr(dK), _ptr(dV))
    if rc:
        raise ValueError(f"ora_attend_bwd_kv rc={rc}")
    return dK, dV
