"""Seeded synthetic workloads for hierarchical block-sparse attention.

This module draws inputs only; it holds none of the method's arithmetic. The
CPU oracle and the CUDA path both receive the tensors it returns, so they see
bit-identical inputs. The C generator (``synth.c``) is built into
``synth/_build/libsynth.so`` by :func:`build`.

The five workloads mirror the long-context settings the PISA abstract and the
PHBA summary discuss (4K to 1M tokens, MHA and GQA, prefill and decode); the
structure of the data (per-block key offsets, planted needle blocks) stands in
for the retrieval datasets those pages evaluate on, which are not available.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_OUT = os.path.join(_HERE, "_build", "libsynth.so")

F32, BF16 = 0, 1
NEEDLE_UNIFORM, NEEDLE_LOGUNIFORM, NEEDLE_DECODE = 0, 1, 2


@dataclass(frozen=True)
class Workload:
    """Shape and value recipe of one synthetic workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    Nq: int
    q_offset: int
    d: int
    b: int
    topk: int
    cap: int
    dtype: int  # F32 or BF16
    seed: int
    n_needle: int
    needle_mode: int
    sigma_off: float = 0.5
    needle_noise: float = 0.1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def nb(self) -> int:
        return (self.N + self.b - 1) // self.b

    @property
    def decode(self) -> bool:
        return self.Nq == 1 and self.q_offset == self.N - 1

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads, in order: a tiny fp32 causal case; 32K MHA; 64K GQA;
# 128K GQA decode; 1M MHA prefill.
WORKLOADS = [
    Workload("tiny_causal_f32_4k", 1, 2, 2, 4096, 4096, 0, 64, 64, 8, 16, F32, 0, 2, NEEDLE_UNIFORM),
    Workload("mha_bf16_32k", 1, 16, 16, 32768, 32768, 0, 128, 64, 16, 32, BF16, 1, 4, NEEDLE_UNIFORM),
    Workload("gqa_bf16_64k", 2, 32, 8, 65536, 65536, 0, 128, 64, 32, 64, BF16, 2, 8, NEEDLE_UNIFORM),
    Workload("decode_gqa_bf16_128k", 32, 32, 8, 131072, 1, 131071, 128, 64, 32, 64, BF16, 3, 4, NEEDLE_DECODE),
    Workload("mha_bf16_1m", 1, 8, 8, 1048576, 1048576, 0, 128, 128, 64, 128, BF16, 4, 8, NEEDLE_LOGUNIFORM),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP) into synth/_build."""
    if force or not os.path.exists(_OUT) or os.path.getmtime(_OUT) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_OUT), exist_ok=True)
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11", _SRC, "-o", _OUT + ".tmp", "-lm"]
        )
        os.replace(_OUT + ".tmp", _OUT)
    return _OUT


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.syn_workload.restype = ctypes.c_int
        lib.syn_workload.argtypes = [
            ctypes.c_uint64] + [ctypes.c_int] * 9 + [ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_double] + [ctypes.c_void_p] * 4
        lib.syn_fill_normal.restype = ctypes.c_int
        lib.syn_fill_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_uint64, ctypes.c_double]
        _lib = lib
    return _lib


def generate(w: Workload, pin: bool = False):
    """Draw (Q, K, V, owner) as CPU tensors for workload ``w``.

    Q: [B, Hq, Nq, d]; K, V: [B, Hkv, N, d] in the workload dtype;
    owner: [B, Hkv, nb] int32, the query block whose needle overwrote key
    block j (-1 if none).
    """
    lib = _load()
    dt = w.torch_dtype
    Q = torch.empty((w.B, w.Hq, w.Nq, w.d), dtype=dt, pin_memory=pin)
    K = torch.empty((w.B, w.Hkv, w.N, w.d), dtype=dt, pin_memory=pin)
    V = torch.empty((w.B, w.Hkv, w.N, w.d), dtype=dt, pin_memory=pin)
    owner = torch.empty((w.B, w.Hkv, w.nb), dtype=torch.int32)
    rc = lib.syn_workload(w.seed, w.B, w.Hq, w.Hkv, w.N, w.Nq, w.q_offset, w.d, w.b, w.dtype,
                          w.sigma_off, w.n_needle, w.needle_mode, w.needle_noise,
                          Q.data_ptr(), K.data_ptr(), V.data_ptr(), owner.data_ptr())
    if rc != 0:
        raise ValueError(f"synth: bad workload {w}")
    return Q, K, V, owner


def normal(seed: int, stream: int, shape, dtype=torch.float32, scale: float = 1.0) -> torch.Tensor:
    """Seeded N(0, scale^2) tensor drawn from one counter stream."""
    lib = _load()
    t = torch.empty(shape, dtype=dtype)
    code = F32 if dtype == torch.float32 else BF16
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(dtype)
    lib.syn_fill_normal(seed, stream, t.data_ptr(), code, t.numel(), scale)
    return t


STREAM_DO = 6  # the upstream gradient dO of the backward pass (streams 0-5 are the forward inputs)
STREAM_RET, STREAM_WRITE, STREAM_QS = 7, 8, 9  # prefix-state gates and the state branch's query


def phba_gates(w: Workload, M: int, retention_bias: float = 1.5):
    """Seeded prefix-state gates (A retention, W write), fp32 [B, Hkv, N, M] CPU tensors in (0, 1):
    sigmoid(N(0,1) + retention_bias) and sigmoid(N(0,1)). The bias keeps most retention gates near
    0.8, so a state remembers a few dozen tokens."""
    A = torch.sigmoid(normal(w.seed, STREAM_RET, (w.B, w.Hkv, w.N, M)) + retention_bias).contiguous()
    W = torch.sigmoid(normal(w.seed, STREAM_WRITE, (w.B, w.Hkv, w.N, M))).contiguous()
    return A, W


def state_query(w: Workload) -> torch.Tensor:
    """A seeded query for the state branch, distinct from Q: [B, Hq, Nq, d] in the workload dtype."""
    return normal(w.seed, STREAM_QS, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)


def grad_output(w: Workload, pin: bool = False) -> torch.Tensor:
    """Seeded upstream gradient dO [B, Hq, Nq, d] ~ N(0, 1) in the workload dtype (CPU tensor)."""
    t = normal(w.seed, STREAM_DO, (w.B, w.Hq, w.Nq, w.d), w.torch_dtype)
    return t.pin_memory() if pin else t


def normal_np(seed: int, stream: int, shape, scale: float = 1.0) -> np.ndarray:
    return normal(seed, stream, shape, torch.float32, scale).double().numpy()
