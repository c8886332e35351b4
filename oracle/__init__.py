"""CPU oracle for one Mixture-of-Experts layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it.

The arithmetic lives in ``moe_oracle.cpp`` (plain C++, fp32 on bf16-rounded
operands); this module only builds that file with g++ and marshals numpy
arrays through ctypes.  bf16 tensors travel as ``numpy.uint16`` bit patterns.

Definitions follow "Fine-grained Computation-Communication Overlap via
Tile-level Signaling and Scheduling for Mixture-of-Experts", Section 2.1
(route, expert computation, weighted reduction) and Section 3.2.1 (the
expert-grouped row layout); see ``moe_oracle.h`` for the readings taken where
the paper is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LOCK = threading.Lock()
_LIBS: dict[str, ctypes.CDLL] = {}


def lib_path(mutant: int = 0, out_dir: str | None = None) -> str:
    name = "liboracle_moe.so" if mutant == 0 else f"liboracle_moe_mutant{mutant}.so"
    return os.path.join(out_dir or _HERE, name)


def build(mutant: int = 0, out_dir: str | None = None, force: bool = False) -> str:
    """Compile moe_oracle.cpp into a shared library (g++, OpenMP, no fast-math,
    no FMA contraction so the arithmetic is exactly the written sequence)."""
    path = lib_path(mutant, out_dir)
    if (not force and os.path.exists(path)
            and os.path.getmtime(path) >= max(os.path.getmtime(_SRC),
                                              os.path.getmtime(os.path.join(_HERE, "moe_oracle.h")))):
        return path
    tmp = path + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, mutant: int = 0, out_dir: str | None = None):
        path = build(mutant, out_dir)
        self.lib = ctypes.CDLL(path)
        self.mutant = mutant
        L = self.lib
        P = ctypes.c_void_p
        I = ctypes.c_int
        L.oracle_set_threads.argtypes = [I]
        L.oracle_set_threads.restype = I
        L.oracle_get_threads.restype = I
        L.oracle_route.argtypes = [P, I, I, I, P, P]
        L.oracle_permute.argtypes = [P, I, I, I, P, P, P, P]
        L.oracle_gather.argtypes = [P, I, I, I, P, P]
        L.oracle_ffn_row.argtypes = [P, I, I, P, P, P, I, P]
        L.oracle_expert_ffn.argtypes = [P, P, I, I, I, P, P, P, I, I, P]
        L.oracle_combine.argtypes = [P, P, P, I, I, I, P]
        L.oracle_moe_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P]
        L.oracle_moe_tokens.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, I, P]
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        for fn in ("oracle_route", "oracle_permute", "oracle_gather", "oracle_ffn_row",
                   "oracle_expert_ffn", "oracle_combine", "oracle_moe_forward",
                   "oracle_moe_tokens"):
            getattr(L, fn).restype = I

    # -- helpers -------------------------------------------------------------
    @staticmethod
    def _p(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    @staticmethod
    def _c(a, dtype):
        a = np.ascontiguousarray(a)
        if a.dtype != dtype:
            raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
        return a

    def _check(self, rc, what):
        if rc != 0:
            raise ValueError(f"{what} failed with code {rc}")

    def set_threads(self, n: int) -> int:
        return self.lib.oracle_set_threads(int(n))

    # -- steps ---------------------------------------------------------------
    def route(self, logits, k):
        logits = self._c(logits, np.float32)
        T, E = logits.shape
        idx = np.empty((T, k), np.int32)
        gate = np.empty((T, k), np.float32)
        self._check(self.lib.oracle_route(self._p(logits), T, E, k, self._p(idx), self._p(gate)),
                    "oracle_route")
        return idx, gate

    def permute(self, topk_idx, E):
        topk_idx = self._c(topk_idx, np.int32)
        T, k = topk_idx.shape
        R = T * k
        counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        perm = np.empty(R, np.int32)
        row_of = np.empty(R, np.int32)
        self._check(self.lib.oracle_permute(self._p(topk_idx), T, E, k, self._p(counts),
                                            self._p(offsets), self._p(perm), self._p(row_of)),
                    "oracle_permute")
        return counts, offsets, perm, row_of

    def gather(self, x, perm, k):
        x = self._c(x, np.uint16)
        perm = self._c(perm, np.int32)
        T, d = x.shape
        xp = np.empty((perm.shape[0], d), np.uint16)
        self._check(self.lib.oracle_gather(self._p(x), T, d, k, self._p(perm), self._p(xp)),
                    "oracle_gather")
        return xp

    def ffn_row(self, x_row, W1e, W3e, W2e, fp32_h=False):
        x_row = self._c(x_row, np.uint16)
        W1e, W3e, W2e = (self._c(w, np.uint16) for w in (W1e, W3e, W2e))
        d, f = W1e.shape
        y = np.empty(d, np.uint16)
        self._check(self.lib.oracle_ffn_row(self._p(x_row), d, f, self._p(W1e), self._p(W3e),
                                            self._p(W2e), int(fp32_h), self._p(y)),
                    "oracle_ffn_row")
        return y

    def expert_ffn(self, x_perm, offsets, W1, W3, W2, fp32_h=False, identity=False, d=None, f=None):
        x_perm = self._c(x_perm, np.uint16)
        offsets = self._c(offsets, np.int32)
        E = offsets.shape[0] - 1
        if identity:
            d = x_perm.shape[1]
            f = f or 1
            ptrs = (None, None, None)
        else:
            W1, W3, W2 = (self._c(w, np.uint16) for w in (W1, W3, W2))
            _, d, f = W1.shape
            ptrs = (self._p(W1), self._p(W3), self._p(W2))
        y = np.empty_like(x_perm)
        self._check(self.lib.oracle_expert_ffn(self._p(x_perm), self._p(offsets), E, d, f, *ptrs,
                                               int(fp32_h), int(identity), self._p(y)),
                    "oracle_expert_ffn")
        return y

    def combine(self, y, row_of, topk_gate):
        y = self._c(y, np.uint16)
        row_of = self._c(row_of, np.int32)
        topk_gate = self._c(topk_gate, np.float32)
        T, k = topk_gate.shape
        d = y.shape[1]
        out = np.empty((T, d), np.uint16)
        self._check(self.lib.oracle_combine(self._p(y), self._p(row_of), self._p(topk_gate),
                                            T, d, k, self._p(out)), "oracle_combine")
        return out

    def forward(self, x, logits, W1, W3, W2, k, fp32_h=False, identity=False):
        """Whole layer; returns dict(out, topk_idx, topk_gate, counts, offsets, perm)."""
        x = self._c(x, np.uint16)
        logits = self._c(logits, np.float32)
        T, d = x.shape
        E = logits.shape[1]
        if identity:
            f = 1
            ptrs = (None, None, None)
        else:
            W1, W3, W2 = (self._c(w, np.uint16) for w in (W1, W3, W2))
            f = W1.shape[2]
            ptrs = (self._p(W1), self._p(W3), self._p(W2))
        R = T * k
        res = dict(out=np.empty((T, d), np.uint16), topk_idx=np.empty((T, k), np.int32),
                   topk_gate=np.empty((T, k), np.float32), counts=np.empty(E, np.int32),
                   offsets=np.empty(E + 1, np.int32), perm=np.empty(R, np.int32))
        self._check(self.lib.oracle_moe_forward(
            self._p(x), self._p(logits), *ptrs, T, d, f, E, k, int(fp32_h), int(identity),
            self._p(res["out"]), self._p(res["topk_idx"]), self._p(res["topk_gate"]),
            self._p(res["counts"]), self._p(res["offsets"]), self._p(res["perm"])),
            "oracle_moe_forward")
        return res

    def tokens(self, x, topk_idx, topk_gate, W1, W3, W2, tokens, fp32_h=False, identity=False):
        """Definition path for the listed tokens (no permutation)."""
        x = self._c(x, np.uint16)
        topk_idx = self._c(topk_idx, np.int32)
        topk_gate = self._c(topk_gate, np.float32)
        tokens = self._c(np.asarray(tokens, np.int32), np.int32)
        T, d = x.shape
        k = topk_idx.shape[1]
        if identity:
            E, f = int(topk_idx.max()) + 1, 1
            ptrs = (None, None, None)
        else:
            W1, W3, W2 = (self._c(w, np.uint16) for w in (W1, W3, W2))
            E, _, f = W1.shape
            ptrs = (self._p(W1), self._p(W3), self._p(W2))
        out = np.empty((tokens.shape[0], d), np.uint16)
        self._check(self.lib.oracle_moe_tokens(
            self._p(x), self._p(topk_idx), self._p(topk_gate), *ptrs, T, d, f, E, k,
            int(fp32_h), int(identity), self._p(tokens), int(tokens.shape[0]), self._p(out)),
            "oracle_moe_tokens")
        return out

    def f32_to_bf16(self, v: float) -> int:
        return int(self.lib.oracle_f32_to_bf16(float(v)))

    def bf16_to_f32(self, h: int) -> float:
        return float(self.lib.oracle_bf16_to_f32(int(h)))


_DEFAULT: Oracle | None = None


def get() -> Oracle:
    """The oracle itself (mutant 0), built on first use."""
    global _DEFAULT
    with _LOCK:
        if _DEFAULT is None:
            _DEFAULT = Oracle(0)
        return _DEFAULT
