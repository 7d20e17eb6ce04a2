"""CPU oracle for the MoE token-routing path (ctypes loader for moe_oracle.cpp).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``token_dispatch_topk_b200``) never imports it and shares no code with it.

Every function takes and returns numpy arrays; bf16 tensors travel as their raw
``uint16`` bit patterns.  The arithmetic lives in ``moe_oracle.cpp``; this file
only allocates output arrays and marshals pointers.

Parity pins: every function is pinned by ``tests/test_oracle_*.py``
(hand-worked examples under ``tests/golden/``, closed forms, brute force over
all subsets, a stable library sort, exact rational accumulation, invariants),
and ``tests/test_oracle_mutants.py`` shows that planted mistakes fail them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

# Built without fused multiply-add contraction and without fast-math, so the
# only fused operations are the explicit std::fma calls in the combine.
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32


def compile_oracle(src: str, out: str) -> str:
    """g++ one oracle source file into a shared library (atomic rename)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["g++", *CXXFLAGS, "-o", tmp, src], check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile moe_oracle.cpp into libmoe_oracle.so (if stale) and return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_oracle(SOURCE, _LIB)
    return _LIB


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid argument (rc={rc})")


class Oracle:
    """The oracle functions bound to one compiled copy of moe_oracle.cpp."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        lib.oracle_topk_softmax.argtypes = [_P, ctypes.c_int, _I64, _I32, _I32, ctypes.c_int, _P, _P]
        lib.oracle_topk_softmax.restype = ctypes.c_int
        lib.oracle_topk_sigmoid.argtypes = [_P, ctypes.c_int, _I64, _I32, _I32, ctypes.c_int, _P, _P]
        lib.oracle_topk_sigmoid.restype = ctypes.c_int
        lib.oracle_align_capacity.argtypes = [_I64, _I32, _I32, _I32]
        lib.oracle_align_capacity.restype = _I64
        lib.oracle_align_permute.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P]
        lib.oracle_align_permute.restype = ctypes.c_int
        lib.oracle_gather.argtypes = [_P, _I64, _I32, _I32, _P, _I32, ctypes.c_int, _P]
        lib.oracle_gather.restype = ctypes.c_int
        lib.oracle_combine.argtypes = [_P, _P, _P, _I64, _I32, _I32, _P]
        lib.oracle_combine.restype = ctypes.c_int
        lib.oracle_reduce_partials.argtypes = [_P, _I32, _I64, _I32, _P]
        lib.oracle_reduce_partials.restype = ctypes.c_int
        self._lib = lib
        self.path = lib_path

    def topk_softmax(self, logits: np.ndarray, k: int, renormalize: bool):
        """logits: [T, E] float32, or uint16 holding bf16 bits.  Returns (weights f32 [T,k], ids i32 [T,k])."""
        logits = np.ascontiguousarray(logits)
        if logits.dtype == np.uint16:
            dtype = 1
        elif logits.dtype == np.float32:
            dtype = 0
        else:
            raise TypeError(f"logits must be float32 or bf16 bits (uint16), got {logits.dtype}")
        T, E = logits.shape
        w = np.empty((T, k), np.float32)
        ids = np.empty((T, k), np.int32)
        _check(self._lib.oracle_topk_softmax(_ptr(logits), dtype, T, E, k, int(bool(renormalize)),
                                             _ptr(w), _ptr(ids)), "topk_softmax")
        return w, ids

    def topk_sigmoid(self, logits: np.ndarray, k: int, renormalize: bool):
        """Sigmoid-scored top-k: the same selection, weights 1/(1+exp(-x)) (optionally renormalised)."""
        logits = np.ascontiguousarray(logits)
        if logits.dtype == np.uint16:
            dtype = 1
        elif logits.dtype == np.float32:
            dtype = 0
        else:
            raise TypeError(f"logits must be float32 or bf16 bits (uint16), got {logits.dtype}")
        T, E = logits.shape
        w = np.empty((T, k), np.float32)
        ids = np.empty((T, k), np.int32)
        _check(self._lib.oracle_topk_sigmoid(_ptr(logits), dtype, T, E, k, int(bool(renormalize)),
                                             _ptr(w), _ptr(ids)), "topk_sigmoid")
        return w, ids

    def align_capacity(self, T: int, k: int, E_local: int, block_size: int) -> int:
        return int(self._lib.oracle_align_capacity(T, k, E_local, block_size))

    def align_permute(self, topk_ids: np.ndarray, E_global: int, block_size: int,
                      expert_map: Optional[np.ndarray] = None, E_local: Optional[int] = None) -> dict:
        """topk_ids: [T, k] int32.  Returns a dict of the align outputs (numpy int32 arrays) + capacity."""
        topk_ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
        T, k = topk_ids.shape
        if E_local is None:
            E_local = E_global
        emap = None if expert_map is None else np.ascontiguousarray(expert_map, dtype=np.int32)
        C = self.align_capacity(T, k, E_local, block_size)
        if C < 0:
            raise ValueError("oracle align: invalid sizes")
        NB = (C + block_size - 1) // block_size
        out = dict(
            counts=np.empty(E_local, np.int32),
            offsets=np.empty(E_local + 1, np.int32),
            sorted_token_ids=np.empty(C, np.int32),
            expert_ids=np.empty(NB, np.int32),
            num_tokens_post_pad=np.empty(1, np.int32),
            inv_perm=np.empty(T * k, np.int32),
        )
        rc = self._lib.oracle_align_permute(
            _ptr(topk_ids), T, k, E_global, _ptr(emap), E_local, block_size,
            _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["sorted_token_ids"]), _ptr(out["expert_ids"]),
            _ptr(out["num_tokens_post_pad"]), _ptr(out["inv_perm"]))
        _check(rc, "align_permute")
        out["capacity"] = C
        return out

    def gather(self, hidden: np.ndarray, k: int, sorted_token_ids: np.ndarray, num_tokens_post_pad: int,
               capacity: int, zero_pad: bool = False, fill: int = 0xFFFF) -> np.ndarray:
        """hidden: [T, H] uint16 (bf16 bits).  Returns permuted [capacity, H] uint16.

        Rows the gather never writes keep ``fill`` so that a caller can tell them apart."""
        hidden = np.ascontiguousarray(hidden, dtype=np.uint16)
        T, H = hidden.shape
        permuted = np.full((capacity, H), fill, np.uint16)
        sti = np.ascontiguousarray(sorted_token_ids, dtype=np.int32)
        _check(self._lib.oracle_gather(_ptr(hidden), T, H, k, _ptr(sti), int(num_tokens_post_pad),
                                       int(bool(zero_pad)), _ptr(permuted)), "gather")
        return permuted

    def combine(self, expert_out: np.ndarray, topk_weights: np.ndarray, inv_perm: np.ndarray) -> np.ndarray:
        """expert_out: [rows, H] uint16 (bf16 bits); topk_weights: [T, k] f32; inv_perm: [T*k] i32.
        Returns out [T, H] uint16 (bf16 bits)."""
        y = np.ascontiguousarray(expert_out, dtype=np.uint16)
        w = np.ascontiguousarray(topk_weights, dtype=np.float32)
        ip = np.ascontiguousarray(inv_perm, dtype=np.int32).reshape(-1)
        T, k = w.shape
        H = y.shape[1]
        assert ip.size == T * k
        if T * k:
            assert int(ip.max()) < y.shape[0], "inv_perm row beyond expert_out"
        out = np.empty((T, H), np.uint16)
        _check(self._lib.oracle_combine(_ptr(y), _ptr(w), _ptr(ip), T, k, H, _ptr(out)), "combine")
        return out


    def reduce_partials(self, partials: np.ndarray) -> np.ndarray:
        """partials: [n, rows, H] uint16 (bf16 bits), one partial combine per rank.  Returns [rows, H]
        uint16: the fp32 sum in ascending rank order from +0, rounded once to bf16."""
        p = np.ascontiguousarray(partials, dtype=np.uint16)
        n, rows, H = p.shape
        out = np.empty((rows, H), np.uint16)
        _check(self._lib.oracle_reduce_partials(_ptr(p), n, rows, H, _ptr(out)), "reduce_partials")
        return out


_default: Optional[Oracle] = None


def default() -> Oracle:
    """The oracle built from the committed moe_oracle.cpp."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def topk_softmax(logits, k, renormalize):
    return default().topk_softmax(logits, k, renormalize)


def topk_sigmoid(logits, k, renormalize):
    return default().topk_sigmoid(logits, k, renormalize)


def align_capacity(T, k, E_local, block_size):
    return default().align_capacity(T, k, E_local, block_size)


def align_permute(topk_ids, E_global, block_size, expert_map=None, E_local=None):
    return default().align_permute(topk_ids, E_global, block_size, expert_map, E_local)


def gather(hidden, k, sorted_token_ids, num_tokens_post_pad, capacity, zero_pad=False, fill=0xFFFF):
    return default().gather(hidden, k, sorted_token_ids, num_tokens_post_pad, capacity, zero_pad, fill)


def combine(expert_out, topk_weights, inv_perm):
    return default().combine(expert_out, topk_weights, inv_perm)


def reduce_partials(partials):
    return default().reduce_partials(partials)
