"""Compile the C oracle (test infrastructure) into oracle/liboracle.so and load it.

Only tests, the smoke check and the benchmark's CPU-baseline legs call this.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lora_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", SRC, "-o", LIB]
        subprocess.check_call(cmd)
    return LIB


_lib = None


def load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_lora_apply.restype = ctypes.c_int
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def lora_apply_c(X, Y_base, ids, A, B, scales, nthreads: int = 0):
    """Same contract as lora_oracle.lora_apply, computed by the C oracle."""
    lib = load()
    X = np.ascontiguousarray(X, dtype=np.float32)
    Yb = np.ascontiguousarray(Y_base, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, d_in = X.shape
    d_out = Yb.shape[1]
    S = len(A)
    ranks = np.array([0 if a is None else a.shape[1] for a in A], dtype=np.int32)
    sc = np.ascontiguousarray(scales, dtype=np.float32)
    a_off = np.zeros(S, dtype=np.int64)
    b_off = np.zeros(S, dtype=np.int64)
    a_parts, b_parts = [], []
    oa = ob = 0
    for i in range(S):
        a_off[i], b_off[i] = oa, ob
        if A[i] is not None:
            a = np.ascontiguousarray(A[i], dtype=np.float32).ravel()
            b = np.ascontiguousarray(B[i], dtype=np.float32).ravel()
            a_parts.append(a)
            b_parts.append(b)
            oa += a.size
            ob += b.size
    A_all = np.concatenate(a_parts) if a_parts else np.zeros(1, np.float32)
    B_all = np.concatenate(b_parts) if b_parts else np.zeros(1, np.float32)
    Y = np.empty((T, d_out), dtype=np.float64)
    err = lib.oracle_lora_apply(_p(X), ctypes.c_int(T), ctypes.c_int(d_in), ctypes.c_int(d_out),
                                _p(Yb), _p(ids), ctypes.c_int(S), _p(ranks), _p(sc),
                                _p(A_all), _p(a_off), _p(B_all), _p(b_off), _p(Y),
                                ctypes.c_int(nthreads))
    return Y, int(err)


def max_threads() -> int:
    return int(load().oracle_max_threads())
