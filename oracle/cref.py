"""ctypes loader of the plain C++ oracle (``oracle/decode_ref.cpp``).

TEST INFRASTRUCTURE ONLY (tests and the bench's CPU legs).  ``build()`` compiles
the library in-tree with g++ (-O2, no fast-math); ``decode`` runs it on torch or
numpy bf16 inputs and returns float64 results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "decode_ref.cpp")
LIB = os.path.join(_HERE, "libsaga_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SOURCE):
        subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", "-o",
                        LIB + ".tmp", SOURCE], check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.saga_oracle_decode.restype = I
        lib.saga_oracle_decode.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, P, P, P]
        _lib = lib
    return _lib


def _bf16_bits(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 bit array -> contiguous uint16 numpy array."""
    if hasattr(t, "view") and hasattr(t, "dtype") and str(t.dtype) == "torch.bfloat16":
        import torch
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(t, dtype=np.uint16)


def decode(q, k_cache, v_cache, seq_lens, h_q: int, h_k: int, h_v: int, N: int, threads: int = 1):
    """(out [B, h_q, d], sel_idx [B, h_q, N], sel_logit [B, h_q, N]) in float64."""
    lib = _load()
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k_cache), _bf16_bits(v_cache)
    lens = np.ascontiguousarray(np.asarray(seq_lens), dtype=np.int32)
    B, _, L_max, d = kb.shape
    out = np.zeros((B, h_q, d))
    idx = np.zeros((B, h_q, N), dtype=np.int32)
    logit = np.zeros((B, h_q, N))
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = lib.saga_oracle_decode(ptr(qb), ptr(kb), ptr(vb), ptr(lens), B, L_max, h_q, h_k, h_v, d, N,
                                threads, ptr(out), ptr(idx), ptr(logit))
    if rc != 0:
        raise ValueError("saga_oracle_decode: invalid arguments")
    return out, idx, logit
