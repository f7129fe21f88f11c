"""fp64 CPU oracle for causal multi-head attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline leg of
the benchmark are the only callers.  The CUDA library never imports, loads or
calls anything here, and this package imports nothing from the library.

The arithmetic lives in ``forge_attn_oracle.c`` (plain C, fp64, the full T x T
score matrix); this module only compiles it with gcc, loads it with ctypes and
loops over heads.  Every function takes numpy float64 arrays shaped
``[B, H, T, d]`` (``lse``/``D``: ``[B, H, T]``) and returns new arrays.

Definitions follow the Forge paper ("Building an LLM Training Framework from
Scratch in C++ and Metal on Apple Silicon"), sections "Attention kernel design"
(softmax with a saved per-row log-sum-exp) and "Ecosystem survey" (backward as
D = rowsum(dO o O), then dQ and dK/dV).  The C file's header lists the formulas
and the readings taken where the paper is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "forge_attn_oracle.c")
LIBRARY = os.path.join(_HERE, "libforge_attn_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(source: str = SOURCE, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math) and return the path."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", *extra_flags, "-o", output,
           source, "-lm"]
    subprocess.run(cmd, check=True)
    return output


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


class Oracle:
    """ctypes handle on one compiled copy of the oracle."""

    def __init__(self, path: str = LIBRARY):
        if path == LIBRARY and (not os.path.exists(path)
                                or os.path.getmtime(path) < os.path.getmtime(SOURCE)):
            build()
        lib = ctypes.CDLL(path)
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_fwd.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                        _dp, _dp]
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_int, _dp, _dp, _dp, _dp, ctypes.c_int,
                                         _ip, _dp, _dp, _dp, ctypes.c_int, _ip, _dp, _dp]
        self.lib = lib
        self.path = path

    # -- one head ---------------------------------------------------------------
    def fwd_head(self, q, k, v, scale, causal, want_p=False):
        T, d = q.shape
        q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        o = np.empty((T, d))
        lse = np.empty(T)
        p = np.empty((T, T)) if want_p else None
        rc = self.lib.oracle_attn_fwd(T, d, float(scale), int(causal), _ptr(q), _ptr(k),
                                      _ptr(v), _ptr(o), _ptr(lse), _ptr(p))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_fwd failed with {rc}")
        return (o, lse, p) if want_p else (o, lse)

    def bwd_head(self, q, k, v, dO, scale, causal, want_ds=False):
        T, d = q.shape
        q, k, v, dO = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, dO))
        dq, dk, dv = (np.empty((T, d)) for _ in range(3))
        ds = np.empty((T, T)) if want_ds else None
        dvec = np.empty(T) if want_ds else None
        rc = self.lib.oracle_attn_bwd(T, d, float(scale), int(causal), _ptr(q), _ptr(k),
                                      _ptr(v), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                                      _ptr(ds), _ptr(dvec))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_bwd failed with {rc}")
        return (dq, dk, dv, ds, dvec) if want_ds else (dq, dk, dv)

    def rows_head(self, q, k, v, dO, scale, causal, qidx=(), kidx=()):
        """Sampled rows of one head: (o, lse, dq) at qidx, (dk, dv) at kidx."""
        T, d = q.shape
        q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
        dO = None if dO is None else np.ascontiguousarray(dO, dtype=np.float64)
        qi = np.ascontiguousarray(qidx, dtype=np.int32)
        ki = np.ascontiguousarray(kidx, dtype=np.int32)
        nq, nk = len(qi), len(ki)
        o = np.empty((nq, d))
        lse = np.empty(nq)
        dq = np.empty((nq, d)) if dO is not None else None
        dk = np.empty((nk, d))
        dv = np.empty((nk, d))
        rc = self.lib.oracle_attn_rows(T, d, float(scale), int(causal), _ptr(q), _ptr(k),
                                       _ptr(v), _ptr(dO), nq, qi.ctypes.data_as(_ip),
                                       _ptr(o), _ptr(lse), _ptr(dq), nk,
                                       ki.ctypes.data_as(_ip), _ptr(dk), _ptr(dv))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_rows failed with {rc}")
        return o, lse, dq, dk, dv

    # -- [B, H, T, d] -------------------------------------------------------------
    @staticmethod
    def _heads(x):
        B, H = x.shape[:2]
        return [(b, h) for b in range(B) for h in range(H)]

    def fwd(self, q, k, v, scale, causal, threads=1):
        B, H, T, d = q.shape
        o = np.empty((B, H, T, d))
        lse = np.empty((B, H, T))

        def one(bh):
            b, h = bh
            o[b, h], lse[b, h] = self.fwd_head(q[b, h], k[b, h], v[b, h], scale, causal)

        _run(one, self._heads(q), threads)
        return o, lse

    def bwd(self, q, k, v, dO, scale, causal, threads=1):
        B, H, T, d = q.shape
        dq, dk, dv = (np.empty((B, H, T, d)) for _ in range(3))

        def one(bh):
            b, h = bh
            dq[b, h], dk[b, h], dv[b, h] = self.bwd_head(q[b, h], k[b, h], v[b, h],
                                                         dO[b, h], scale, causal)

        _run(one, self._heads(q), threads)
        return dq, dk, dv


def _run(fn, items, threads):
    # ctypes drops the GIL inside the C call, so heads run in parallel threads.
    if threads <= 1:
        for it in items:
            fn(it)
        return
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(fn, items))


_default = None


def default() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
