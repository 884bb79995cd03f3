"""CPU oracle for windowed INT8 recurrent-state decode (LeapQuant).

TEST INFRASTRUCTURE ONLY.  The product library never imports, loads or calls
this package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` do.  It shares no code with the CUDA path.

The arithmetic lives in ``lq_oracle.c`` (plain C, FP64 state, FP32 codec
decisions); this module compiles it with gcc on first use and marshals NumPy
arrays through ctypes.  See the C file for the passages each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lq_oracle.c")
_SO = os.path.join(_HERE, "liblq_oracle.so")
_lock = threading.Lock()
_lib = None

GATE_SCALAR, GATE_CHANNEL = 0, 1            # GDN, KDA
MODE_WINDOW, MODE_NAIVE, MODE_FP32 = 0, 1, 2
SELECT_L2, SELECT_MAXABS = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle shared library next to its source; return its path."""
    with _lock:
        stale = (not os.path.exists(_SO)) or os.path.getmtime(_SO) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _SO + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                   "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _SO)
    return _SO


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "d_k", "d_v", "window", "n_comp_rows", "n_comp_cols", "gate", "mode", "smooth", "select")]


@dataclass(frozen=True)
class Params:
    d_k: int
    d_v: int
    window: int = 64
    n_comp_rows: int = 2
    n_comp_cols: int = 2
    gate: int = GATE_SCALAR
    mode: int = MODE_WINDOW
    smooth: int = 1
    select: int = SELECT_L2

    def c(self) -> _Params:
        return _Params(self.d_k, self.d_v, self.window, self.n_comp_rows, self.n_comp_cols,
                       self.gate, self.mode, self.smooth, self.select)

    @property
    def gdim(self) -> int:
        return 1 if self.gate == GATE_SCALAR else self.d_k

    @property
    def n_comp(self) -> int:
        return 0 if self.mode == MODE_NAIVE else self.n_comp_rows + self.n_comp_cols

    @property
    def n_vec(self) -> int:
        return 0 if self.mode == MODE_NAIVE else self.n_comp_rows * self.d_k + self.n_comp_cols * self.d_v


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        dp, fp = P(ctypes.c_double), P(ctypes.c_float)
        i8p, i32p = P(ctypes.c_int8), P(ctypes.c_int32)
        pp = P(_Params)
        lib.lqo_step.argtypes = [pp, dp, dp, dp, dp, dp, ctypes.c_double, dp]
        lib.lqo_step.restype = None
        lib.lqo_encode.argtypes = [pp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                   dp, i8p, fp, fp, i32p, fp]
        lib.lqo_encode.restype = None
        lib.lqo_num_encodings.argtypes = [pp, ctypes.c_int]
        lib.lqo_num_encodings.restype = ctypes.c_int
        lib.lqo_run_heads.argtypes = [pp, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp, dp, dp,
                                      dp, dp, dp, dp, i8p, fp, fp, i32p, fp]
        lib.lqo_run_heads.restype = None
        lib.lqo_max_threads.argtypes = [ctypes.c_int]
        lib.lqo_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def step(p: Params, S, q, k, v, g, beta):
    """One dense token of the recurrence.  Returns (S_t, o_t); S is not modified."""
    lib = _load()
    S = _f64(S).copy()
    o = np.zeros(p.d_v, np.float64)
    cp = p.c()
    lib.lqo_step(ctypes.byref(cp), _ptr(S, ctypes.c_double), _ptr(_f64(q), ctypes.c_double),
                 _ptr(_f64(k), ctypes.c_double), _ptr(_f64(v), ctypes.c_double),
                 _ptr(_f64(np.atleast_1d(g)), ctypes.c_double), float(beta), _ptr(o, ctypes.c_double))
    return S, o


@dataclass
class Encoded:
    Q: np.ndarray          # int8 [d_v, d_k]
    sigma: np.ndarray      # f32 [d_v]
    s: np.ndarray          # f32 [d_k]
    comp_rows: np.ndarray  # int32 [n_rows]
    comp_cols: np.ndarray  # int32 [n_cols]
    row_vecs: np.ndarray   # f32 [n_rows, d_k]  (k-vectors of row compensators)
    col_vecs: np.ndarray   # f32 [n_cols, d_v]  (v-vectors of column compensators)
    S_tilde: np.ndarray    # f64 [d_v, d_k]  decoded window-start state


def encode(p: Params, S, n_rows: int | None = None, n_cols: int | None = None,
           smooth: int | None = None, select: int | None = None) -> Encoded:
    """Apply the state codec to one dense state (see ``lqo_encode``)."""
    lib = _load()
    nr = p.n_comp_rows if n_rows is None else n_rows
    nc = p.n_comp_cols if n_cols is None else n_cols
    sm = p.smooth if smooth is None else smooth
    sel = p.select if select is None else select
    S = _f64(S).reshape(p.d_v, p.d_k).copy()
    Q = np.zeros((p.d_v, p.d_k), np.int8)
    sigma = np.zeros(p.d_v, np.float32)
    s = np.zeros(p.d_k, np.float32)
    idx = np.zeros(max(nr + nc, 1), np.int32)
    vec = np.zeros(max(nr * p.d_k + nc * p.d_v, 1), np.float32)
    cp = p.c()
    lib.lqo_encode(ctypes.byref(cp), nr, nc, sm, sel, _ptr(S, ctypes.c_double),
                   _ptr(Q, ctypes.c_int8), _ptr(sigma, ctypes.c_float), _ptr(s, ctypes.c_float),
                   _ptr(idx, ctypes.c_int32), _ptr(vec, ctypes.c_float))
    return Encoded(Q, sigma, s, idx[:nr].copy(), idx[nr:nr + nc].copy(),
                   vec[:nr * p.d_k].reshape(nr, p.d_k).copy(),
                   vec[nr * p.d_k:nr * p.d_k + nc * p.d_v].reshape(nc, p.d_v).copy(), S)


@dataclass
class RunResult:
    o: np.ndarray                # f64 [n, T, d_v]
    S_final: np.ndarray          # f64 [n, d_v, d_k]
    Q: np.ndarray | None         # int8 [n, n_enc, d_v, d_k]
    sigma: np.ndarray | None     # f32 [n, n_enc, d_v]
    s: np.ndarray | None         # f32 [n, n_enc, d_k]
    idx: np.ndarray | None       # int32 [n, n_enc, n_comp]
    vec: np.ndarray | None       # f32 [n, n_enc, n_vec]


def num_encodings(p: Params, T: int) -> int:
    cp = p.c()
    return _load().lqo_num_encodings(ctypes.byref(cp), T)


def run(p: Params, S0, q, k, v, g, beta, snapshots: bool = True, n_threads: int = 0) -> RunResult:
    """Run n independent heads through T tokens.

    Shapes (head-major): S0 [n, d_v, d_k]; q, k [n, T, d_k]; v [n, T, d_v];
    g [n, T] (GDN) or [n, T, d_k] (KDA); beta [n, T].
    """
    lib = _load()
    q = _f64(q)
    n, T = q.shape[0], q.shape[1]
    S0 = _f64(S0).reshape(n, p.d_v, p.d_k)
    k = _f64(k).reshape(n, T, p.d_k)
    v = _f64(v).reshape(n, T, p.d_v)
    g = _f64(g).reshape(n, T, p.gdim)
    beta = _f64(beta).reshape(n, T)
    o = np.zeros((n, T, p.d_v), np.float64)
    S_final = np.zeros((n, p.d_v, p.d_k), np.float64)
    ne = num_encodings(p, T)
    Qs = sig = ss = idx = vec = None
    if snapshots and ne > 0:
        Qs = np.zeros((n, ne, p.d_v, p.d_k), np.int8)
        sig = np.zeros((n, ne, p.d_v), np.float32)
        ss = np.zeros((n, ne, p.d_k), np.float32)
        idx = np.zeros((n, ne, max(p.n_comp, 1)), np.int32)
        vec = np.zeros((n, ne, max(p.n_vec, 1)), np.float32)
    cp = p.c()
    D = ctypes.c_double
    lib.lqo_run_heads(ctypes.byref(cp), n, T, n_threads, _ptr(S0, D), _ptr(q, D), _ptr(k, D),
                      _ptr(v, D), _ptr(g, D), _ptr(beta, D), _ptr(o, D), _ptr(S_final, D),
                      _ptr(Qs, ctypes.c_int8), _ptr(sig, ctypes.c_float), _ptr(ss, ctypes.c_float),
                      _ptr(idx, ctypes.c_int32), _ptr(vec, ctypes.c_float))
    if idx is not None:
        idx = idx[..., :p.n_comp]
        vec = vec[..., :p.n_vec]
    return RunResult(o, S_final, Qs, sig, ss, idx, vec)


def max_threads(n_threads: int = 0) -> int:
    """Host threads the oracle's OpenMP loop uses (after requesting n_threads)."""
    return _load().lqo_max_threads(n_threads)
