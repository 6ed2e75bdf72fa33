"""fp64 CPU oracle for Sketch Attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline`` /
``--impl reference`` legs may import this package. The CUDA library never calls it
and shares no code with it; the product path fails loudly when its CUDA extension
is missing instead of falling back here.

What it computes is written out in ``sa_oracle.cpp`` (plain C++, fp64, the
unfolded definition K = X W_k, V = X W_v, prototype-wise softmax, mass-weighted
mean). Sources: the "100,000 videos in your pocket" blog, section "1. Sketch
Attention compresses the history"; the evolve.pub review of arXiv 2609.08443,
"Summary" and the FAQ on how Sketch Attention differs from standard attention.

``stca_forward`` / ``stca_backward`` (``stca_oracle.cpp``) are the candidate-to-sketch
cross attention that reads the sketch (the sketch branch of STCA, one sketch read per
user for all of its candidates): blog sections "2. STCA reasons at two time scales" and
"3. The system makes it cheap enough to matter". They are pinned by
``tests/test_oracle_stca_pins.py``.

``codec`` (``codec.py``, numpy) is the sketch cache codec: bf16, and FP8 E4M3 with one
scale per row, built from the formats' definitions; pinned bit for bit against torch's
conversions by ``tests/test_oracle_codec_pins.py``.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force at 50 digits, autograd and finite
differences for the backward). The paper's analytic FLOP ratios (49.9x, 63.9x)
are not computed here: parity unpinned, context only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.cpp")
_LIB = os.path.join(_HERE, "libsa_oracle.so")
_STCA_SRC = os.path.join(_HERE, "stca_oracle.cpp")
_STCA_LIB = os.path.join(_HERE, "libstca_oracle.so")
_lock = threading.Lock()
_lib = None
_stca_lib = None


def _build_one(src: str, lib: str, force: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(src):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["g++", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c++17", "-o", tmp, src]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile the oracles with g++ (OpenMP). Returns the path of the Sketch Attention
    oracle's shared object (the cross-attention oracle is built beside it)."""
    _build_one(_STCA_SRC, _STCA_LIB, force)
    return _build_one(_SRC, _LIB, force)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SA_ORACLE_LIB lets the mutation test load a deliberately broken build.
            lib = ctypes.CDLL(os.environ.get("SA_ORACLE_LIB") or build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int64)
            lib.sa_oracle_forward.restype = ctypes.c_int
            lib.sa_oracle_forward.argtypes = [dp, ip, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                              dp, ctypes.c_int, dp, dp, dp, dp, dp, dp, ctypes.c_int]
            lib.sa_oracle_backward.restype = ctypes.c_int
            lib.sa_oracle_backward.argtypes = [dp, ip, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                               dp, ctypes.c_int, dp, dp, dp, dp,
                                               dp, dp, dp, dp, ctypes.c_int]
            _lib = lib
    return _lib


def _load_stca():
    global _stca_lib
    with _lock:
        if _stca_lib is None:
            # STCA_ORACLE_LIB lets the mutation test load a deliberately broken build.
            path = os.environ.get("STCA_ORACLE_LIB") or _build_one(_STCA_SRC, _STCA_LIB, False)
            lib = ctypes.CDLL(path)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int64)
            i32, i64 = ctypes.c_int, ctypes.c_int64
            lib.stca_oracle_forward.restype = i32
            lib.stca_oracle_forward.argtypes = [dp, ip, i32, i64, i32, dp, i32, dp, dp, dp,
                                                dp, dp, i32]
            lib.stca_oracle_backward.restype = i32
            lib.stca_oracle_backward.argtypes = [dp, ip, i32, i64, i32, dp, i32, dp, dp, dp,
                                                 dp, dp, dp, dp, dp, dp, i32]
            lib.stca_oracle_forward_keys.restype = i32
            lib.stca_oracle_forward_keys.argtypes = [dp, ip, i32, i64, i32, dp, ip, i64, dp, dp,
                                                     dp, dp, dp, i32]
            lib.stca_oracle_backward_keys.restype = i32
            lib.stca_oracle_backward_keys.argtypes = [dp, ip, i32, i64, i32, dp, ip, i64, dp, dp,
                                                      dp, dp, dp, dp, dp, dp, dp, i32]
            _stca_lib = lib
    return _stca_lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check_rc(rc: int) -> None:
    if rc == 1:
        raise ValueError("oracle: bad sizes")
    if rc == 2:
        raise ValueError("oracle: offsets must start at 0, be non-decreasing and end at n_total")
    if rc != 0:
        raise RuntimeError(f"oracle: error {rc}")


def forward(X, offsets, P, Wk, Wv, nthreads: int = 0) -> dict:
    """Sketch Attention forward in fp64.

    X [n_total, d], offsets [R+1] (int64), P [k, d], Wk [d, d], Wv [d, d].
    Returns a dict with sketch [R, k, d], mass [R, k], lse [n_total], xsketch [R, k, d].
    """
    X = _f64(X)
    P, Wk, Wv = _f64(P), _f64(Wk), _f64(Wv)
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    n_total, d = X.shape
    k = P.shape[0]
    R = off.shape[0] - 1
    assert P.shape == (k, d) and Wk.shape == (d, d) and Wv.shape == (d, d)
    sketch = np.zeros((R, k, d))
    mass = np.zeros((R, k))
    lse = np.zeros(n_total)
    xsk = np.zeros((R, k, d))
    rc = _load().sa_oracle_forward(_ptr(X), _ptr(off, ctypes.c_int64), R, n_total, d, _ptr(P), k,
                                   _ptr(Wk), _ptr(Wv), _ptr(sketch), _ptr(mass), _ptr(lse),
                                   _ptr(xsk), int(nthreads))
    _check_rc(rc)
    return {"sketch": sketch, "mass": mass, "lse": lse, "xsketch": xsk}


def backward(X, offsets, P, Wk, Wv, dsketch, dmass=None, nthreads: int = 0) -> dict:
    """Gradients of L given dL/dsketch [R, k, d] and optional dL/dmass [R, k].

    Returns dX [n_total, d] and dP [k, d], dWk [d, d], dWv [d, d] summed over users.
    """
    X = _f64(X)
    P, Wk, Wv = _f64(P), _f64(Wk), _f64(Wv)
    G = _f64(dsketch)
    Gm = None if dmass is None else _f64(dmass)
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    n_total, d = X.shape
    k = P.shape[0]
    R = off.shape[0] - 1
    assert G.shape == (R, k, d)
    assert Gm is None or Gm.shape == (R, k)
    dX = np.zeros((n_total, d))
    dP = np.zeros((k, d))
    dWk = np.zeros((d, d))
    dWv = np.zeros((d, d))
    rc = _load().sa_oracle_backward(_ptr(X), _ptr(off, ctypes.c_int64), R, n_total, d, _ptr(P), k,
                                    _ptr(Wk), _ptr(Wv), _ptr(G), _ptr(Gm), _ptr(dX), _ptr(dP),
                                    _ptr(dWk), _ptr(dWv), int(nthreads))
    _check_rc(rc)
    return {"dX": dX, "dP": dP, "dWk": dWk, "dWv": dWv}


def _stca_args(Q, cand_offsets, S, Wq, WK, WV):
    Q, S = _f64(Q), _f64(S)
    Wq, WK, WV = _f64(Wq), _f64(WK), _f64(WV)
    off = np.ascontiguousarray(np.asarray(cand_offsets, dtype=np.int64))
    n_cand, d = Q.shape
    R = off.shape[0] - 1
    assert S.ndim == 3 and S.shape[0] == R and S.shape[2] == d
    assert Wq.shape == (d, d) and WK.shape == (d, d) and WV.shape == (d, d)
    return Q, off, S, Wq, WK, WV, n_cand, d, R, S.shape[1]


def stca_forward(Q, cand_offsets, S, Wq, WK, WV, nthreads: int = 0) -> dict:
    """Candidate-to-sketch cross attention in fp64.

    Q [n_cand, d] candidates (users' groups concatenated), cand_offsets [R+1] (int64),
    S [R, k, d] the users' sketches, Wq, WK, WV [d, d]. Returns out [n_cand, d] and
    lse [n_cand] (the log-sum-exp of each candidate's scores over the k rows).
    """
    Q, off, S, Wq, WK, WV, n_cand, d, R, k = _stca_args(Q, cand_offsets, S, Wq, WK, WV)
    out = np.zeros((n_cand, d))
    lse = np.zeros(n_cand)
    rc = _load_stca().stca_oracle_forward(_ptr(Q), _ptr(off, ctypes.c_int64), R, n_cand, d,
                                          _ptr(S), k, _ptr(Wq), _ptr(WK), _ptr(WV), _ptr(out),
                                          _ptr(lse), int(nthreads))
    _check_rc(rc)
    return {"out": out, "lse": lse}


def stca_backward(Q, cand_offsets, S, Wq, WK, WV, dout, nthreads: int = 0) -> dict:
    """Gradients given dL/dout [n_cand, d]: dQ [n_cand, d], dS [R, k, d] (what flows into
    each user's sketch, i.e. Sketch Attention's dL/dsketch) and dWq, dWK, dWV [d, d]
    summed over users."""
    Q, off, S, Wq, WK, WV, n_cand, d, R, k = _stca_args(Q, cand_offsets, S, Wq, WK, WV)
    G = _f64(dout)
    assert G.shape == (n_cand, d)
    dQ = np.zeros((n_cand, d))
    dS = np.zeros((R, k, d))
    dWq, dWK, dWV = np.zeros((d, d)), np.zeros((d, d)), np.zeros((d, d))
    rc = _load_stca().stca_oracle_backward(_ptr(Q), _ptr(off, ctypes.c_int64), R, n_cand, d,
                                           _ptr(S), k, _ptr(Wq), _ptr(WK), _ptr(WV), _ptr(G),
                                           _ptr(dQ), _ptr(dS), _ptr(dWq), _ptr(dWK), _ptr(dWV),
                                           int(nthreads))
    _check_rc(rc)
    return {"dQ": dQ, "dS": dS, "dWq": dWq, "dWK": dWK, "dWV": dWV}


def _keys_args(Q, cand_offsets, Kx, key_offsets, Wq, WK, WV):
    Q, Kx = _f64(Q), _f64(Kx)
    Wq, WK, WV = _f64(Wq), _f64(WK), _f64(WV)
    coff = np.ascontiguousarray(np.asarray(cand_offsets, dtype=np.int64))
    koff = np.ascontiguousarray(np.asarray(key_offsets, dtype=np.int64))
    n_cand, d = Q.shape
    R = coff.shape[0] - 1
    assert koff.shape == (R + 1,) and Kx.ndim == 2 and Kx.shape[1] == d
    assert Wq.shape == (d, d) and WK.shape == (d, d) and WV.shape == (d, d)
    return Q, coff, Kx, koff, Wq, WK, WV, n_cand, d, R


def stca_forward_keys(Q, cand_offsets, Kx, key_offsets, Wq, WK, WV, nthreads: int = 0) -> dict:
    """Cross attention with ragged key rows: user u's candidates attend over
    Kx[key_offsets[u]:key_offsets[u+1]]. A user with candidates but no key rows gets
    out = 0 and lse = -inf."""
    Q, coff, Kx, koff, Wq, WK, WV, n_cand, d, R = _keys_args(Q, cand_offsets, Kx, key_offsets,
                                                             Wq, WK, WV)
    out = np.zeros((n_cand, d))
    lse = np.zeros(n_cand)
    rc = _load_stca().stca_oracle_forward_keys(
        _ptr(Q), _ptr(coff, ctypes.c_int64), R, n_cand, d, _ptr(Kx), _ptr(koff, ctypes.c_int64),
        Kx.shape[0], _ptr(Wq), _ptr(WK), _ptr(WV), _ptr(out), _ptr(lse), int(nthreads))
    _check_rc(rc)
    return {"out": out, "lse": lse}


def stca_backward_keys(Q, cand_offsets, Kx, key_offsets, Wq, WK, WV, dout,
                       nthreads: int = 0) -> dict:
    """Gradients of stca_forward_keys given dL/dout: dQ, dKx [n_keys, d], dWq, dWK, dWV."""
    Q, coff, Kx, koff, Wq, WK, WV, n_cand, d, R = _keys_args(Q, cand_offsets, Kx, key_offsets,
                                                             Wq, WK, WV)
    G = _f64(dout)
    assert G.shape == (n_cand, d)
    dQ = np.zeros((n_cand, d))
    dK = np.zeros(Kx.shape)
    dWq, dWK, dWV = np.zeros((d, d)), np.zeros((d, d)), np.zeros((d, d))
    rc = _load_stca().stca_oracle_backward_keys(
        _ptr(Q), _ptr(coff, ctypes.c_int64), R, n_cand, d, _ptr(Kx), _ptr(koff, ctypes.c_int64),
        Kx.shape[0], _ptr(Wq), _ptr(WK), _ptr(WV), _ptr(G), _ptr(dQ), _ptr(dK), _ptr(dWq),
        _ptr(dWK), _ptr(dWV), int(nthreads))
    _check_rc(rc)
    return {"dQ": dQ, "dKx": dK, "dWq": dWq, "dWK": dWK, "dWV": dWV}


def recent_suffix(X, offsets, L: int):
    """The recent branch's key rows: the last min(n_u, L) tokens of every user's history,
    concatenated, with their offsets (row selection only)."""
    X = np.asarray(X)
    off = np.asarray(offsets, dtype=np.int64)
    rows, koff = [], [0]
    for u in range(len(off) - 1):
        a, b = int(off[u]), int(off[u + 1])
        rows.append(np.arange(max(a, b - L), b, dtype=np.int64))
        koff.append(koff[-1] + len(rows[-1]))
    idx = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
    return X[idx], np.asarray(koff, dtype=np.int64)
