"""CPU oracle for the LoLA hybrid-attention inference step.

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's CPU-baseline leg, never by the product path. It shares no code with
the CUDA path.

Two independent formulations live here:
  * `run` -- the fp64 C oracle (lola_oracle.c): the interval recurrence of the
    "Inferentiestrategie" section (score, keep top-lambda by SRE, fold the rest,
    combine), threaded over independent (batch, kv-head) streams.
  * `brute` -- a NumPy set-based restatement for tiny inputs that recomputes the
    state from the folded set at every interval (no recurrence) and classifies
    every (query, key) pair directly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lola_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liblola_oracle.so")
_lib = None


class OracleCfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("D", ctypes.c_int32), ("eta", ctypes.c_int32),
                ("lam", ctypes.c_int32), ("eps", ctypes.c_double), ("scorer", ctypes.c_int32),
                ("w_per_head", ctypes.c_int32)]


SCORERS = {"sre": 0, "attention-weight": 1, "softmax-error": 2, "fifo": 3}


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into oracle/_build (idempotent)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        lib.oracle_run.restype = ctypes.c_int
        lib.oracle_run.argtypes = [ctypes.POINTER(OracleCfg), ctypes.c_int, P, P, P, P,
                                   ctypes.c_int, P, P, P, ctypes.c_int, P, P, P, P, P, P, P,
                                   ctypes.c_int, P, P, ctypes.c_int]
        lib.oracle_phi.restype = None
        lib.oracle_phi.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_sre.restype = ctypes.c_double
        lib.oracle_sre.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def phi(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """phi(x) = [softmax(xW), softmax(-xW)] in fp64 for one vector x."""
    lib = _load()
    x = np.ascontiguousarray(x, np.float64)
    W = np.ascontiguousarray(W, np.float64)
    out = np.zeros(2 * W.shape[1], np.float64)
    lib.oracle_phi(_ptr(x), _ptr(W), x.shape[0], out.shape[0], _ptr(out))
    return out


def sre(phik: np.ndarray, v: np.ndarray, H: np.ndarray, s: np.ndarray, eps: float) -> float:
    lib = _load()
    phik = np.ascontiguousarray(phik, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    H = np.ascontiguousarray(H, np.float64)
    s = np.ascontiguousarray(s, np.float64)
    return lib.oracle_sre(_ptr(phik), _ptr(v), _ptr(H), _ptr(s), v.shape[0], phik.shape[0], eps)


class OracleResult:
    """Outputs and per-interval logs of one oracle run.

    out      [B, T, Hq, d] fp64 (rows outside qmask are zero); with compact=True
             [B, n_sel, Hq, d] holding only the qmask positions, in order (rows)
    kept     [n_int, B*Hkv, lam] int32: kept token ids after each interval, ascending, -1 pad
    nkept    [n_int, B*Hkv]
    nq       [n_int, B*Hkv] number of candidates |Q|
    margin   [n_int, B*Hkv] (SRE_(lam) - SRE_(lam+1)) / SRE_(lam); inf when |Q| <= lam
    cand_tok, cand_sre [n_int, B*Hkv, cap] (when requested)
    H, s     final state [B*Hkv, D, d], [B*Hkv, D] (when requested)
    """


def run(q: np.ndarray, k: np.ndarray, v: np.ndarray, W: np.ndarray, *, window: int,
        lambda_: int, intervals: Sequence[int], eps: float = 1e-6,
        qmask: Optional[np.ndarray] = None, want_cands: bool = False,
        want_state: bool = False, threads: Optional[int] = None,
        compact: bool = False, scorer: str = "sre") -> OracleResult:
    """Runs the recurrence from an empty state over tokens split into `intervals`.
    compact=True (with qmask) stores only the outputs of the masked positions.
    scorer: "sre" (the method), or the alternatives "attention-weight",
    "softmax-error" and "fifo" (see lola_oracle.c); cand_sre then logs that score."""
    lib = _load()
    q = np.ascontiguousarray(q, np.float32)
    k = np.ascontiguousarray(k, np.float32)
    v = np.ascontiguousarray(v, np.float32)
    W = np.ascontiguousarray(W, np.float32)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    D = 2 * W.shape[-1]
    per_head = W.ndim == 3          # W [Hkv, d, D/2]: one feature-map matrix per kv-head
    if per_head and W.shape[0] != Hkv:
        raise ValueError("per-head W needs one matrix per kv-head")
    ints = np.ascontiguousarray(np.asarray(intervals, np.int32))
    n_int = len(ints)
    ns = B * Hkv
    cfg = OracleCfg(B, Hq, Hkv, d, D, window, lambda_, eps, SCORERS[scorer], 1 if per_head else 0)
    r = OracleResult()
    out_row = None
    n_out = T
    if compact and qmask is not None:
        sel = np.flatnonzero(np.asarray(qmask) != 0)
        out_row = np.full(T, -1, np.int32)
        out_row[sel] = np.arange(len(sel), dtype=np.int32)
        n_out = len(sel)
        r.rows = sel
    r.out = np.zeros((B, n_out, Hq, d), np.float64)
    lam_alloc = max(lambda_, 1)
    r.kept = np.full((n_int, ns, lam_alloc), -1, np.int32)
    r.nkept = np.zeros((n_int, ns), np.int32)
    r.nq = np.zeros((n_int, ns), np.int32)
    r.margin = np.zeros((n_int, ns), np.float64)
    cap = lambda_ + (int(ints.max()) if n_int else 0)
    r.cand_tok = np.full((n_int, ns, cap), -1, np.int32) if want_cands else None
    r.cand_sre = np.zeros((n_int, ns, cap), np.float64) if want_cands else None
    r.H = np.zeros((ns, D, d), np.float64) if want_state else None
    r.s = np.zeros((ns, D), np.float64) if want_state else None
    qm = None if qmask is None else np.ascontiguousarray(qmask, np.uint8)
    nt = threads if threads else max(1, len(os.sched_getaffinity(0)))
    rc = lib.oracle_run(ctypes.byref(cfg), T, _ptr(q), _ptr(k), _ptr(v), _ptr(W), n_int,
                        _ptr(ints), _ptr(qm), _ptr(out_row), n_out, _ptr(r.out),
                        _ptr(r.kept) if lambda_ > 0 else None, _ptr(r.nkept), _ptr(r.nq),
                        _ptr(r.margin), _ptr(r.cand_tok), _ptr(r.cand_sre), cap,
                        _ptr(r.H), _ptr(r.s), nt)
    if rc != 0:
        raise ValueError(f"oracle_run rejected its arguments (code {rc})")
    if lambda_ == 0:
        r.kept = np.zeros((n_int, ns, 0), np.int32)
    r.intervals = ints
    return r
