"""Thin Python binding of the LoLA C ABI (include/lola.h).

Argument marshalling only: every step of the inference path runs in the CUDA
kernels of liblola.so. PyTorch provides device memory and the current stream.
There is no CPU fallback: without the built library or a CUDA device the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblola.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "lola.h")

LOLA_F32, LOLA_BF16 = 0, 1
STATUS = {0: "LOLA_OK", 1: "LOLA_ERR_INVALID_ARG", 2: "LOLA_ERR_SHAPE", 3: "LOLA_ERR_DTYPE",
          4: "LOLA_ERR_STATE", 5: "LOLA_ERR_WORKSPACE", 6: "LOLA_ERR_CUDA",
          7: "LOLA_ERR_TIMEOUT", 8: "LOLA_ERR_DEVICE"}


class LolaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_status_string(code)})")
        self.code = code


class lola_config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("feat_dim", ctypes.c_int32), ("window", ctypes.c_int32),
                ("lambda_", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("decode_interval", ctypes.c_int32), ("max_prefill_tokens", ctypes.c_int32),
                ("eps", ctypes.c_float), ("dtype", ctypes.c_int32), ("scorer", ctypes.c_int32),
                ("w_per_kv_head", ctypes.c_int32)]


SCORERS = {"sre": 0, "attention-weight": 1, "softmax-error": 2, "fifo": 3}


_lib = None


def load_library() -> ctypes.CDLL:
    """Loads liblola.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"liblola.so not built at {LIB_PATH}; run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    C = ctypes.POINTER(lola_config)
    sigs = {
        "lola_state_bytes": (I32, [C, ctypes.POINTER(SZ)]),
        "lola_state_stream_bytes": (I32, [C, ctypes.POINTER(SZ)]),
        "lola_init_state": (I32, [C, P, P, SZ, P, ctypes.POINTER(P)]),
        "lola_reset_state": (I32, [P, P]),
        "lola_prefill_chunk": (I32, [P, P, P, P, I64, P, P]),
        "lola_prefill_host": (I32, [P, P, P, P, I64, P, P, SZ, I64, P]),
        "lola_prefill_host_staging_bytes": (I32, [C, I64, ctypes.POINTER(SZ)]),
        "lola_decode_step": (I32, [P, P, P, P, P, P]),
        "lola_decode_step_static": (I32, [P, P, P, P, P, P]),
        "lola_position": (I64, [P]),
        "lola_get_cache_indices": (I32, [P, P, P, P]),
        "lola_set_selection_log": (I32, [P, P, I64]),
        "lola_set_selection_override": (I32, [P, P, I64]),
        "lola_set_score_log": (I32, [P, P, P, I64]),
        "lola_set_fault_injection": (I32, [P, I32, I64]),
        "lola_sync": (I32, [P, P]),
        "lola_free_state": (I32, [P]),
        "lola_status_string": (ctypes.c_char_p, [I32]),
        "lola_set_timing": (I32, [P, ctypes.c_int]),
        "lola_set_prefill_schedule": (I32, [P, I32, I32]),
        "lola_prefill_plan": (I32, [C, I32, I32, I32, I64, ctypes.POINTER(I32), ctypes.POINTER(I32),
                                    ctypes.POINTER(I32)]),
        "lola_timing_read": (I32, [P, P, P]),
        "lola_launch_count": (I64, []),
        "lola_selftest_umma": (I32, [ctypes.c_int, P, P, P, ctypes.c_int, ctypes.c_int, P, P]),
    }
    for name, (res, args) in sigs.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def header_symbols() -> list:
    """Function names declared in include/lola.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(lola_\w+)\s*\(", text, re.M)))


def _status_string(code: int) -> str:
    try:
        return load_library().lola_status_string(code).decode()
    except Exception:
        return "?"


def _check(code: int, what: str):
    if code != 0:
        raise LolaError(code, what)


def make_config(*, batch, n_q_heads, n_kv_heads, head_dim, feat_dim, window, lambda_, chunk,
                decode_interval, max_prefill_tokens=0, eps=1e-6, dtype="bf16",
                scorer="sre", w_per_kv_head=False) -> lola_config:
    return lola_config(batch, n_q_heads, n_kv_heads, head_dim, feat_dim, window, lambda_, chunk,
                       decode_interval, max_prefill_tokens, eps,
                       LOLA_F32 if dtype in ("f32", "float32") else LOLA_BF16, SCORERS[scorer],
                       1 if w_per_kv_head else 0)


def config_from_workload(w, max_prefill_tokens: Optional[int] = None, **over) -> lola_config:
    kw = dict(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
              head_dim=w.head_dim, feat_dim=w.feat_dim, window=w.window, lambda_=w.lambda_,
              chunk=w.chunk, decode_interval=w.decode_interval,
              max_prefill_tokens=max_prefill_tokens or w.seq_len, eps=w.eps, dtype=w.dtype,
              scorer=getattr(w, "scorer", "sre"), w_per_kv_head=getattr(w, "w_per_head", False))
    kw.update(over)
    return make_config(**kw)


# ---- C-ABI entry points with the same names (pointer arguments are ints) ----

def lola_state_bytes(cfg: lola_config) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().lola_state_bytes(ctypes.byref(cfg), ctypes.byref(n)), "lola_state_bytes")
    return n.value


def lola_state_stream_bytes(cfg: lola_config) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().lola_state_stream_bytes(ctypes.byref(cfg), ctypes.byref(n)),
           "lola_state_stream_bytes")
    return n.value


def lola_init_state(cfg: lola_config, W: int, workspace: int, nbytes: int, stream: int) -> int:
    h = ctypes.c_void_p(0)
    _check(load_library().lola_init_state(ctypes.byref(cfg), W, workspace, nbytes, stream,
                                          ctypes.byref(h)), "lola_init_state")
    return h.value


def lola_reset_state(h: int, stream: int):
    _check(load_library().lola_reset_state(h, stream), "lola_reset_state")


def lola_prefill_chunk(h: int, q: int, k: int, v: int, n_tokens: int, out: int, stream: int):
    _check(load_library().lola_prefill_chunk(h, q, k, v, n_tokens, out, stream),
           "lola_prefill_chunk")


def lola_prefill_host(h: int, q: int, k: int, v: int, n_tokens: int, out: int, staging: int,
                      staging_bytes: int, piece_tokens: int, stream: int):
    """Prefill from host buffers, the copies pipelined with the compute in pieces."""
    _check(load_library().lola_prefill_host(h, q, k, v, n_tokens, out, staging, staging_bytes,
                                            piece_tokens, stream), "lola_prefill_host")


def lola_prefill_host_staging_bytes(cfg: lola_config, piece_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().lola_prefill_host_staging_bytes(ctypes.byref(cfg), piece_tokens, ctypes.byref(n)),
           "lola_prefill_host_staging_bytes")
    return n.value


def lola_decode_step(h: int, q: int, k: int, v: int, out: int, stream: int):
    _check(load_library().lola_decode_step(h, q, k, v, out, stream), "lola_decode_step")


def lola_decode_step_static(h: int, q: int, k: int, v: int, out: int, stream: int):
    """Decode step whose temporaries come from a fixed device array inside the
    library; for callers that cannot allocate device memory on demand."""
    _check(load_library().lola_decode_step_static(h, q, k, v, out, stream),
           "lola_decode_step_static")


def lola_position(h: int) -> int:
    return load_library().lola_position(h)


def lola_get_cache_indices(h: int, idx: int, count: int, stream: int):
    _check(load_library().lola_get_cache_indices(h, idx, count, stream), "lola_get_cache_indices")


def lola_set_selection_log(h: int, buf: int, capacity: int):
    _check(load_library().lola_set_selection_log(h, buf, capacity), "lola_set_selection_log")


def lola_set_fault_injection(handle, where: int, wait_limit_ns: int) -> None:
    _check(load_library().lola_set_fault_injection(handle, where, wait_limit_ns), "lola_set_fault_injection")


def lola_set_score_log(handle, sre_ptr: int, tok_ptr: int, capacity: int) -> None:
    _check(load_library().lola_set_score_log(handle, sre_ptr, tok_ptr, capacity), "lola_set_score_log")


def lola_set_selection_override(h: int, buf: int, n_intervals: int):
    _check(load_library().lola_set_selection_override(h, buf, n_intervals),
           "lola_set_selection_override")


def lola_sync(h: int, stream: int):
    _check(load_library().lola_sync(h, stream), "lola_sync")


def lola_set_timing(h: int, enable: bool):
    _check(load_library().lola_set_timing(h, 1 if enable else 0), "lola_set_timing")


# lola_schedule: how a prefill call overlaps its chain and its attention
SCHEDULES = {"auto": 0, "one-chain": 1, "segments": 2}


def lola_set_prefill_schedule(h: int, mode: int, intervals_per_segment: int = 0):
    _check(load_library().lola_set_prefill_schedule(h, mode, intervals_per_segment),
           "lola_set_prefill_schedule")


def lola_prefill_plan(cfg: lola_config, n_tokens: int, mode: str = "auto", intervals_per_segment: int = 0,
                      sms: int = 148) -> tuple:
    """(schedule name, intervals per segment, segments) of a prefill call of n_tokens."""
    mo, ln, ns = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load_library().lola_prefill_plan(ctypes.byref(cfg), SCHEDULES[mode], intervals_per_segment, sms,
                                            n_tokens, ctypes.byref(mo), ctypes.byref(ln), ctypes.byref(ns)),
           "lola_prefill_plan")
    name = {v: k for k, v in SCHEDULES.items()}[mo.value]
    return name, ln.value, ns.value


PHASES = ("phi", "chain", "attn", "finalize", "append", "update", "decode", "reset")


def lola_timing_read(h: int) -> dict:
    """Per-phase (total ms, count) of the events recorded since the last read."""
    ms = (ctypes.c_double * 8)()
    n = (ctypes.c_int64 * 8)()
    _check(load_library().lola_timing_read(h, ms, n), "lola_timing_read")
    return {PHASES[i]: (ms[i], n[i]) for i in range(8)}


def lola_launch_count() -> int:
    return load_library().lola_launch_count()


def lola_free_state(h: int):
    _check(load_library().lola_free_state(h), "lola_free_state")


# ---- convenience wrapper over torch device memory ----

class LolaState:
    """Owns a device workspace (torch) and a state handle."""

    def __init__(self, cfg: lola_config, W, device="cuda"):
        import torch
        self.torch = torch
        if not torch.cuda.is_available():
            raise RuntimeError("LolaState needs a CUDA device")
        self.cfg = cfg
        self.device = torch.device(device)
        self.dtype = torch.float32 if cfg.dtype == LOLA_F32 else torch.bfloat16
        self.nbytes = lola_state_bytes(cfg)
        self.workspace = torch.empty(self.nbytes, dtype=torch.uint8, device=self.device)
        self.W = self._dev(W)
        self.handle = lola_init_state(cfg, self.W.data_ptr(), self.workspace.data_ptr(),
                                      self.nbytes, self._stream())
        self._keep = []

    def _stream(self) -> int:
        return self.torch.cuda.current_stream(self.device).cuda_stream

    def _dev(self, x):
        t = self.torch.as_tensor(x)
        return t.to(device=self.device, dtype=self.dtype).contiguous()

    @property
    def streams(self) -> int:
        return self.cfg.batch * self.cfg.n_kv_heads

    def reset(self):
        lola_reset_state(self.handle, self._stream())

    def set_prefill_schedule(self, mode: str = "auto", intervals_per_segment: int = 0):
        """How the following prefill calls overlap the chain and the attention:
        "auto", "one-chain" or "segments" (see SCHEDULES)."""
        lola_set_prefill_schedule(self.handle, SCHEDULES[mode], intervals_per_segment)

    def prefill(self, q, k, v, out=None):
        q, k, v = self._dev(q), self._dev(k), self._dev(v)
        n = q.shape[1]
        if out is None:
            out = self.torch.empty_like(q)
        lola_prefill_chunk(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), n,
                           out.data_ptr(), self._stream())
        return out

    def prefill_host(self, q, k, v, out, piece_tokens, staging=None):
        """Prefill from host tensors q, k, v (pinned, contiguous, the state's dtype) into
        the host tensor out; copies and compute overlap piece by piece. staging: a device
        uint8 tensor of lola_prefill_host_staging_bytes bytes (allocated here if None)."""
        nbytes = lola_prefill_host_staging_bytes(self.cfg, piece_tokens)
        if staging is None:
            staging = self.torch.empty(nbytes, dtype=self.torch.uint8, device=self.device)
        for t in (q, k, v, out):
            if t.device.type != "cpu" or not t.is_contiguous() or t.dtype != self.dtype:
                raise ValueError("prefill_host takes contiguous host tensors of the state's dtype")
        lola_prefill_host(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), q.shape[1], out.data_ptr(),
                          staging.data_ptr(), staging.numel(), piece_tokens, self._stream())
        return out

    def decode(self, q, k, v, out=None):
        q, k, v = self._dev(q), self._dev(k), self._dev(v)
        if out is None:
            out = self.torch.empty_like(q)
        lola_decode_step(self.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         self._stream())
        return out

    @property
    def position(self) -> int:
        return lola_position(self.handle)

    def cache_indices(self):
        idx = self.torch.empty((self.cfg.batch, self.cfg.n_kv_heads, max(self.cfg.lambda_, 1)),
                               dtype=self.torch.int32, device=self.device)
        cnt = self.torch.empty((self.cfg.batch, self.cfg.n_kv_heads), dtype=self.torch.int32,
                               device=self.device)
        lola_get_cache_indices(self.handle, idx.data_ptr(), cnt.data_ptr(), self._stream())
        return idx[..., : self.cfg.lambda_], cnt

    def enable_selection_log(self, capacity: int):
        buf = self.torch.full((capacity, self.streams, self.cfg.lambda_ + 1), -2,
                              dtype=self.torch.int32, device=self.device)
        lola_set_selection_log(self.handle, buf.data_ptr(), capacity)
        self._keep.append(buf)
        return buf

    def enable_score_log(self, capacity: int):
        """Per-candidate SRE log: returns (sre float32, tok int32) device tensors of
        shape [capacity, streams, lambda + max(chunk, decode_interval)] (tok -1 unused)."""
        qc = self.cfg.lambda_ + max(self.cfg.chunk, self.cfg.decode_interval)
        sre = self.torch.zeros((capacity, self.streams, qc), dtype=self.torch.float32, device=self.device)
        tok = self.torch.full((capacity, self.streams, qc), -1, dtype=self.torch.int32, device=self.device)
        lola_set_score_log(self.handle, sre.data_ptr(), tok.data_ptr(), capacity)
        self._keep += [sre, tok]
        return sre, tok

    def set_selection_override(self, kept):
        """kept: int32 [n_int, streams, lambda+1] (count, ascending ids, -1 pad)."""
        buf = self.torch.as_tensor(kept, dtype=self.torch.int32).to(self.device).contiguous()
        lola_set_selection_override(self.handle, buf.data_ptr(), buf.shape[0])
        self._keep.append(buf)
        return buf

    def sync(self):
        lola_sync(self.handle, self._stream())

    def close(self):
        if getattr(self, "handle", None):
            lola_free_state(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
