"""Seeded synthetic workloads for the LoLA hybrid-attention inference step.

This module holds the workload definitions (shapes, cache sizes, value
distributions) and the seeded host-side input generators. It holds none of the
method's arithmetic: no feature map, no attention, no scoring. Both the CUDA
path (through the tests and the benchmark) and the CPU oracle read inputs made
here, so the two sides always see identical values.

Distributions follow the workloads described for LoLA (Low-Rank Linear
Attention with Sparse Caching, arXiv 2505.23666): N(0,1) queries, keys and
values; a seeded Gaussian feature-map matrix W ~ N(0,1)/sqrt(d); planted
"needle" pairs whose keys are near-collinear (cosine 0.9) with an earlier key
but carry a fresh value (the memory-collision case of the paper's problem
statement); and, for the 8B-shaped case, a shared rank-16 component of
magnitude 0.5 on keys and values. Values are rounded once to the workload's
dtype, and every consumer reads those rounded values.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

SEED_BASE = 20260000


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    wid: int                 # 1-based workload id, also the seed offset
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    feat_dim: int            # D: feature dimension of phi (W is head_dim x D/2)
    window: int              # eta
    lambda_: int             # sparse-cache capacity
    chunk: int               # prefill update interval C
    decode_interval: int     # decode update interval C_dec
    seq_len: int             # prefill tokens (T)
    decode_steps: int        # decode steps after the prefill (0 = prefill only)
    dtype: str               # "f32" or "bf16"
    eps: float = 1e-6
    needles: int = 0         # planted near-collinear key pairs
    lowrank: int = 0         # rank of the shared key/value component (0 = none)
    lowrank_scale: float = 0.0
    scorer: str = "sre"      # cache scoring: "sre" (the method) or an ablation
                             # ("attention-weight", "softmax-error", "fifo")
    w_per_head: bool = False  # one feature-map matrix per kv-head (W [H_kv, d, D/2])

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64,
                     feat_dim=64, window=64, lambda_=32, chunk=64, decode_interval=64,
                     seq_len=512, decode_steps=0, dtype="f32"),
    "prefill-1b": Workload("prefill-1b", 2, batch=1, n_q_heads=32, n_kv_heads=8,
                           head_dim=64, feat_dim=128, window=64, lambda_=512, chunk=64,
                           decode_interval=64, seq_len=4096, decode_steps=0,
                           dtype="bf16", needles=64),
    "decode-batched": Workload("decode-batched", 3, batch=64, n_q_heads=32,
                               n_kv_heads=8, head_dim=64, feat_dim=128, window=64,
                               lambda_=512, chunk=64, decode_interval=64, seq_len=4096,
                               decode_steps=256, dtype="bf16"),
    "prefill-8b": Workload("prefill-8b", 4, batch=4, n_q_heads=32, n_kv_heads=8,
                           head_dim=128, feat_dim=256, window=64, lambda_=1024,
                           chunk=64, decode_interval=64, seq_len=16384,
                           decode_steps=0, dtype="bf16", lowrank=16, lowrank_scale=0.5),
    "long-context": Workload("long-context", 5, batch=1, n_q_heads=32, n_kv_heads=8,
                             head_dim=128, feat_dim=256, window=64, lambda_=2048,
                             chunk=128, decode_interval=64, seq_len=65536,
                             decode_steps=512, dtype="bf16", needles=256),
    # the same long-context stream at 128K and 256K tokens (same seed and feature map;
    # the state and cache bytes do not grow with the sequence)
    "long-context-128k": Workload("long-context-128k", 5, batch=1, n_q_heads=32, n_kv_heads=8,
                                  head_dim=128, feat_dim=256, window=64, lambda_=2048,
                                  chunk=128, decode_interval=64, seq_len=131072,
                                  decode_steps=512, dtype="bf16", needles=256),
    "long-context-256k": Workload("long-context-256k", 5, batch=1, n_q_heads=32, n_kv_heads=8,
                                  head_dim=128, feat_dim=256, window=64, lambda_=2048,
                                  chunk=128, decode_interval=64, seq_len=262144,
                                  decode_steps=512, dtype="bf16", needles=256),
    # the pages' own cache setting for the 4K single-needle evaluation (window 256,
    # sparse cache 256) on the 8B-shaped heads, with planted needles as in prefill-1b
    "pages-4k": Workload("pages-4k", 6, batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
                         feat_dim=256, window=256, lambda_=256, chunk=64, decode_interval=64,
                         seq_len=4096, decode_steps=64, dtype="bf16", needles=64),
    # token-by-token update intervals (C = C_dec = 1)
    "token-by-token": Workload("token-by-token", 7, batch=2, n_q_heads=4, n_kv_heads=2,
                               head_dim=64, feat_dim=64, window=16, lambda_=24, chunk=1,
                               decode_interval=1, seq_len=96, decode_steps=32, dtype="f32"),
}


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the workload dtype; returns float32 holding them."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype != "bf16":
        raise ValueError(dtype)
    # round-to-nearest-even on the upper 16 bits (NaN-free inputs)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32).reshape(x.shape)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 values already on the bf16 grid -> uint16 bit patterns."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_W(w: Workload) -> np.ndarray:
    """Feature-map matrix W [d, D/2] ~ N(0,1)/sqrt(d), rounded to the dtype; with
    w_per_head one independent matrix per kv-head, [H_kv, d, D/2]."""
    rng = np.random.Generator(np.random.PCG64([SEED_BASE + w.wid, 1]))
    shape = (w.head_dim, w.feat_dim // 2)
    if w.w_per_head:
        shape = (w.n_kv_heads,) + shape
    W = _normal(rng, shape) / np.float32(np.sqrt(w.head_dim))
    return round_to_dtype(W, w.dtype)


def _plant_needles(k: np.ndarray, n_needles: int, window: int, chunk: int,
                   rng: np.random.Generator) -> np.ndarray:
    """Replace n_needles keys by keys at cosine 0.9 with a uniformly chosen
    earlier key of the same (batch, kv-head) stream. k: [B, T, H, d].
    Needle positions are shared by all streams; directions are independent."""
    B, T, H, d = k.shape
    lo, hi = window + chunk, T - window - chunk
    if n_needles <= 0 or hi - lo < n_needles:
        return np.empty((0, 2), np.int64)
    pos = np.sort(rng.choice(np.arange(lo, hi), size=n_needles, replace=False))
    src = np.array([rng.integers(0, j) for j in pos], dtype=np.int64)
    for b in range(B):
        for h in range(H):
            ks = k[b, src, h, :].astype(np.float64)                  # [n, d]
            nrm = np.linalg.norm(ks, axis=1, keepdims=True)
            khat = ks / nrm
            u = rng.standard_normal(size=ks.shape)
            u -= np.sum(u * khat, axis=1, keepdims=True) * khat      # orthogonal part
            u /= np.linalg.norm(u, axis=1, keepdims=True)
            k[b, pos, h, :] = (nrm * (0.9 * khat + np.sqrt(0.19) * u)).astype(np.float32)
    return np.stack([pos, src], axis=1)


def _lowrank(rng: np.random.Generator, shape, rank: int, scale: float) -> np.ndarray:
    """scale * (a @ U^T) with U [d, rank] orthonormal and a ~ N(0, d/rank)."""
    B, T, H, d = shape
    U, _ = np.linalg.qr(rng.standard_normal(size=(d, rank)))
    a = rng.standard_normal(size=(B, T, H, rank)).astype(np.float32)
    a *= np.float32(np.sqrt(d / rank))
    return np.float32(scale) * (a @ U.T.astype(np.float32))


def make_inputs(w: Workload, T: Optional[int] = None, part: str = "prefill",
                batch: Optional[int] = None):
    """Seeded q, k, v for a workload, as float32 arrays on the dtype grid.

    part="prefill": T tokens (default w.seq_len) with the workload's structure.
    part="decode": w.decode_steps fresh N(0,1) tokens (independent stream).
    Layout: q [B, T, H_q, d], k and v [B, T, H_kv, d] (token-major per batch).
    Returns (q, k, v, meta) where meta records planted needles.
    """
    if T is None:
        T = w.seq_len if part == "prefill" else w.decode_steps
    B = w.batch if batch is None else batch
    sub = {"prefill": 2, "decode": 3}[part]
    rng = np.random.Generator(np.random.PCG64([SEED_BASE + w.wid, sub]))
    q = _normal(rng, (B, T, w.n_q_heads, w.head_dim))
    k = _normal(rng, (B, T, w.n_kv_heads, w.head_dim))
    v = _normal(rng, (B, T, w.n_kv_heads, w.head_dim))
    meta = {"needles": np.empty((0, 2), np.int64)}
    if part == "prefill":
        if w.lowrank:
            k += _lowrank(rng, k.shape, w.lowrank, w.lowrank_scale)
            v += _lowrank(rng, v.shape, w.lowrank, w.lowrank_scale)
        if w.needles:
            meta["needles"] = _plant_needles(k, w.needles, w.window, w.chunk, rng)
    return (round_to_dtype(q, w.dtype), round_to_dtype(k, w.dtype),
            round_to_dtype(v, w.dtype), meta)


def make_random(shape, seed: int, dtype: str = "f32", scale: float = 1.0) -> np.ndarray:
    """Generic seeded N(0, scale^2) array on the dtype grid (for tests)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return round_to_dtype(_normal(rng, shape) * np.float32(scale), dtype)
