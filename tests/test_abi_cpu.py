"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/lola.h declares, sizes workspaces, and rejects bad
arguments with the documented status codes before touching the device."""
import ctypes

import pytest

from hybrid_linear_attention_lola_b200 import build as B
from hybrid_linear_attention_lola_b200 import lola as L
from hybrid_linear_attention_lola_b200 import workloads as wl


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def test_exports_every_header_symbol(lib):
    names = L.header_symbols()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n


def test_state_bytes_for_every_workload(lib):
    for w in wl.WORKLOADS.values():
        cfg = L.config_from_workload(w, max_prefill_tokens=min(w.seq_len, 16384))
        n = L.lola_state_bytes(cfg)
        assert n > 0 and n % 256 == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("head_dim,feat_dim,g", [(32, 32, 1), (64, 128, 4), (128, 256, 8), (128, 64, 3)])
def test_state_bytes_across_shapes(lib, dtype, head_dim, feat_dim, g):
    # every documented head_dim / feat_dim / group size keeps a launch shape that fits
    cfg = L.make_config(batch=3, n_q_heads=2 * g, n_kv_heads=2, head_dim=head_dim, feat_dim=feat_dim,
                        window=64, lambda_=512, chunk=64, decode_interval=64, max_prefill_tokens=128,
                        eps=1e-6, dtype=dtype)
    n = L.lola_state_bytes(cfg)
    assert n > 0 and n % 256 == 0


def test_stream_bytes_constant_in_sequence_length(lib):
    w = wl.WORKLOADS["long-context"]
    sizes = {L.lola_state_stream_bytes(L.config_from_workload(w, max_prefill_tokens=n))
             for n in (128, 4096, 65536)}
    assert len(sizes) == 1
    # H|s fp32 + cache K/V bf16 + indices + ring K/V bf16 + flags
    d, D, lam, eta, C = 128, 256, 2048, 64, 128
    R = 256                         # power of two >= eta + C + 1
    assert sizes.pop() == D * d * 4 + D * 4 + 2 * lam * d * 2 + lam * 4 + 2 * R * d * 2 + C


@pytest.mark.parametrize("field,value,code", [
    ("dtype", 7, 3), ("head_dim", 48, 1), ("feat_dim", 48, 1), ("n_q_heads", 12, 1),
    ("decode_interval", 70, 1), ("chunk", 0, 1), ("lambda_", -1, 1), ("window", -2, 1),
    ("max_prefill_tokens", 100, 1), ("eps", -1.0, 1), ("n_q_heads", 80, 1),
])
def test_config_validation(lib, field, value, code):
    cfg = L.config_from_workload(wl.WORKLOADS["prefill-1b"])
    setattr(cfg, field, value)
    n = ctypes.c_size_t(0)
    assert lib.lola_state_bytes(ctypes.byref(cfg), ctypes.byref(n)) == code


def test_null_arguments_rejected_without_device(lib):
    cfg = L.config_from_workload(wl.WORKLOADS["tiny"])
    h = ctypes.c_void_p(0)
    assert lib.lola_init_state(ctypes.byref(cfg), None, None, 0, None, ctypes.byref(h)) == 1
    assert lib.lola_prefill_chunk(None, None, None, None, 64, None, None) == 1
    assert lib.lola_decode_step(None, None, None, None, None, None) == 1
    assert lib.lola_sync(None, None) == 1
    assert lib.lola_set_prefill_schedule(None, 0, 0) == 1
    assert lib.lola_state_bytes(None, None) == 1
    assert lib.lola_position(None) == -1
    assert lib.lola_free_state(None) == 0


def test_status_strings(lib):
    for code in range(9):
        assert lib.lola_status_string(code)
    assert b"unknown" in lib.lola_status_string(99)


def test_workspace_checked_before_any_device_work(lib):
    # a misaligned or short workspace is refused before the library touches the device
    # (the pointers below are never dereferenced)
    cfg = L.config_from_workload(wl.WORKLOADS["prefill-1b"])
    need = ctypes.c_size_t(0)
    assert lib.lola_state_bytes(ctypes.byref(cfg), ctypes.byref(need)) == 0
    W = (ctypes.c_float * 4)()
    h = ctypes.c_void_p(0)
    misaligned = ctypes.c_void_p(0x100000 + 8)
    assert lib.lola_init_state(ctypes.byref(cfg), W, misaligned, need.value, None, ctypes.byref(h)) == 5
    aligned = ctypes.c_void_p(0x100000)
    assert lib.lola_init_state(ctypes.byref(cfg), W, aligned, need.value - 1, None, ctypes.byref(h)) == 5
    assert h.value is None


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_no_cache_config_is_sized(lib, dtype):
    # lambda = 0 (window + linear state only) is a valid configuration for both dtypes
    cfg = L.config_from_workload(wl.WORKLOADS["prefill-1b"])
    cfg.lambda_ = 0
    cfg.dtype = 0 if dtype == "f32" else 1
    n = ctypes.c_size_t(0)
    assert lib.lola_state_bytes(ctypes.byref(cfg), ctypes.byref(n)) == 0
    assert n.value > 0


def test_host_prefill_staging_bytes(lib):
    # two slots of q, k, v and out pieces, each rounded up to 256 bytes
    w = wl.WORKLOADS["prefill-8b"]
    cfg = L.config_from_workload(w, max_prefill_tokens=w.seq_len)
    piece = 4096
    e = 2
    q = w.batch * piece * w.n_q_heads * w.head_dim * e
    kv = w.batch * piece * w.n_kv_heads * w.head_dim * e
    up = lambda x: (x + 255) // 256 * 256
    assert L.lola_prefill_host_staging_bytes(cfg, piece) == 2 * (2 * up(q) + 2 * up(kv))
    n = ctypes.c_size_t(0)
    assert lib.lola_prefill_host_staging_bytes(ctypes.byref(cfg), 100, ctypes.byref(n)) == 2   # not a multiple of the chunk
    assert lib.lola_prefill_host_staging_bytes(ctypes.byref(cfg), 2 * w.seq_len, ctypes.byref(n)) == 5  # past max_prefill_tokens
    assert lib.lola_prefill_host(None, None, None, None, 64, None, None, 0, 64, None) == 1


def test_prefill_plan(lib):
    """The schedule each call gets (pure host): per-segment launches where the chain holds
    more than a third of a 148-SM device, one chain launch elsewhere; 16-interval segments,
    at least four of at least 8 intervals in a short call, at most 64 per call."""
    w8 = wl.WORKLOADS["prefill-8b"]         # 32 streams, chain on 64 SMs
    c8 = L.config_from_workload(w8, max_prefill_tokens=w8.seq_len)
    assert L.lola_prefill_plan(c8, w8.seq_len) == ("segments", 16, 16)
    assert L.lola_prefill_plan(c8, 2048) == ("segments", 8, 4)            # a 32-interval piece
    assert L.lola_prefill_plan(c8, 64) == ("segments", 1, 1)              # one interval
    assert L.lola_prefill_plan(c8, w8.seq_len, sms=256) == ("one-chain", 16, 16)
    assert L.lola_prefill_plan(c8, w8.seq_len, "one-chain", 1) == ("one-chain", 4, 64)   # at most 64
    assert L.lola_prefill_plan(c8, w8.seq_len, "segments", 3) == ("segments", 4, 64)
    assert L.lola_prefill_plan(c8, w8.seq_len, "segments", 100) == ("segments", 100, 3)
    wl_ = wl.WORKLOADS["long-context"]      # 8 streams, chain on 40 SMs, 512 intervals
    cl = L.config_from_workload(wl_, max_prefill_tokens=wl_.seq_len)
    assert L.lola_prefill_plan(cl, wl_.seq_len) == ("one-chain", 16, 32)
    assert L.lola_prefill_plan(cl, wl_.seq_len, "segments") == ("segments", 32, 16)
    w1 = wl.WORKLOADS["prefill-1b"]         # 8 streams, 64 intervals
    c1 = L.config_from_workload(w1, max_prefill_tokens=w1.seq_len)
    assert L.lola_prefill_plan(c1, w1.seq_len) == ("one-chain", 16, 4)
    # fp32 runs the SIMT chain and attention: one segment whatever the setting
    cf = L.config_from_workload(w1, max_prefill_tokens=w1.seq_len, dtype="f32")
    assert L.lola_prefill_plan(cf, w1.seq_len, "one-chain", 8) == ("segments", 64, 1)
    o = [ctypes.c_int32(0) for _ in range(3)]
    ref = [ctypes.byref(x) for x in o]
    assert lib.lola_prefill_plan(ctypes.byref(c8), 3, 0, 148, 64, *ref) == 1       # unknown mode
    assert lib.lola_prefill_plan(ctypes.byref(c8), 0, -1, 148, 64, *ref) == 1      # negative length
    assert lib.lola_prefill_plan(ctypes.byref(c8), 0, 0, 0, 64, *ref) == 1         # no SMs
    assert lib.lola_prefill_plan(ctypes.byref(c8), 0, 0, 148, 100, *ref) == 2      # not a multiple of chunk
    assert lib.lola_prefill_plan(ctypes.byref(c8), 0, 0, 148, 2 * w8.seq_len, *ref) == 5
    assert lib.lola_prefill_plan(ctypes.byref(c8), 0, 0, 148, 64, None, None, None) == 1
