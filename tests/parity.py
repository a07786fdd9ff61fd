"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare them.

Selection rule for comparisons (the top-lambda choice is a discrete decision
taken on floating-point SREs): where the oracle's lambda-th vs (lambda+1)-th
SRE margin exceeds 1e-3 relative, the GPU's kept set must equal the oracle's
exactly; under that margin the GPU's set must be a valid top-lambda within the
band (every token on which the two sets differ has an oracle SRE within 1e-3
relative of the oracle's lambda-th SRE) and the case is counted.
"""
from __future__ import annotations

import numpy as np

import oracle

MARGIN = 1e-3


def intervals_for(plan, chunk, decode_interval, pos0=0):
    """Interval lengths of a plan [("prefill", n) | ("decode", steps)], mirroring
    the engine: prefill runs n/chunk intervals; decode opens an interval of
    decode_interval steps whenever the position reaches the end of the last."""
    ints = []
    pos, iend = pos0, pos0
    for kind, n in plan:
        if kind == "prefill":
            assert pos == iend and n % chunk == 0
            ints += [chunk] * (n // chunk)
            pos += n
            iend = pos
        else:
            for _ in range(n):
                if pos == iend:
                    ints.append(decode_interval)
                    iend = pos + decode_interval
                pos += 1
    return ints


def override_from(r, lam, ns_gpu=None, stream_map=None):
    """Engine override buffer [n_int, ns_gpu, lam+1] from an oracle run. Streams
    the oracle did not run (subset runs) get count -1: not forced."""
    n_int, ns = r.nkept.shape
    ns_gpu = ns if ns_gpu is None else ns_gpu
    smap = list(range(ns)) if stream_map is None else stream_map
    buf = np.full((n_int, ns_gpu, lam + 1), -1, np.int32)
    for so, sg in enumerate(smap):
        buf[:, sg, 0] = r.nkept[:, so]
        if lam:
            buf[:, sg, 1:] = r.kept[:, so]
    return buf


def run_gpu(cfg, W, q, k, v, plan, override=None, log_cap=None, device="cuda"):
    """Runs the plan through the C ABI. q,k,v are float32 numpy arrays on the
    dtype grid, [B, T, H, d] with T = all prefill + decode tokens in order.
    Returns (out float32 [B, T, Hq, d], selection log or None)."""
    import torch
    from hybrid_linear_attention_lola_b200.lola import LolaState

    S = LolaState(cfg, torch.from_numpy(W), device)
    log = S.enable_selection_log(log_cap) if log_cap else None
    if override is not None:
        S.set_selection_override(torch.from_numpy(override))
    dt = S.dtype
    qd = torch.from_numpy(q).to(device=device, dtype=dt)
    kd = torch.from_numpy(k).to(device=device, dtype=dt)
    vd = torch.from_numpy(v).to(device=device, dtype=dt)
    outs = []
    t = 0
    for kind, n in plan:
        if kind == "prefill":
            o = S.prefill(qd[:, t:t + n].contiguous(), kd[:, t:t + n].contiguous(),
                          vd[:, t:t + n].contiguous())
            outs.append(o)
            t += n
        else:
            for _ in range(n):
                o = S.decode(qd[:, t].contiguous(), kd[:, t].contiguous(), vd[:, t].contiguous())
                outs.append(o[:, None])
                t += 1
    S.sync()
    out = torch.cat(outs, dim=1).float().cpu().numpy()
    lg = log.cpu().numpy() if log is not None else None
    S.close()
    return out, lg


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def compare_selections(gpu_log, r, lam, stream_map=None):
    """Returns (n_checked, n_exact, n_under_margin_diff, hard_mismatches list).
    stream_map: oracle stream index -> GPU stream index (subset runs)."""
    n_int, ns_o = r.nkept.shape
    checked = exact = under = 0
    hard = []
    for ci in range(n_int):
        for so in range(ns_o):
            sg = so if stream_map is None else stream_map[so]
            row = gpu_log[ci, sg]
            cnt = int(row[0])
            gset = set(int(x) for x in row[1:1 + cnt])
            oset = set(int(x) for x in r.kept[ci, so] if x >= 0) if lam else set()
            checked += 1
            if gset == oset and cnt == r.nkept[ci, so]:
                exact += 1
                continue
            m = r.margin[ci, so]
            if m > MARGIN or r.cand_sre is None:
                hard.append((ci, so, float(m), sorted(gset ^ oset)[:8]))
                continue
            toks = list(r.cand_tok[ci, so])
            sres = {int(t): float(s) for t, s in zip(toks, r.cand_sre[ci, so]) if t >= 0}
            ordered = sorted(sres.values(), reverse=True)
            s_lam = ordered[lam - 1]
            ok = len(gset) == len(oset) and all(
                t in sres and abs(sres[t] - s_lam) <= MARGIN * s_lam for t in gset ^ oset)
            if ok:
                under += 1
            else:
                hard.append((ci, so, float(m), sorted(gset ^ oset)[:8]))
    return checked, exact, under, hard
