"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances (derived from the arithmetic; the target is 1e-3 relative for fp32 accumulation):
  * token / dense score of key s with head set R:
        |gpu - oracle| <= 1e-3 * A_s + 1e-5 * Abar_s
    A_s    = sum_{j in R} |w_j| |q_j . k_s|        (size of the terms actually summed)
    Abar_s = sum_{j in R} |w_j| |q_j| |k_s|        (floor for A_s ~ 0; fp32 dot products of 128
             terms err by at most ~128 * 2^-24 * sum_i |q_i k_i| <= 7.6e-6 * |q| |k|)
  * router score of head j over blocks b:
        |gpu - oracle| <= |w_j| (1e-3 * sum_b |q_j . kbar_b| + 1e-5 * |q_j| sum_b mean_{s in b} |k_s|)
    (the block means are fp32 sums of up to B keys, whose rounding scales with the keys, not
    with their mean)
  * block means: |gpu - oracle| <= 2 c 2^-24 mean_{s}|k_{s,i}| + 2^-23 |oracle|  (c keys summed)
  * block-filter score of block b with head set R (block mean of c keys):
        |gpu - oracle| <= 1e-3 * sum_{j in R} |w_j| |q_j . kbar_b|
                          + (1e-5 + 2 c 2^-24) * sum_{j in R} |w_j| |q_j| mean_{s in b} |k_s|
    (the fp32 mean errs by up to 2 c 2^-24 of the mean key size, so its dot product with q_j by
    that much of |q_j| mean |k_s|; the dot product itself by the same floor as a token score)
Selections (top-h heads, top-k tokens): tau is the oracle's k-th value; the tie band is every item
whose oracle value is within tol_item + tol_tau of tau.  The GPU set must have the right size, no
duplicates, only valid ids; every oracle item outside the band must be in the GPU set and every
GPU item outside the band must be in the oracle set.  Items swapped inside the band are counted.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

SCORE_REL = 1e-3
SCORE_FLOOR = 1e-5


def score_tol(q, w, k, n, heads=None):
    """Per-key tolerance [n] of one query's score with the given heads (None = all heads)."""
    q = np.asarray(q, np.float64)
    w = np.asarray(w, np.float64)
    hs = np.arange(q.shape[0]) if heads is None else np.asarray(heads)
    K = np.asarray(k[:n], np.float64)
    Q = q[hs]
    W = np.abs(w[hs])
    D = Q @ K.T
    A = W @ np.abs(D)
    Abar = (W * np.linalg.norm(Q, axis=1)).sum() * np.linalg.norm(K, axis=1)
    return SCORE_REL * A + SCORE_FLOOR * Abar


def router_tol(q, w, k, n, B):
    q = np.asarray(q, np.float64)
    w = np.asarray(w, np.float64)
    K = np.asarray(k[:n], np.float64)
    M = -(-n // B)
    if M == 0:
        return np.zeros(q.shape[0])
    means = np.stack([K[b * B:min((b + 1) * B, n)].mean(axis=0) for b in range(M)])
    norms = np.linalg.norm(K, axis=1)
    mean_norm = np.array([norms[b * B:min((b + 1) * B, n)].mean() for b in range(M)])
    D = q @ means.T
    return np.abs(w) * (SCORE_REL * np.abs(D).sum(axis=1) + SCORE_FLOOR * np.linalg.norm(q, axis=1) * mean_norm.sum())


def block_tol(q, w, k, n, B, heads):
    """Per-block tolerance [ceil(n/B)] of one query's block-filter scores with the given heads."""
    q = np.asarray(q, np.float64)
    w = np.asarray(w, np.float64)
    K = np.asarray(k[:n], np.float64)
    M = -(-n // B)
    if M == 0:
        return np.zeros(0)
    hs = np.asarray(heads)
    Q = q[hs]
    W = np.abs(w[hs])
    means = np.stack([K[b * B:min((b + 1) * B, n)].mean(axis=0) for b in range(M)])
    norms = np.linalg.norm(K, axis=1)
    mean_norm = np.array([norms[b * B:min((b + 1) * B, n)].mean() for b in range(M)])
    count = np.array([min((b + 1) * B, n) - b * B for b in range(M)], np.float64)
    A = W @ np.abs(Q @ means.T)
    floor = (SCORE_FLOOR + 2 * count * 2.0 ** -24) * (W * np.linalg.norm(Q, axis=1)).sum() * mean_norm
    return SCORE_REL * A + floor


def pool_tol(k, n, B, kbar_oracle):
    K = np.abs(np.asarray(k[:n], np.float64))
    M = -(-n // B)
    out = np.empty_like(kbar_oracle)
    for b in range(M):
        blk = K[b * B:min((b + 1) * B, n)]
        c = blk.shape[0]
        out[b] = 2 * c * 2.0 ** -24 * blk.mean(axis=0) + 2.0 ** -23 * np.abs(kbar_oracle[b])
    return out


@dataclass
class SelectionReport:
    swaps: int = 0
    band: int = 0


def check_selection(gpu_ids, ora_ids, values, tol, kk, what=""):
    """Compare one selection.  values/tol are indexed by id (oracle values of every candidate)."""
    gpu_ids = np.asarray(gpu_ids)
    ora_ids = np.asarray(ora_ids)
    g = gpu_ids[gpu_ids >= 0]
    o = ora_ids[ora_ids >= 0]
    assert np.all(gpu_ids[len(g):] == -1), f"{what}: -1 padding must come last"
    assert len(g) == len(o), f"{what}: size {len(g)} != oracle {len(o)}"
    assert len(np.unique(g)) == len(g), f"{what}: duplicate ids"
    gs, os_ = set(g.tolist()), set(o.tolist())
    rep = SelectionReport()
    if gs == os_:
        return rep
    assert all(0 <= x < len(values) for x in gs), f"{what}: id out of range"
    # tau: the oracle's last selected value (the selection is sorted by value desc in the oracle)
    tau_id = int(o[-1])
    tau = values[tau_id]
    lim = tol + tol[tau_id]
    inband = lambda x: abs(values[x] - tau) <= lim[x]
    bad_o = [x for x in os_ - gs if not inband(x)]
    bad_g = [x for x in gs - os_ if not inband(x)]
    assert not bad_o, f"{what}: oracle picks {bad_o[:5]} missing on the GPU (values {[values[x] for x in bad_o[:5]]}, tau {tau})"
    assert not bad_g, f"{what}: GPU picks {bad_g[:5]} outside the oracle set (values {[values[x] for x in bad_g[:5]]}, tau {tau})"
    rep.swaps = len(gs - os_)
    rep.band = int(sum(inband(x) for x in range(len(values)) if np.isfinite(values[x])))
    return rep


def check_close(gpu, ora, tol, what=""):
    gpu = np.asarray(gpu, np.float64)
    ora = np.asarray(ora, np.float64)
    err = np.abs(gpu - ora)
    bad = np.nonzero(~(err <= tol))[0]
    assert bad.size == 0, (f"{what}: {bad.size} values out of tolerance; first at {bad[:5]}: gpu {gpu[bad[:5]]} "
                           f"oracle {ora[bad[:5]]} tol {np.asarray(tol)[bad[:5]]}")
    return float(np.max(err / np.maximum(tol, 1e-300))) if err.size else 0.0
