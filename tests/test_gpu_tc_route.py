"""Tensor-core router of queries that share one bf16 key cache (chunked prefill) against the
oracle: router scores within the router tolerance, routed head sets equal up to the tie band.

Covers several head counts (8, 32, 64, 128 query-head rows per query block of 128 rows), block
sizes, prefixes that end on, just before and just after a block boundary, empty and one-key
prefixes, L not a multiple of B, query counts that leave a partial query block, and a call the
host splits into two launches."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(L, T, H_I, B, seed):
    wl = W.small(3, L=L, T=T, chunk=T, H_I=H_I, B=B, dtype="bf16", seed=7000 + seed)
    k = W.shared_keys(wl)
    q, w = W.shared_queries(wl, 0, T)
    g = np.random.default_rng(seed)
    n = g.integers(0, L + 1, size=T).astype(np.int32)
    edge = [0, 1, B - 1, B, B + 1, 2 * B, 2 * B + 1, L - 1, L, 255 * B, 256 * B, 257 * B + 3]
    edge = [x for x in edge if 0 <= x <= L]
    n[: len(edge)] = edge
    return k, q, w, n


def _check(L_, k, q, w, n, B, h, rows=None):
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    kbar = L_.misa_pool_keys(kd, B)
    heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    hh, rr = host(heads), host(r)
    rows = range(q.shape[0]) if rows is None else rows
    sel = np.asarray(list(rows))
    o_r, o_h = oracle.get().route_batch(q[sel], w[sel], k, 0, n[sel], B, h)
    for i, t in enumerate(sel.tolist()):
        nt = int(n[t])
        if nt == 0:
            assert np.all(rr[t] == 0) and hh[t].tolist() == list(range(h)), f"t={t}: empty prefix"
            continue
        tol = P.router_tol(q[t], w[t], k, nt, B)
        P.check_close(rr[t], o_r[i], tol, f"t={t} n={nt} router")
        P.check_selection(hh[t], o_h[i], o_r[i], tol, h, f"t={t} n={nt} heads")
    L_.misa_device_check()


@pytest.mark.parametrize("L,T,H_I,B,h", [
    (70000, 96, 64, 128, 8),    # 2 queries per block; up to 547 pooled blocks (3 tiles)
    (5000, 100, 32, 64, 8),     # 4 queries per block
    (3001, 70, 128, 16, 16),    # 1 query per block, 188 pooled blocks
    (2000, 130, 16, 256, 4),    # 8 queries per block, 8 pooled blocks
    (1500, 65, 8, 7, 3),        # 16 queries per block, B not a power of two
])
def test_shared_cache_router_matches_the_oracle(L, T, H_I, B, h):
    L_ = lib()
    k, q, w, n = _case(L, T, H_I, B, seed=L + T)
    _check(L_, k, q, w, n, B, h)


def test_router_call_split_over_launches():
    """64 heads: 2 queries per block and at most 8192 queries per launch: 8200 queries take two."""
    L_ = lib()
    L, T, H_I, B = 1000, 8200, 64, 64
    k, q, w, n = _case(L, T, H_I, B, seed=3)
    g = np.random.default_rng(5)
    rows = sorted(set(range(0, 30)) | set(range(8180, 8200)) | set(g.choice(T, 50, replace=False).tolist()))
    _check(L_, k, q, w, n, B, 8, rows)
