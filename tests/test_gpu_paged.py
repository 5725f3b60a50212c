"""Paged key caches on the GPU.  The paged calls run the same arithmetic as the contiguous ones
(pooling and the router's partial-block mean sum rows in the same order; the scorer's gather path
multiplies the same rows with the same fragments), so their results must equal the contiguous
path's bit for bit on the same logical caches.  The final selections are also checked against the
oracle, which reads the pool through its own page-table gather."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _paged_layout(k, ns, page_size, seed, share_prefix_pages=0, spare=7):
    """Scatter contiguous caches k [T, L, d] into a shuffled pool; sequences 0 and 1 share their
    first `share_prefix_pages` pages (k[1] must equal k[0] there)."""
    g = np.random.default_rng(seed)
    T, L, d = k.shape
    lp = -(-L // page_size)
    num_pages = T * lp + spare
    perm = g.permutation(num_pages)
    pool = g.standard_normal((num_pages, page_size, d)).astype(np.float32)  # spare pages hold junk
    table = np.full((T, lp + 1), -1, np.int32)
    padded = np.zeros((T, lp * page_size, d), np.float32)
    padded[:, :L] = k
    for t in range(T):
        for p in range(lp):
            if t == 1 and p < share_prefix_pages:
                table[t, p] = table[0, p]
                continue
            table[t, p] = perm[t * lp + p]
            pool[table[t, p]] = padded[t, p * page_size:(p + 1) * page_size]
        table[t, -(-int(ns[t]) // page_size):] = -1 if t % 2 else num_pages + 5  # never read
    return pool, table


@pytest.mark.parametrize("page_size,ns", [
    (64, [8192, 8192, 8000, 5001]),
    (16, [8192, 8191, 777, 1]),
    (100, [8192, 3000, 8100, 0]),   # pages that do not divide B
])
def test_paged_equals_contiguous(page_size, ns):
    L_ = lib()
    wl = W.small(4, L=8192, n_seq=4, T=4, seed=300 + page_size)
    k, q, w, _, _ = W.decode_batch(wl)
    ns = np.array(ns, np.int32)
    k[1, :3 * page_size] = k[0, :3 * page_size]
    kb = k.astype(np.float32)
    kb = torch.from_numpy(kb).to(torch.bfloat16).float().numpy()  # the values the GPU holds
    pool, table = _paged_layout(kb, ns, page_size, seed=page_size, share_prefix_pages=3)
    B, h, kk, kp = wl.B, wl.h, 512, 2048
    kd, qd, wd, nd = dev(kb, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(ns, torch.int32)
    pd, td = dev(pool, torch.bfloat16), dev(table, torch.int32)

    kbar = L_.misa_pool_keys(kd, B)
    kbar_p = L_.misa_pool_keys_paged(pd, td, B, L=wl.L)
    for t in range(4):  # blocks inside the prefix (pages past it are not in the table)
        nb = int(ns[t]) // B
        assert torch.equal(kbar[t, :nb], kbar_p[t, :nb]), f"q{t}: pooled keys differ"
    heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    heads_p, r_p = L_.misa_route_paged(qd, wd, pd, td, kbar_p, nd, B, h, L=wl.L, want_r=True)
    assert torch.equal(r, r_p) and torch.equal(heads, heads_p), "router differs"
    cand, cv = L_.misa_score_topk(qd, wd, kd, nd, heads, kp)
    cand_p, cv_p = L_.misa_score_topk_paged(qd, wd, pd, td, nd, heads, kp, L=wl.L)
    for t in range(4):
        a, b = host(cand)[t], host(cand_p)[t]
        assert sorted(a.tolist()) == sorted(b.tolist()), f"q{t}: candidates differ"
        assert sorted(host(cv)[t].tolist()) == sorted(host(cv_p)[t].tolist()), f"q{t}: candidate scores differ"
    fin, fv = L_.misa_hier_rerank(qd, wd, kd, nd, cand, kk)
    fin_p, fv_p = L_.misa_hier_rerank_paged(qd, wd, pd, td, nd, cand, kk, L=wl.L)
    for t in range(4):
        assert sorted(host(fin)[t].tolist()) == sorted(host(fin_p)[t].tolist()), f"q{t}: re-rank differs"
    L_.misa_device_check()

    # against the oracle, which gathers the logical caches through the table itself
    o = oracle.get()
    logical = o.paged_caches(pool, table, ns, wl.L)
    orc = o.indexer(oracle.MODE_DAGGER, q, w, logical, wl.L * 128, ns, B, h, kk, kp=kp)
    F = o.scores(q, w, logical, wl.L * 128, ns, ld=wl.L)
    hp = host(heads_p)
    for t in range(4):
        nt = int(ns[t])
        if nt == 0:
            assert np.all(host(fin_p)[t] == -1)
            continue
        rt = P.router_tol(q[t], w[t], logical[t], nt, B)
        P.check_selection(hp[t], orc["heads"][t], orc["r"][t], rt, h, f"paged q{t} heads")
        if set(hp[t].tolist()) != set(orc["heads"][t].tolist()):
            continue
        I = o.scores(q[t:t + 1], w[t:t + 1], logical[t], 0, ns[t:t + 1], heads=orc["heads"][t:t + 1], ld=nt)[0]
        st = P.score_tol(q[t], w[t], logical[t], nt, orc["heads"][t])
        P.check_selection(host(cand_p)[t], orc["cand"][t], I, st, kp, f"paged q{t} candidates")
        if set(host(cand_p)[t].tolist()) == set(orc["cand"][t].tolist()):
            c = orc["cand"][t][orc["cand"][t] >= 0]
            Fv = np.full(nt, np.nan)
            Fv[c] = F[t][c]
            ft = np.full(nt, np.inf)
            ft[c] = P.score_tol(q[t], w[t], logical[t], nt, None)[c]
            P.check_selection(host(fin_p)[t], orc["idx"][t], Fv, ft, kk, f"paged q{t} final")
