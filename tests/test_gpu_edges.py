"""Edge cases of the CUDA path against the oracle: empty and ragged prefixes, sizes that are not
multiples of any tile, exact ties, the invariants of the method on the GPU, maximum sizes."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _clustered_small(L, T, H_I=64, seed=0, dtype="bf16", B=64):
    wl = W.small(2, L=L, n_seq=T, T=T, H_I=H_I, B=B, dtype=dtype, seed=1000 + seed)
    k, q, w, n, _ = W.decode_batch(wl)
    return wl, k, q, w


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_prefixes_shared_cache(dtype):
    """One shared cache of L = 3001 keys, prefixes 0, 1, 2, 15, 16, 17, 1000, 2999, 3001."""
    L_ = lib()
    wl = W.small(3, L=3001, T=3001, chunk=3001, dtype=dtype)
    k = W.shared_keys(wl)
    q, w = W.shared_queries(wl, 0, wl.T)
    ns = np.array([0, 1, 2, 15, 16, 17, 1000, 2999, 3001], np.int32)
    q, w = q[ns % wl.T], w[ns % wl.T]
    B, h, kk, kp = 64, 8, 256, 1024
    kd, qd, wd, nd = dev(k, DT[dtype]), dev(q, DT[dtype]), dev(w, torch.float32), dev(ns, torch.int32)
    kbar = L_.misa_pool_keys(kd, B)
    heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    o = oracle.get()
    orc = o.indexer(oracle.MODE_DAGGER, q, w, k, 0, ns, B, h, kk, kp=kp)
    rr, hh = host(r), host(heads)
    oh = dev(orc["heads"], torch.int32)
    cand, _ = L_.misa_score_topk(qd, wd, kd, nd, oh, kp)
    I_o = o.scores(q, w, k, 0, ns, heads=orc["heads"], ld=wl.L)
    fin, fv = L_.misa_hier_rerank(qd, wd, kd, nd, dev(orc["cand"], torch.int32), kk)
    dix, _ = L_.dsa_dense_topk(qd, wd, kd, nd, kk)
    od = o.indexer(oracle.MODE_DSA, q, w, k, 0, ns, B, h, kk)
    F = o.scores(q, w, k, 0, ns, ld=wl.L)
    cand, fin, dix = host(cand), host(fin), host(dix)
    for t, n in enumerate(ns.tolist()):
        if n == 0:
            assert np.all(cand[t] == -1) and np.all(fin[t] == -1) and np.all(dix[t] == -1)
            assert np.all(rr[t] == 0) and hh[t].tolist() == list(range(h))
            continue
        rt = P.router_tol(q[t], w[t], k, n, B)
        P.check_close(rr[t], orc["r"][t], rt, f"n={n} router")
        P.check_selection(hh[t], orc["heads"][t], orc["r"][t], rt, h, f"n={n} heads")
        st = P.score_tol(q[t], w[t], k, n, orc["heads"][t])
        P.check_selection(cand[t], orc["cand"][t], I_o[t][:n], st, kp, f"n={n} candidates")
        ft = P.score_tol(q[t], w[t], k, n, None)
        Fv = np.full(n, np.nan)
        c = orc["cand"][t][orc["cand"][t] >= 0]
        Fv[c] = F[t][c]
        P.check_selection(fin[t], orc["idx"][t], Fv, np.where(np.isnan(Fv), np.inf, ft), kk, f"n={n} re-rank")
        P.check_selection(dix[t], od["idx"][t], F[t][:n], ft, kk, f"n={n} dense")
        if n <= kk:
            assert sorted(dix[t][:n].tolist()) == list(range(n)) and np.all(dix[t][n:] == -1)
    # the standalone selection, on the scores and on rows whose boundary holds many exact ties
    # (the upper half of every row set to 0)
    I_gpu = L_.misa_token_scores(qd, wd, kd, nd, oh)
    zero = I_gpu.clone()
    zero[:, wl.L // 2:] = 0.0
    for rows in (I_gpu, zero):
        a, _ = L_.misa_topk_select(rows, nd, kk)
        vals = host(rows).astype(np.float64)
        for t, n in enumerate(ns.tolist()):
            want = np.argsort(-vals[t][:n], kind="stable")[:kk]
            got = host(a)[t]
            assert sorted(got[got >= 0].tolist()) == sorted(want.tolist()), f"n={n} select"


def test_full_routing_is_dense_on_gpu():
    """h = H_I: the routed path is the dense indexer, bit for bit (heads summed in the same order)."""
    L_ = lib()
    wl, k, q, w = _clustered_small(5000, 4, H_I=32)
    kd, qd, wd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32)
    nd = dev(np.array([5000, 4999, 1234, 77], np.int32), torch.int32)
    kbar = L_.misa_pool_keys(kd, 64)
    heads, _ = L_.misa_route(qd, wd, kd, kbar, nd, 64, 32)
    ia, va = L_.misa_score_topk(qd, wd, kd, nd, heads, 300)
    ib, vb = L_.dsa_dense_topk(qd, wd, kd, nd, 300)
    for t in range(4):
        oa, ob = np.argsort(host(ia)[t]), np.argsort(host(ib)[t])
        assert np.array_equal(host(ia)[t][oa], host(ib)[t][ob]) and np.array_equal(host(va)[t][oa], host(vb)[t][ob])
    sa = L_.misa_token_scores(qd, wd, kd, nd, heads)
    sb = L_.misa_token_scores(qd, wd, kd, nd, None)
    for t, n in enumerate([5000, 4999, 1234, 77]):
        assert torch.equal(sa[t, :n], sb[t, :n])


def test_dagger_with_all_candidates_is_dense():
    """k' >= n_t: MISA-dagger selects the dense indexer's tokens."""
    L_ = lib()
    wl, k, q, w = _clustered_small(3000, 3, H_I=64)
    kd, qd, wd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32)
    nd = dev(np.array([3000, 2500, 100], np.int32), torch.int32)
    res = L_.misa_indexer(qd, wd, kd, L_.misa_pool_keys(kd, 64), nd, 64, 8, 256, kp=4096)
    ib, vb = L_.dsa_dense_topk(qd, wd, kd, nd, 256)
    for t in range(3):
        assert set(host(res["idx"])[t].tolist()) == set(host(ib)[t].tolist())


def test_exact_ties_go_to_the_lower_index():
    """64 distinct key rows repeated 50 times: every score value appears 50 times, and the
    top-k boundary cuts through groups of equal scores."""
    L_ = lib()
    rng = np.random.default_rng(4)
    base = W.round_bf16(rng.standard_normal((64, 128)).astype(np.float32))
    k = np.tile(base, (50, 1))  # L = 3200
    q = W.round_bf16(rng.standard_normal((2, 16, 128)).astype(np.float32))
    w = (rng.standard_normal((2, 16)) / 4).astype(np.float32)
    n = np.array([3200, 3100], np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    o = oracle.get()
    for kk in (1, 75, 130, 1000):
        dix, _ = L_.dsa_dense_topk(qd, wd, kd, nd, kk)
        od = o.indexer(oracle.MODE_DSA, q, w, k, 0, n, 64, 16, kk)
        for t in range(2):
            assert set(host(dix)[t].tolist()) == set(od["idx"][t].tolist()), (kk, t)
    # re-rank with a shuffled candidate list that holds ties: the smaller token ids win
    cand = np.stack([rng.permutation(3200)[:2000] for _ in range(2)]).astype(np.int32)
    cand[:, ::97] = -1
    cand[1, 5] = 3150  # outside query 1's prefix: an empty slot
    fin, _ = L_.misa_hier_rerank(qd, wd, kd, nd, dev(cand, torch.int32), 333)
    for t in range(2):
        want, _ = o.rerank(q[t], w[t], k, int(n[t]), cand[t], 333)
        assert set(host(fin)[t].tolist()) == set(want.tolist())


def test_head_counts_not_multiple_of_eight_and_max_pool():
    """h = 5 of H_I = 16, and H_I = 128 with h = 8 and h = 128 (largest head pool)."""
    L_ = lib()
    o = oracle.get()
    for H_I, h in ((16, 5), (128, 8), (128, 128)):
        wl, k, q, w = _clustered_small(2100, 2, H_I=H_I, seed=H_I + h)
        n = np.array([2100, 2043], np.int32)
        kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
        heads, r = L_.misa_route(qd, wd, kd, L_.misa_pool_keys(kd, 64), nd, 64, h, want_r=True)
        orc = o.indexer(oracle.MODE_MISA, q, w, k, 2100 * 128, n, 64, h, 200)
        oh = dev(orc["heads"], torch.int32)
        idx, _ = L_.misa_score_topk(qd, wd, kd, nd, oh, 200)
        I_o = o.scores(q, w, k, 2100 * 128, n, heads=orc["heads"], ld=2100)
        for t in range(2):
            nt = int(n[t])
            rt = P.router_tol(q[t], w[t], k[t], nt, 64)
            P.check_selection(host(heads)[t], orc["heads"][t], orc["r"][t], rt, h, f"H_I={H_I} h={h} heads")
            st = P.score_tol(q[t], w[t], k[t], nt, orc["heads"][t])
            P.check_selection(host(idx)[t], orc["idx"][t], I_o[t][:nt], st, 200, f"H_I={H_I} h={h} top-k")


def test_largest_candidate_set():
    """k' = 16384 (the largest accepted) on a 40000-key cache."""
    L_ = lib()
    wl, k, q, w = _clustered_small(40000, 2, H_I=64, seed=9, B=128)
    n = np.array([40000, 39999], np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    res = L_.misa_indexer(qd, wd, kd, L_.misa_pool_keys(kd, 128), nd, 128, 8, 2048, kp=16384)
    o = oracle.get()
    orc = o.indexer(oracle.MODE_DAGGER, q, w, k, 40000 * 128, n, 128, 8, 2048, kp=16384)
    fin, _ = L_.misa_hier_rerank(qd, wd, kd, nd, dev(orc["cand"], torch.int32), 2048)
    F = o.dense_scores_at(q, w, k, 40000 * 128, n, orc["cand"])
    for t in range(2):
        nt = int(n[t])
        Fv = np.full(nt, np.nan)
        Fv[orc["cand"][t]] = F[t]
        ft = np.full(nt, np.inf)
        ft[orc["cand"][t]] = P.score_tol(q[t], w[t], k[t], nt, None)[orc["cand"][t]]
        P.check_selection(host(fin)[t], orc["idx"][t], Fv, ft, 2048, "k'=16384 re-rank")
        assert (host(res["cand"])[t] >= 0).sum() == 16384


def test_zero_queries_is_a_no_op():
    L_ = lib()
    q = torch.empty((0, 64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    n = torch.empty((0,), dtype=torch.int32, device="cuda")
    k = torch.zeros((100, 128), dtype=torch.bfloat16, device="cuda")
    kbar = L_.misa_pool_keys(k, 16)
    heads, _ = L_.misa_route(q, w, k, kbar, n, 16, 8)
    idx, _ = L_.misa_score_topk(q, w, k, n, heads, 10)
    assert heads.shape == (0, 8) and idx.shape == (0, 10)


def test_pool_block_range_and_repeatability():
    L_ = lib()
    wl, k, q, w = _clustered_small(4000, 2, H_I=64, seed=3)
    kd = dev(k, torch.bfloat16)
    full = L_.misa_pool_keys(kd, 128)
    part = torch.full_like(full, 7.0)
    L_.misa_pool_keys(kd, 128, kbar=part, block_begin=10, block_end=12)
    assert torch.equal(part[:, 10:12], full[:, 10:12])
    assert torch.all(part[:, :10] == 7.0) and torch.all(part[:, 12:] == 7.0)
    qd, wd = dev(q, torch.bfloat16), dev(w, torch.float32)
    nd = dev(np.array([4000, 3999], np.int32), torch.int32)
    a = L_.misa_indexer(qd, wd, kd, full, nd, 128, 8, 512, kp=1500)
    b = L_.misa_indexer(qd, wd, kd, full, nd, 128, 8, 512, kp=1500)
    assert torch.equal(a["heads"], b["heads"]), "routed heads differ between identical runs"
    for key in ("idx", "cand"):
        for t in range(2):  # the selected sets are reproducible; their order is not specified
            x, y = host(a[key])[t], host(b[key])[t]
            assert sorted(x.tolist()) == sorted(y.tolist()), f"{key} differs between identical runs"
    for t in range(2):
        oa, ob = np.argsort(host(a["idx"])[t]), np.argsort(host(b["idx"])[t])
        assert np.array_equal(host(a["vals"])[t][oa], host(b["vals"])[t][ob])


def test_prepared_selection_matches_score_topk():
    """misa_token_scores leaving the selection's first stage in a workspace, then
    misa_topk_select(ws_prepared) equals misa_score_topk and the plain selection, for per-query
    caches (the scoring kernel builds the stage) and a shared cache (a separate pass does)."""
    L_ = lib()
    wl, k, q, w = _clustered_small(20000, 6, H_I=64, seed=21, B=128)
    n = np.array([20000, 19999, 12345, 4097, 2048, 100], np.int32)
    for shared in (False, True):
        kk_ = k[0] if shared else k
        kd, qd = dev(kk_, torch.bfloat16), dev(q, torch.bfloat16)
        wd, nd = dev(w, torch.float32), dev(n, torch.int32)
        heads, _ = L_.misa_route(qd, wd, kd, L_.misa_pool_keys(kd, 128), nd, 128, 8)
        a, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, 3000)
        ws = L_.Workspace()
        scores = L_.misa_token_scores(qd, wd, kd, nd, heads, select_topk=3000, select_ws=ws)
        b, _ = L_.misa_topk_select(scores, nd, 3000, ws=ws, ws_prepared=True)
        c, _ = L_.misa_topk_select(scores, nd, 3000)
        for t in range(6):
            sa, sb, sc = (sorted(host(x)[t].tolist()) for x in (a, b, c))
            assert sa == sb == sc, (shared, t)
