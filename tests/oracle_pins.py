"""Pins for the CPU oracle: checks that tie it to something other than itself.

Each ``check_*`` takes an ``oracle.Oracle`` and raises AssertionError on a mismatch.  The test
module runs them on the real oracle (all must pass); the mutation test runs them on copies of
the oracle with one plausible mistake planted (each copy must fail at least one).

What pins what (definitions from "MISA: Mixture of Indexer Sparse Attention for Long-Context
LLM Inference", gist.science/paper/2605.07363, "Methodology: MISA" and "Hierarchical Variant"):
  * hand-computed fixture (tests/golden/hand_example.json): block means, router scores, routed
    heads, token scores, top-k with exact ties, dense scores, MISA-dagger;
  * special cases that reduce to numpy routines: B = 1 pools to the keys themselves, B >= n
    pools to ``numpy.mean``; top-k equals a stable ``numpy.argsort``;
  * brute force on tiny integer inputs: the routed set by enumerating every h-subset;
  * exact invariants: scaling q, k or w by 2 scales every score by 2 and keeps every selection;
    relabelling heads permutes the router scores; h = H_I is the dense indexer bit for bit;
    k' >= n makes MISA-dagger the dense indexer, k' = k makes it MISA, and the dense top-k
    restricted to the candidates is always kept; keys past a query's prefix change nothing;
  * a planted needle (the tiny fp32 workload) is routed and selected;
  * the block filter composed with MISA ("HISA: Efficient Hierarchical Indexing for Fine-Grained
    Sparse Attention", abstract): hand-derived cases, every block kept is MISA, B = 1 turns block
    scores into token scores, block scores sum to the routed heads' router scores, and the
    selection is MISA's top-k restricted to the kept blocks;
  * paged key caches: a shuffled pool built page by page with numpy, shared prefix pages and
    unused table entries gather back to the contiguous caches, and every indexer agrees bit for bit.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

from long_context_sparse_mean_b200 import workloads as wlmod

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_example.json")


def _load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


def check_hand_example(o):
    g = _load_golden()
    k = np.array(g["keys"], np.float32)
    q = np.array(g["q"], np.float32)
    w = np.array(g["w"], np.float32)
    B = g["B"]
    for qc in g["queries"]:
        n = qc["n"]
        assert np.array_equal(o.pool_keys(k, B, n), np.array(qc["kbar"], np.float64)), "block means"
        r, heads = o.route(q, w, k, n, B, 1)
        assert np.array_equal(r, np.array(qc["r"], np.float64)), f"router scores n={n}: {r}"
        assert list(heads) == qc["h1"]["heads"], f"routed head n={n}: {heads}"
        I = o.token_scores(q, w, heads, k, n)
        assert np.array_equal(I, np.array(qc["h1"]["I"], np.float64)), f"token scores h=1 n={n}: {I}"
        top, _ = o.topk(I, 2)
        assert list(top) == qc["h1"]["top2"], f"top-2 h=1 n={n}: {top}"
        if "h2" in qc:
            _, heads2 = o.route(q, w, k, n, B, 2)
            assert list(heads2) == qc["h2"]["heads"], heads2
            I2 = o.token_scores(q, w, heads2, k, n)
            assert np.array_equal(I2, np.array(qc["h2"]["I"], np.float64)), I2
            assert list(o.topk(I2, 2)[0]) == qc["h2"]["top2"]
            assert list(o.topk(I2, 4)[0]) == qc["h2"]["top4"]
            F = o.token_scores(q, w, np.arange(3), k, n)
            assert np.array_equal(F, np.array(qc["dense"]["F"], np.float64)), F
            for kk, key in ((2, "top2"), (4, "top4")):
                dsa = o.indexer(2, q[None], w[None], k, 0, np.array([n]), B, 3, kk)
                assert list(dsa["idx"][0]) == qc["dense"][key], dsa["idx"]
            dag = o.indexer(1, q[None], w[None], k, 0, np.array([n]), B, 1, 2, kp=3)
            assert list(dag["cand"][0]) == qc["dagger_h1_kp3"]["cand"], dag["cand"]
            assert sorted(dag["idx"][0]) == sorted(qc["dagger_h1_kp3"]["top2"]), dag["idx"]


def check_topk_vs_stable_argsort(o):
    rng = np.random.default_rng(7)
    for n, k in ((1, 1), (10, 3), (257, 64), (1000, 999), (50, 80)):
        v = rng.integers(-5, 6, size=n).astype(np.float64)  # many exact ties
        ids, vals = o.topk(v, k)
        ref = np.argsort(-v, kind="stable")[:k]
        m = min(n, k)
        assert np.array_equal(ids[:m], ref[:m]), (n, k)
        assert np.all(ids[m:] == -1)
        assert np.array_equal(vals[:m], v[ref[:m]])


def check_topk_with_ids(o):
    rng = np.random.default_rng(8)
    v = rng.integers(0, 4, size=40).astype(np.float64)
    ids = rng.permutation(1000)[:40].astype(np.int32)
    ids[::7] = -1  # empty slots are skipped
    got, _ = o.topk(v, 12, ids)
    # brute force: rank every valid item by (value desc, id asc) by counting the items it loses to
    valid = [a for a in range(40) if ids[a] >= 0]
    want = [ids[a] for a in valid
            if sum((v[b] > v[a]) or (v[b] == v[a] and ids[b] < ids[a]) for b in valid) < 12]
    assert sorted(got.tolist()) == sorted(want)


def check_pool_special_cases(o):
    rng = np.random.default_rng(9)
    k = rng.standard_normal((37, 16)).astype(np.float32)
    assert np.array_equal(o.pool_keys(k, 1), k.astype(np.float64)), "B = 1 pools to the keys"
    for B in (37, 64):
        got = o.pool_keys(k, B)
        assert got.shape == (1, 16)
        assert np.allclose(got[0], k.astype(np.float64).mean(axis=0), rtol=1e-14, atol=1e-15)
    kc = np.tile(np.array([0.5, -2.0, 3.0, 0.0], np.float32), (10, 1))
    assert np.array_equal(o.pool_keys(kc, 4), np.tile(kc[0].astype(np.float64), (3, 1)))
    full = o.pool_keys(k, 8)  # 4 full blocks and one of 5 keys
    k64 = k.astype(np.float64)
    assert np.allclose(full[:4], k64[:32].reshape(4, 8, 16).mean(axis=1), rtol=1e-14, atol=1e-15)
    assert np.allclose(full[4], k64[32:].mean(axis=0), rtol=1e-14, atol=1e-15)


def _np_router_scores(q, w, k, n, B):
    q, w, k = (np.asarray(a, np.float64) for a in (q, w, k))
    M = -(-n // B)
    means = np.stack([k[b * B:min((b + 1) * B, n)].mean(axis=0) for b in range(M)])
    return w * np.maximum(q @ means.T, 0.0).sum(axis=1)


def _brute_top_set(vals, h):
    """The h-subset whose every member beats every non-member (value desc, index asc)."""
    H = len(vals)
    for S in itertools.combinations(range(H), h):
        if all((vals[a] > vals[b]) or (vals[a] == vals[b] and a < b)
               for a in S for b in range(H) if b not in S):
            return set(S)
    raise AssertionError("no consistent subset")


def check_router_bruteforce(o):
    rng = np.random.default_rng(10)
    for trial in range(30):
        H_I, d = 4, 4
        L = int(rng.integers(1, 11))
        B = int(rng.integers(1, 5))
        h = int(rng.integers(1, H_I + 1))
        q = rng.integers(-3, 4, size=(H_I, d)).astype(np.float32)
        w = rng.integers(-2, 3, size=H_I).astype(np.float32)
        k = rng.integers(-3, 4, size=(L, d)).astype(np.float32)
        n = int(rng.integers(0, L + 1))
        r, heads = o.route(q, w, k, n, B, h)
        if n > 0:
            assert np.allclose(r, _np_router_scores(q, w, k, n, B), rtol=1e-12, atol=1e-12), trial
        else:
            assert np.all(r == 0.0)
        assert set(heads.tolist()) == _brute_top_set(r, h), (trial, r, heads)
        assert all(r[heads[a]] >= r[heads[a + 1]] for a in range(h - 1)), "heads by descending r"


def check_scores_bruteforce(o):
    rng = np.random.default_rng(11)
    for trial in range(20):
        H_I, d, n = 5, 3, int(rng.integers(1, 9))
        q = rng.integers(-3, 4, size=(H_I, d)).astype(np.float32)
        w = rng.integers(-2, 3, size=H_I).astype(np.float32)
        k = rng.integers(-3, 4, size=(n, d)).astype(np.float32)
        heads = rng.permutation(H_I)[: int(rng.integers(1, H_I + 1))]
        I = o.token_scores(q, w, heads, k, n)
        for s in range(n):
            want = 0.0
            for j in sorted(heads):
                dot = sum(float(q[j, i]) * float(k[s, i]) for i in range(d))
                want += float(w[j]) * max(dot, 0.0)
            assert I[s] == want, (trial, s, I[s], want)


def _small_clustered(seed=0, H_I=8, d=16, L=300):
    rng = np.random.default_rng(100 + seed)
    k = rng.standard_normal((L, d)).astype(np.float32)
    q = rng.standard_normal((H_I, d)).astype(np.float32)
    w = (rng.standard_normal(H_I) / math.sqrt(H_I)).astype(np.float32)
    return q, w, k


def check_scaling(o):
    q, w, k = _small_clustered(1)
    n, B, h = 250, 16, 3
    r, heads = o.route(q, w, k, n, B, h)
    I = o.token_scores(q, w, heads, k, n)
    top = o.topk(I, 20)[0]
    for name, (q2, w2, k2) in {"k": (q, w, 2 * k), "q": (2 * q, w, k), "w": (q, 2 * w, k)}.items():
        r2, heads2 = o.route(q2, w2, k2, n, B, h)
        assert np.array_equal(r2, 2 * r), f"router scores scale with {name}"
        assert np.array_equal(heads2, heads), f"routing unchanged under scaling of {name}"
        I2 = o.token_scores(q2, w2, heads2, k2, n)
        assert np.array_equal(I2, 2 * I), f"token scores scale with {name}"
        assert np.array_equal(o.topk(I2, 20)[0], top)


def check_head_permutation(o):
    q, w, k = _small_clustered(2)
    n, B, h = 300, 32, 4
    r, heads = o.route(q, w, k, n, B, h)
    perm = np.random.default_rng(3).permutation(q.shape[0])
    r2, heads2 = o.route(q[perm], w[perm], k, n, B, h)
    assert np.array_equal(r2, r[perm]), "router scores follow the head labels"
    assert set(perm[heads2].tolist()) == set(heads.tolist())


def check_full_routing_is_dense(o):
    q, w, k = _small_clustered(3)
    n = np.array([300, 123, 7], np.int32)
    Q = np.stack([q, q[::-1], q * 0.5])
    W = np.stack([w, -w, w])
    H_I = q.shape[0]
    for kk in (1, 10, 64):
        m = o.indexer(0, Q, W, k, 0, n, 16, H_I, kk)
        dd = o.indexer(2, Q, W, k, 0, n, 16, H_I, kk)
        assert np.array_equal(m["idx"], dd["idx"]), "h = H_I reproduces the dense indexer"
        assert np.array_equal(m["idx_v"], dd["idx_v"]), "bit-identical scores"


def check_dagger_invariants(o):
    q, w, k = _small_clustered(4, H_I=8, d=16, L=400)
    Q = np.stack([q, q[::-1]])
    W = np.stack([w, w[::-1]])
    n = np.array([400, 333], np.int32)
    B, h, kk = 25, 2, 16
    dsa = o.indexer(2, Q, W, k, 0, n, B, h, kk)
    misa = o.indexer(0, Q, W, k, 0, n, B, h, kk)
    full = o.indexer(1, Q, W, k, 0, n, B, h, kk, kp=400)
    assert np.array_equal(full["idx"], dsa["idx"]), "k' >= n makes MISA-dagger the dense indexer"
    same = o.indexer(1, Q, W, k, 0, n, B, h, kk, kp=kk)
    for t in range(2):
        assert set(same["idx"][t]) == set(misa["idx"][t]), "k' = k makes MISA-dagger MISA"
    prev = -1
    for kp in (16, 32, 64, 128, 256, 400):
        dag = o.indexer(1, Q, W, k, 0, n, B, h, kk, kp=kp)
        rec = 0
        for t in range(2):
            C = set(dag["cand"][t]) - {-1}
            S = set(dag["idx"][t]) - {-1}
            D = set(dsa["idx"][t]) - {-1}
            assert (D & C) <= S, "dense top-k tokens inside the candidate set are kept"
            rec += len(D & S)
        assert rec >= prev, "recovery does not drop as k' grows"
        prev = rec


def check_prefix_only(o):
    q, w, k = _small_clustered(5)
    n, B, h = 201, 16, 3
    k2 = k.copy()
    k2[n:] = 1000.0 * np.sign(k2[n:]) + 3.0
    a = o.indexer(1, q[None], w[None], k, 0, np.array([n]), B, h, 20, kp=60)
    b = o.indexer(1, q[None], w[None], k2, 0, np.array([n]), B, h, 20, kp=60)
    for key in ("r", "heads", "cand", "idx", "idx_v"):
        assert np.array_equal(a[key], b[key]), f"keys past the prefix changed {key}"
    assert a["idx"].max() < n and a["cand"].max() < n


def check_empty_and_short(o):
    q, w, k = _small_clustered(6)
    H_I = q.shape[0]
    e = o.indexer(1, q[None], w[None], k, 0, np.array([0]), 16, 3, 5, kp=9)
    assert np.all(e["idx"] == -1) and np.all(e["cand"] == -1), "empty prefix selects nothing"
    assert list(e["heads"][0]) == [0, 1, 2], "all router scores tie at 0 -> lowest heads"
    s = o.indexer(0, q[None], w[None], k, 0, np.array([3]), 16, 3, 5)
    assert sorted(s["idx"][0][:3]) == [0, 1, 2] and list(s["idx"][0][3:]) == [-1, -1]
    d = o.indexer(2, q[None], w[None], k, 0, np.array([3]), 16, H_I, 5)
    assert sorted(d["idx"][0][:3]) == [0, 1, 2] and list(d["idx"][0][3:]) == [-1, -1]


def check_negative_weight_sign(o):
    q, w, k = _small_clustered(7)
    w = np.abs(w)
    w[[1, 4]] *= -1.0  # signed weights: a negative head scores <= 0 on the router
    r, heads = o.route(q, w, k, 300, 16, 4)
    assert r[1] <= 0 and r[4] <= 0
    assert 1 not in heads and 4 not in heads


def check_planted_needles(o):
    wl = wlmod.WORKLOADS[1]
    inp = wlmod.shared_inputs(wl)
    res = o.indexer(1, inp.q, inp.w, inp.k, 0, inp.n, wl.B, wl.h, wl.topk, kp=4 * wl.topk)
    dsa = o.indexer(2, inp.q, inp.w, inp.k, 0, inp.n, wl.B, wl.h, wl.topk)
    misa = o.indexer(0, inp.q, inp.w, inp.k, 0, inp.n, wl.B, wl.h, wl.topk)
    for t in range(wl.T):
        assert set(inp.needle_heads.tolist()) <= set(res["heads"][t].tolist()), "needle heads routed"
        for out in (res, dsa, misa):
            assert set(inp.needle_pos.tolist()) <= set(out["idx"][t].tolist()), "needle tokens selected"


def check_batch_matches_single_query(o):
    """The batched drivers (router, scores, MISA, MISA-dagger, dense scores of listed tokens,
    pooling) give per query exactly what the single-query functions give (which the brute-force
    pins cover), for one shared cache with a different prefix per query and for one cache per
    query."""
    rng = np.random.default_rng(12)
    T, H_I, d, L, B, h, kk, kp = 6, 8, 16, 90, 7, 3, 10, 25
    q = rng.integers(-3, 4, size=(T, H_I, d)).astype(np.float32)
    w = rng.integers(-2, 3, size=(T, H_I)).astype(np.float32)
    shared = rng.integers(-3, 4, size=(L, d)).astype(np.float32)
    caches = rng.integers(-3, 4, size=(T, L, d)).astype(np.float32)
    n = np.array([0, 1, 6, 7, 50, 90], np.int32)
    for k, kss, kt in ((shared, 0, lambda t: shared), (caches, L * d, lambda t: caches[t])):
        r_b, h_b = o.route_batch(q, w, k, kss, n, B, h)
        I_b = o.scores(q, w, k, kss, n, heads=h_b, ld=L)
        misa = o.indexer(0, q, w, k, kss, n, B, h, kk)
        dag = o.indexer(1, q, w, k, kss, n, B, h, kk, kp=kp)
        ids = rng.integers(-2, L + 2, size=(T, 12)).astype(np.int32)
        F_b = o.dense_scores_at(q, w, k, kss, n, ids)
        for t in range(T):
            nt = int(n[t])
            r1, h1 = o.route(q[t], w[t], kt(t), nt, B, h)
            assert np.array_equal(r_b[t], r1) and np.array_equal(h_b[t], h1), ("router", kss, t)
            assert np.array_equal(misa["heads"][t], h1) and np.array_equal(misa["r"][t], r1), ("indexer r", kss, t)
            I1 = o.token_scores(q[t], w[t], h1, kt(t), nt)
            assert np.array_equal(I_b[t][:nt], I1) and np.all(np.isnan(I_b[t][nt:])), ("scores", kss, t)
            sel, _ = o.topk(I1, kk)
            assert np.array_equal(misa["idx"][t], sel), ("MISA top-k", kss, t)
            cand, _ = o.topk(I1, kp)
            assert np.array_equal(dag["cand"][t], cand), ("candidates", kss, t)
            fin, _ = o.rerank(q[t], w[t], kt(t), nt, cand, kk)
            assert np.array_equal(dag["idx"][t], fin), ("re-rank", kss, t)
            F1 = o.token_scores(q[t], w[t], np.arange(H_I, dtype=np.int32), kt(t), nt)
            want = np.array([F1[i] if 0 <= i < nt else 0.0 for i in ids[t]])
            assert np.array_equal(F_b[t], want), ("dense scores at ids", kss, t)
    pooled = o.pool_batch(caches, L * d, T, L, d, B)
    for t in range(T):
        assert np.array_equal(pooled[t], o.pool_keys(caches[t], B)), ("pool", t)


def check_batch_against_numpy(o):
    """Batched router (alone and inside the indexer driver) and token scores against NumPy written
    out per query (float64, integer
    inputs, so exact up to rounding of the block means), for a shared cache with a different prefix
    per query and for one cache per query."""
    rng = np.random.default_rng(13)
    T, H_I, d, L, B, h = 5, 6, 8, 40, 6, 2
    q = rng.integers(-3, 4, size=(T, H_I, d)).astype(np.float32)
    w = rng.integers(-2, 3, size=(T, H_I)).astype(np.float32)
    shared = rng.integers(-3, 4, size=(L, d)).astype(np.float32)
    caches = rng.integers(-3, 4, size=(T, L, d)).astype(np.float32)
    n = np.array([1, 5, 6, 23, 40], np.int32)
    heads = np.stack([rng.permutation(H_I)[:h] for _ in range(T)]).astype(np.int32)
    for k, kss, kt in ((shared, 0, lambda t: shared), (caches, L * d, lambda t: caches[t])):
        r_b, _ = o.route_batch(q, w, k, kss, n, B, h)
        r_i = o.indexer(0, q, w, k, kss, n, B, h, 3)["r"]
        I_b = o.scores(q, w, k, kss, n, heads=heads, ld=L)
        for t in range(T):
            nt = int(n[t])
            want_r = _np_router_scores(q[t], w[t], kt(t), nt, B)
            assert np.allclose(r_b[t], want_r, rtol=1e-12, atol=1e-12), ("router", kss, t)
            assert np.allclose(r_i[t], want_r, rtol=1e-12, atol=1e-12), ("indexer router", kss, t)
            K = kt(t)[:nt].astype(np.float64)
            hs = np.sort(heads[t])
            want_I = (w[t][hs].astype(np.float64)[:, None] *
                      np.maximum(q[t][hs].astype(np.float64) @ K.T, 0.0)).sum(axis=0)
            assert np.allclose(I_b[t][:nt], want_I, rtol=0, atol=1e-12), ("scores", kss, t)


def check_block_filter_hand_example(o):
    """Hand-derived cases of the block filter composed with MISA (tests/golden/hand_example.json,
    "block_filter"): block scores, kept blocks, selected tokens, with exact ties."""
    g = _load_golden()
    k = np.array(g["keys"], np.float32)
    q = np.array(g["q"], np.float32)
    w = np.array(g["w"], np.float32)
    for c in g["block_filter"]["cases"]:
        n, B, h, m, kk = c["n"], c["B"], c["h"], c["m"], c["k"]
        res = o.block_filter(q[None], w[None], k, 0, np.array([n]), B, h, m, kk)
        tag = f"n={n} B={B} h={h} m={m} k={kk}"
        assert np.array_equal(res["S"][0], np.array(c["S"], np.float64)), f"block scores {tag}: {res['S'][0]}"
        blocks = res["blocks"][0]
        assert list(blocks[:len(c["blocks"])]) == c["blocks"] and np.all(blocks[len(c["blocks"]):] == -1), \
            f"kept blocks {tag}: {blocks}"
        got = res["idx"][0]
        want = c["idx"]
        valid = [s for s in want if s >= 0]
        assert sorted(got[:len(valid)].tolist()) == sorted(valid) and np.all(got[len(valid):] == -1), \
            f"selection {tag}: {got}"
        S1 = o.block_scores(q, w, res["heads"][0], k, n, B)
        assert np.array_equal(S1, res["S"][0]), f"single-query block scores {tag}"


def _kept_tokens(blocks, n, B):
    return {s for b in blocks if b >= 0 for s in range(b * B, min((b + 1) * B, n))}


def check_block_filter_reductions(o):
    """Keeping every block is MISA bit for bit; with B = 1 the block scores are the token scores
    and keeping m >= k blocks is MISA again; with h = H_I and every block kept it is the dense
    indexer."""
    q, w, k = _small_clustered(8, H_I=8, d=16, L=300)
    Q = np.stack([q, q[::-1], 0.5 * q])
    W = np.stack([w, w[::-1], -w])
    n = np.array([300, 217, 9], np.int32)
    H_I = q.shape[0]
    for B, h, kk in ((16, 3, 20), (7, 2, 64), (64, 5, 5)):
        M = -(-300 // B)
        misa = o.indexer(0, Q, W, k, 0, n, B, h, kk)
        for m in (M, M + 3):
            bf = o.block_filter(Q, W, k, 0, n, B, h, m, kk)
            for key in ("r", "heads", "idx", "idx_v"):
                assert np.array_equal(bf[key], misa[key]), f"every block kept: {key} differs (B={B})"
        dense = o.indexer(2, Q, W, k, 0, n, B, h, kk)
        bf = o.block_filter(Q, W, k, 0, n, B, H_I, M, kk)
        assert np.array_equal(bf["idx"], dense["idx"]) and np.array_equal(bf["idx_v"], dense["idx_v"]), \
            f"h = H_I with every block kept is the dense indexer (B={B})"
    for h, kk in ((2, 10), (4, 33)):
        misa = o.indexer(0, Q, W, k, 0, n, 1, h, kk)
        I = o.scores(Q, W, k, 0, n, heads=misa["heads"], ld=300)
        for m in (kk, kk + 7):
            bf = o.block_filter(Q, W, k, 0, n, 1, h, m, kk)
            for t in range(3):
                nt = int(n[t])
                assert np.array_equal(bf["S"][t][:nt], I[t][:nt]), "B = 1: block scores are token scores"
            assert np.array_equal(bf["idx"], misa["idx"]), "B = 1 and m >= k: MISA's selection"


def check_block_filter_invariants(o):
    """Block scores sum to the routed heads' router scores; the kept blocks are the m best block
    scores; the selection is MISA's top-k restricted to the kept blocks' tokens, so MISA's own
    picks inside kept blocks survive; scaling and keys past the prefix act as for MISA; the
    batched driver matches the single-query block scores for a shared cache and per-query caches."""
    rng = np.random.default_rng(14)
    T, H_I, d, L = 5, 8, 16, 260
    q = rng.standard_normal((T, H_I, d)).astype(np.float32)
    w = (rng.standard_normal((T, H_I)) / math.sqrt(H_I)).astype(np.float32)
    shared = rng.standard_normal((L, d)).astype(np.float32)
    caches = rng.standard_normal((T, L, d)).astype(np.float32)
    n = np.array([0, 1, 37, 200, 260], np.int32)
    for k, kss, kt in ((shared, 0, lambda t: shared), (caches, L * d, lambda t: caches[t])):
        for B, h, m, kk in ((16, 3, 4, 20), (13, 2, 1, 8), (32, 4, 3, 100), (10, 1, 0, 5)):
            bf = o.block_filter(q, w, k, kss, n, B, h, m, kk)
            misa = o.indexer(0, q, w, k, kss, n, B, h, kk)
            assert np.array_equal(bf["heads"], misa["heads"]) and np.array_equal(bf["r"], misa["r"]), "routing"
            I = o.scores(q, w, k, kss, n, heads=bf["heads"], ld=L)
            for t in range(T):
                nt = int(n[t])
                Mt = -(-nt // B)
                S = bf["S"][t][:Mt]
                tag = (kss, B, m, t)
                assert np.all(np.isnan(bf["S"][t][Mt:])), tag
                assert np.array_equal(S, o.block_scores(q[t], w[t], bf["heads"][t], kt(t), nt, B)), tag
                routed = float(sum(misa["r"][t][j] for j in bf["heads"][t]))
                assert abs(S.sum() - routed) <= 1e-12 * max(1.0, abs(routed)), ("sum of block scores", tag)
                blocks = bf["blocks"][t]
                want_b = np.argsort(-S, kind="stable")[:m]
                assert np.array_equal(blocks[:len(want_b)], want_b) and np.all(blocks[len(want_b):] == -1), \
                    ("kept blocks", tag)
                kept = _kept_tokens(blocks, nt, B)
                sel = [s for s in bf["idx"][t] if s >= 0]
                assert set(sel) <= kept, ("selection outside the kept blocks", tag)
                assert len(sel) == min(kk, len(kept)) and np.all(bf["idx"][t][len(sel):] == -1), tag
                masked = np.where([s in kept for s in range(nt)], I[t][:nt], -np.inf)
                want = np.argsort(-masked, kind="stable")[:min(kk, len(kept))]
                assert sorted(sel) == sorted(want.tolist()), ("restricted top-k", tag)
                assert np.array_equal(np.sort(bf["idx_v"][t][:len(sel)]), np.sort(I[t][sel])), tag
                assert (set(misa["idx"][t].tolist()) & kept) <= set(sel), ("MISA picks in kept blocks", tag)
    q1, w1, k1 = q[3], w[3], shared
    base = o.block_filter(q1[None], w1[None], k1, 0, np.array([200]), 16, 3, 4, 20)
    for name, (q2, w2, k2) in {"k": (q1, w1, 2 * k1), "q": (2 * q1, w1, k1), "w": (q1, 2 * w1, k1)}.items():
        sc = o.block_filter(q2[None], w2[None], k2, 0, np.array([200]), 16, 3, 4, 20)
        assert np.array_equal(sc["S"], 2 * base["S"]), f"block scores scale with {name}"
        assert np.array_equal(sc["blocks"], base["blocks"]) and np.array_equal(sc["idx"], base["idx"]), name
    k3 = k1.copy()
    k3[200:] = 1000.0 * np.sign(k3[200:]) + 3.0
    past = o.block_filter(q1[None], w1[None], k3, 0, np.array([200]), 16, 3, 4, 20)
    for key in ("r", "heads", "S", "blocks", "idx", "idx_v"):
        assert np.array_equal(past[key], base[key], equal_nan=True), f"keys past the prefix changed {key}"


def _paged(o, pool, table, n, L):
    try:
        return o.paged_caches(pool, table, n, L)
    except ValueError as e:  # a mistake that reads an unused table entry shows up here
        raise AssertionError(str(e))


def check_paged_caches(o):
    """Paged key caches: contiguous caches scattered page by page (numpy) into a shuffled pool with
    spare pages, prefix pages shared between sequences and garbage table entries past each prefix,
    gather back to the same logical caches, and every indexer (MISA, MISA-dagger, dense, block
    filter) gives bit for bit what it gives on the contiguous caches."""
    rng = np.random.default_rng(15)
    T, L, d, ps, H_I = 4, 100, 16, 16, 8
    lp = -(-L // ps)
    caches = rng.integers(-3, 4, size=(T, L, d)).astype(np.float32)
    caches[1, :3 * ps] = caches[0, :3 * ps]  # sequences 0 and 1 share a 48-key prefix
    n = np.array([100, 97, 33, 0], np.int32)
    caches_p = caches.copy()
    for t in range(T):
        caches_p[t, n[t]:] = 0.0
    num_pages = T * lp + 5
    perm = rng.permutation(num_pages)
    pool = rng.integers(-9, 10, size=(num_pages, ps, d)).astype(np.float32)  # spare pages hold junk
    table = np.full((T, lp + 2), -1, np.int32)
    padded = np.zeros((T, lp * ps, d), np.float32)
    padded[:, :L] = caches
    for t in range(T):
        for g in range(-(-int(n[t]) // ps)):
            if t == 1 and g < 3:
                table[t, g] = table[0, g]  # shared physical pages
                continue
            table[t, g] = perm[t * lp + g]
            pool[table[t, g]] = padded[t, g * ps:(g + 1) * ps]
        table[t, -(-int(n[t]) // ps):] = rng.integers(num_pages, 10 * num_pages)  # never read
    got = _paged(o, pool, table, n, L)
    assert np.array_equal(got, caches_p), "paged gather differs from the contiguous caches"
    q = rng.integers(-3, 4, size=(T, H_I, d)).astype(np.float32)
    w = rng.integers(-2, 3, size=(T, H_I)).astype(np.float32)
    B, h, kk, kp = 7, 3, 9, 20
    for mode, extra in ((0, {}), (1, {"kp": kp}), (2, {})):
        a = o.indexer(mode, q, w, got, L * d, n, B, h, kk, **extra)
        b = o.indexer(mode, q, w, caches, L * d, n, B, h, kk, **extra)
        for key in a:
            assert np.array_equal(a[key], b[key]), f"mode {mode}: {key} differs on the paged caches"
    a = o.block_filter(q, w, got, L * d, n, B, h, 4, kk)
    b = o.block_filter(q, w, caches, L * d, n, B, h, 4, kk)
    for key in a:
        assert np.array_equal(a[key], b[key], equal_nan=True), f"block filter: {key} differs on the paged caches"
    bad = table.copy()
    bad[2, 1] = num_pages + 3  # inside the prefix of sequence 2 (33 keys, 3 pages)
    try:
        o.paged_caches(pool, bad, n, L)
    except ValueError:
        pass
    else:
        raise AssertionError("an out-of-range page inside a prefix must be reported")


def check_paged_hand_example(o):
    """The hand example's five keys stored by hand in pages of two (a junk page, the partial last
    page first, the logical pages in reverse order, junk in the unused row): the gathered cache is
    the key list, and the indexer reproduces the hand-computed values of the golden fixture."""
    g = _load_golden()
    keys = np.array(g["keys"], np.float32)
    pool = np.array([[[9, 9], [9, 9]],      # physical page 0: unused
                     [[4, -2], [7, 7]],     # page 1: logical page 2 = {k4}, junk row
                     [[0, 2], [-2, 4]],     # page 2: logical page 1 = {k2, k3}
                     [[1, 0], [3, 2]]],     # page 3: logical page 0 = {k0, k1}
                    np.float32)
    table = np.array([[3, 2, 1], [3, 2, 0]], np.int32)
    n = np.array([5, 4], np.int32)
    got = _paged(o, pool, table, n, 5)
    assert np.array_equal(got[0], keys), f"paged gather of the hand example: {got[0]}"
    assert np.array_equal(got[1][:4], keys[:4]) and np.all(got[1][4] == 0), f"n = 4: {got[1]}"
    q = np.array(g["q"], np.float32)
    w = np.array(g["w"], np.float32)
    Q, Wt = np.stack([q, q]), np.stack([w, w])
    res = o.indexer(0, Q, Wt, got, 5 * 2, n, g["B"], 1, 2)
    for t, qc in enumerate(g["queries"]):
        assert np.array_equal(res["r"][t], np.array(qc["r"], np.float64)), f"paged router scores n={qc['n']}"
        assert list(res["heads"][t]) == qc["h1"]["heads"], f"paged routed head n={qc['n']}"
        assert sorted(res["idx"][t]) == sorted(qc["h1"]["top2"]), f"paged top-2 n={qc['n']}"


ALL_CHECKS = [
    check_hand_example,
    check_topk_vs_stable_argsort,
    check_topk_with_ids,
    check_pool_special_cases,
    check_router_bruteforce,
    check_scores_bruteforce,
    check_scaling,
    check_head_permutation,
    check_full_routing_is_dense,
    check_dagger_invariants,
    check_prefix_only,
    check_empty_and_short,
    check_negative_weight_sign,
    check_planted_needles,
    check_batch_matches_single_query,
    check_batch_against_numpy,
    check_block_filter_hand_example,
    check_block_filter_reductions,
    check_block_filter_invariants,
    check_paged_caches,
    check_paged_hand_example,
]
