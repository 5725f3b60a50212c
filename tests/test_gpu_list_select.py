"""The candidate-list top-k of per-query caches against the oracle and against the plain per-row
selection, including inputs built so that the list cannot hold the answer.

For one bf16 cache per query, misa_score_topk (and misa_token_scores with a selection workspace)
builds a candidate list per query while it scores: each CTA that scores a run of the query's keys
keeps the run's entries at or above a cut placed on the run's own scores and raises the query's
cut key to it; the selection ranks the list's entries at or above the query's cut key, and a row
with fewer than k such entries, or whose list overflowed, takes the exact pass over its score row.
The cases:
  * clustered keys, prefixes below, at and above the list size, k from 1 to 16384, against the
    oracle's top-k under the tie-band rule and against misa_topk_select without the list (the same
    fp32 scores, so the same set);
  * a cache of identical keys: every score ties, the list overflows, and the exact path must return
    the k lowest token ids;
  * strong keys packed into the first 20000 positions: the runs there place their cuts high, the
    query's cut key leaves far fewer than k entries, and the exact path must select the strongest.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _check_against_oracle(q, w, k, n, heads, got, topk, what):
    o = oracle.get()
    T = q.shape[0]
    L = k.shape[1]
    I = o.scores(q, w, k, L * k.shape[2], n, heads=heads, ld=L)
    for t in range(T):
        nt = int(n[t])
        ids, _ = o.topk(I[t][:nt], topk)
        tol = P.score_tol(q[t], w[t], k[t], nt, heads[t])
        P.check_selection(got[t], ids, I[t][:nt], tol, topk, f"{what} q{t} (n_t {nt}, k {topk})")


@pytest.mark.parametrize("topk", [1, 2048, 8192, 16384])
def test_list_selection_matches_oracle_and_plain_selection(topk):
    L_ = lib()
    L = 40000
    n = np.array([40000, 39999, 16384, 16385, 20000, 17000, 5000, 1], np.int32)
    wl = W.small(2, L=L, n_seq=len(n), T=len(n), seed=4200 + topk)
    k, q, w, _, _ = W.decode_batch(wl)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    heads, _ = L_.misa_route(qd, wd, kd, L_.misa_pool_keys(kd, wl.B), nd, wl.B, wl.h)
    idx, vals = L_.misa_score_topk(qd, wd, kd, nd, heads, topk)
    ws = L_.Workspace()
    scores = L_.misa_token_scores(qd, wd, kd, nd, heads, select_topk=topk, select_ws=ws)
    a, _ = L_.misa_topk_select(scores, nd, topk, ws=ws, ws_prepared=True)
    b, _ = L_.misa_topk_select(scores, nd, topk)
    gi, ga, gb = host(idx), host(a), host(b)
    for t in range(len(n)):
        assert sorted(gi[t].tolist()) == sorted(ga[t].tolist()) == sorted(gb[t].tolist()), f"q{t} n_t {n[t]}"
    _check_against_oracle(q, w, k, n, host(heads), gi, topk, "list selection")
    # the scores returned with the selection are the row's scores
    sc = host(scores)
    for t in range(len(n)):
        sel = gi[t][gi[t] >= 0]
        assert np.array_equal(host(vals)[t][: len(sel)], sc[t][sel])


def test_list_overflow_on_identical_keys_takes_the_lowest_ids():
    L_ = lib()
    L, T, topk = 65536, 3, 8192
    wl = W.small(2, L=L, n_seq=T, T=T, seed=4300)
    k, q, w, _, _ = W.decode_batch(wl)
    k[0][:] = k[0][123]  # every key of cache 0 is the same key
    k[1][: L // 2] = k[1][7]  # half of cache 1: a tie that spans far more than the list
    n = np.array([L, L, 40000], np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    heads = dev(np.tile(np.arange(8, dtype=np.int32), (T, 1)), torch.int32)
    idx, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, topk)
    gi = host(idx)
    assert sorted(gi[0].tolist()) == list(range(topk)), "all scores tie: the lowest ids"
    _check_against_oracle(q, w, k, n, host(heads), gi, topk, "identical keys")


def test_list_short_of_k_when_strong_keys_are_packed_together():
    L_ = lib()
    L, T, topk, d, H_I = 131072, 2, 8192, 128, 64
    rng = np.random.default_rng(11)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = W.round_bf16((u + 0.05 * rng.standard_normal((T, H_I, d))).astype(np.float32))
    w = np.zeros((T, H_I), np.float32)
    w[:, :8] = 1.0
    k = W.round_bf16((0.2 * u + 0.05 * rng.standard_normal((T, L, d))).astype(np.float32))
    k[:, :20000] = W.round_bf16((3.0 * u + 0.05 * rng.standard_normal((T, 20000, d))).astype(np.float32))
    n = np.array([L, L], np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    heads = dev(np.tile(np.arange(8, dtype=np.int32), (T, 1)), torch.int32)
    idx, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, topk)
    gi = host(idx)
    for t in range(T):
        assert gi[t].min() >= 0 and gi[t].max() < 20000, "the selection lies among the strong keys"
    _check_against_oracle(q, w, k, n, host(heads), gi, topk, "packed strong keys")
