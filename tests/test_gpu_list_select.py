"""The candidate-list top-k of per-query caches against the oracle and against the plain per-row
selection, including inputs built so that the list cannot hold the answer.

For a few rows longer than the selection kernel's own list, misa_score_topk (and misa_token_scores
with a selection workspace, or misa_topk_select itself) builds a candidate list per row: one CTA
places the row's cut from a sample of its scores (256 evenly spaced runs of 8), CTAs over chunks of
8192 scores append every entry at or above it; the selection ranks the list, and a row with fewer
than k entries, or whose list overflowed, takes the exact pass over its score row.
The cases:
  * clustered keys, prefixes below, at and above the list size, k from 1 to 16384, against the
    oracle's top-k under the tie-band rule and against misa_topk_select (the same fp32 scores, so
    the same set);
  * a cache of identical keys: every score ties, and the k lowest token ids must come back;
  * strong keys packed into the first 20000 positions: the cut lies among them;
  * strong keys placed exactly on the sampled positions: the sample overstates the row, the cut
    leaves far fewer than k entries, and the exact path must select every strong key and the best
    of the rest (for a few rows with lists, and for 320 rows of one shared cache, which take the
    row kernel's own sampled cut).
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
    k[1][: L // 2] = k[1][7]  # half of cache 1: a tie that spans far more than k
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


def test_list_short_of_k_when_the_sample_hits_every_strong_key():
    L_ = lib()
    L, T, topk, d, H_I = 131072, 2, 8192, 128, 64
    rng = np.random.default_rng(12)
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    q = W.round_bf16((u + 0.05 * rng.standard_normal((T, H_I, d))).astype(np.float32))
    w = np.zeros((T, H_I), np.float32)
    w[:, :8] = 1.0
    k = W.round_bf16((0.2 * u + 0.05 * rng.standard_normal((T, L, d))).astype(np.float32))
    # the sample reads runs of 8 scores every (n_t / 256) & ~7 = 512 positions
    pos = np.nonzero(np.arange(L) % 512 < 8)[0]
    k[:, pos] = W.round_bf16((3.0 * u + 0.05 * rng.standard_normal((T, len(pos), d))).astype(np.float32))
    n = np.array([L, L], np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    heads = dev(np.tile(np.arange(8, dtype=np.int32), (T, 1)), torch.int32)
    idx, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, topk)
    gi = host(idx)
    for t in range(T):
        assert set(pos.tolist()) <= set(gi[t].tolist()), "every strong key is selected"
    _check_against_oracle(q, w, k, n, host(heads), gi, topk, "strong keys on the sample")


def test_many_rows_against_oracle_with_rows_the_sample_misleads():
    """320 queries on one shared cache: the many-rows path (one 512-thread CTA per row: a sampled cut,
    a sweep for candidates, the list ranked).  Strong keys sit exactly on the sampled positions of the
    rows with n_t = L, so their sample overstates the row, the cut leaves fewer than k candidates and
    those rows take the exact path; prefixes at and below the list size take every entry."""
    L_ = lib()
    L, T, topk, d, H_I, h = 40000, 320, 2048, 128, 64, 8
    g = np.random.default_rng(13)
    k = W.round_bf16((0.3 * g.standard_normal((L, d))).astype(np.float32))
    seg = (L // 256) & ~7
    pos = np.nonzero((np.arange(L) % seg < 8) & (np.arange(L) < 256 * seg))[0]
    u = np.abs(g.standard_normal(d))
    k[pos] = W.round_bf16((u / np.linalg.norm(u) * 4.0 + 0.05 * g.standard_normal((len(pos), d))).astype(np.float32))
    q = W.round_bf16(g.standard_normal((T, H_I, d)).astype(np.float32))
    w = (g.standard_normal((T, H_I)) / 8).astype(np.float32)
    n = np.concatenate([np.full(64, L), g.integers(1, L + 1, T - 96), [8192, 8193, 1, 0] * 8]).astype(np.int32)
    heads = np.stack([np.sort(g.choice(H_I, h, replace=False)) for _ in range(T)]).astype(np.int32)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    hd = dev(heads, torch.int32)
    idx, vals = L_.misa_score_topk(qd, wd, kd, nd, hd, topk)
    scores = L_.misa_token_scores(qd, wd, kd, nd, hd)
    b, _ = L_.misa_topk_select(scores, nd, topk)
    gi, gb = host(idx), host(b)
    for t in range(T):
        assert sorted(gi[t].tolist()) == sorted(gb[t].tolist()), f"q{t} n_t {n[t]}"
        nt = int(n[t])
        assert (gi[t][min(topk, nt):] == -1).all()
    o = oracle.get()
    I = o.scores(q, w, k, 0, n, heads=heads, ld=L)
    for t in range(T):
        nt = int(n[t])
        ids, _ = o.topk(I[t][:nt], topk)
        tol = P.score_tol(q[t], w[t], k, nt, heads[t])
        P.check_selection(gi[t], ids, I[t][:nt], tol, topk, f"many rows q{t} (n_t {nt})")
    sc = host(scores)
    v = host(vals)
    for t in range(T):
        sel = gi[t][gi[t] >= 0]
        assert np.array_equal(v[t][: len(sel)], sc[t][sel])
