"""misa_score_topk_fused (chunked prefill without score rows) against misa_score_topk and the oracle.

Both calls score with the same tensor-core arithmetic and select exactly, so on every query their
selections must be the same sets with the same values.  Cases:
  * two whole chunks of the 64K causal prefill (4096 queries each, the first chunk's prefixes of
    1..4096 keys and the last chunk's of 61441..65536), routed heads from the GPU router; 64 rows
    of each are also checked against the oracle under the tie-band rule;
  * a cache whose strongest keys all sit in the sampled tiles (every 32nd tile of 128 keys): the
    cut lands above almost every other key, the lists fall short of k, and the queries must be
    redone exactly;
  * a cache of equal keys: every score ties with the cut, every list overflows, the redo keeps the
    lowest token indices;
  * prefixes of at most 4k keys, which skip the cut and list every key;
  * one strong key repeated 3000 times: the k-th place falls inside an exact tie held by the list.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _same(L_, qd, wd, kd, nd, hd, topk, what):
    a, av = L_.misa_score_topk(qd, wd, kd, nd, hd, topk)
    b, bv = L_.misa_score_topk_fused(qd, wd, kd, nd, hd, topk)
    a, av, b, bv = host(a), host(av), host(b), host(bv)
    for t in range(a.shape[0]):
        oa, ob = np.argsort(a[t], kind="stable"), np.argsort(b[t], kind="stable")
        assert np.array_equal(a[t][oa], b[t][ob]), f"{what} q{t}: sets differ"
        assert np.array_equal(av[t][oa], bv[t][ob]), f"{what} q{t}: values differ"
    L_.misa_device_check()
    return b


@pytest.mark.parametrize("chunk", [0, 15])
def test_whole_prefill_chunk(chunk):
    L_ = lib()
    wl = W.WORKLOADS[3]
    ch = wl.chunk
    k = W.shared_keys(wl)
    t0 = chunk * ch
    q, w = W.shared_queries(wl, t0, t0 + ch)
    n = W.prefix_lengths(wl, t0, t0 + ch)
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    kbar = L_.misa_pool_keys(kd, wl.B)
    hd, _ = L_.misa_route(qd, wd, kd, kbar, nd, wl.B, wl.h)
    got = _same(L_, qd, wd, kd, nd, hd, wl.topk, f"chunk {chunk}")
    rows = sorted(set(np.linspace(0, ch - 1, 64).astype(int).tolist()))
    hh = host(hd)[rows]
    o = oracle.get()
    I = o.scores(q[rows], w[rows], k, 0, n[rows], heads=hh, ld=wl.L)
    for i, t in enumerate(rows):
        nt = int(n[t])
        ids, _ = o.topk(I[i][:nt], wl.topk)
        st = P.score_tol(q[t], w[t], k, nt, hh[i])
        P.check_selection(got[t], ids, I[i][:nt], st, wl.topk, f"fused chunk {chunk} q{t0 + t} vs oracle")


def _heads(T, H_I, h, seed):
    g = np.random.default_rng(seed)
    return np.stack([np.sort(g.choice(H_I, h, replace=False)) for _ in range(T)]).astype(np.int32)


def _one_cache_case(kf, T, topk, what, seed):
    L_ = lib()
    g = np.random.default_rng(seed)
    L = kf.shape[0]
    H_I, h = 64, 8
    q = W.round_bf16(g.standard_normal((T, H_I, 128)).astype(np.float32))
    w = np.abs(g.standard_normal((T, H_I))).astype(np.float32) / 8
    n = np.linspace(L // 2, L, T).astype(np.int32)
    hd = dev(_heads(T, H_I, h, seed), torch.int32)
    return _same(L_, dev(q, torch.bfloat16), dev(w, torch.float32), dev(kf, torch.bfloat16), dev(n, torch.int32), hd,
                 topk, what), n


def test_lists_that_fall_short_are_redone():
    """Keys in the sampled tiles (every 32nd tile of 128) are large and point along +1, the others are
    small and point along -1: the sample's cut lies far above every unsampled key."""
    L = 40000
    k = -np.ones((L, 128), np.float32) * 0.05
    for j in range(0, L, 32 * 128):
        k[j:j + 128] = 1.0 + 0.01 * np.arange(128)[:, None] / 128
    _one_cache_case(W.round_bf16(k), 64, 2048, "short lists", 5)


def test_lists_that_overflow_are_redone():
    """Every key equal: every score ties with the cut, so every list overflows; the redo keeps the
    lowest token indices."""
    L = 40000
    k = np.tile(W.round_bf16(np.random.default_rng(7).standard_normal((1, 128)).astype(np.float32)), (L, 1))
    got, n = _one_cache_case(k, 64, 2048, "overflowing lists", 6)
    for t in range(got.shape[0]):
        assert sorted(got[t].tolist()) == list(range(2048)), "all scores tie: the lowest ids"


def test_short_prefixes_take_every_key():
    """Prefixes of at most 4k keys skip the cut (every key is listed), including empty ones."""
    L_ = lib()
    wl = W.small(3, L=9000, T=9000, chunk=256)
    k = W.shared_keys(wl)
    q, w = W.shared_queries(wl, 0, 256)
    n = np.array([0, 1, 5, 2047, 2048, 2049, 8191, 8192, 8193] * 28 + [9000] * 4, np.int32)
    hd = dev(_heads(256, wl.H_I, wl.h, 9), torch.int32)
    _same(L_, dev(q, torch.bfloat16), dev(w, torch.float32), dev(k, torch.bfloat16), dev(n, torch.int32), hd, 2048,
          "short prefixes")


def test_ties_across_the_kth_place_are_ranked_by_token():
    """3000 copies of one strong key among random keys (queries with positive entries, so the copy
    scores far above the rest): each list holds all copies under its cap, the k-th place falls inside
    the tie, and the k lowest tokens among the copies are selected."""
    L_ = lib()
    L, T, H_I, h, topk = 40000, 64, 64, 8, 2048
    g = np.random.default_rng(8)
    k = W.round_bf16(0.3 * g.standard_normal((L, 128)).astype(np.float32))
    pos = np.sort(g.choice(L, 3000, replace=False))
    k[pos] = W.round_bf16(np.abs(g.standard_normal((1, 128))).astype(np.float32))
    q = W.round_bf16(np.abs(g.standard_normal((T, H_I, 128))).astype(np.float32))
    w = np.abs(g.standard_normal((T, H_I))).astype(np.float32) / 8
    n = np.linspace(32000, L, T).astype(np.int32)
    hd = dev(_heads(T, H_I, h, 10), torch.int32)
    got = _same(L_, dev(q, torch.bfloat16), dev(w, torch.float32), dev(k, torch.bfloat16), dev(n, torch.int32), hd,
                topk, "ties at the k-th place")
    for t in range(T):
        tied = pos[pos < n[t]]
        assert len(tied) > topk
        assert sorted(got[t].tolist()) == tied[:topk].tolist(), "the lowest tokens of the tie"
