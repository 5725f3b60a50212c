"""Tensor-core scoring of queries that share one bf16 key cache (the chunked-prefill kernel),
element by element against the oracle.

Covers every head-count class of the kernel (each query's head rows padded to 8, 16, 32, 64 or
128), ragged prefixes that cut key tiles short (0, 1, 127, 128, 129, ..., L keys), L not a
multiple of the 128-key tile, query counts that leave a partial query block, a call that the
host splits into several launches, head lists in any order, and entries at s >= n_t, which
must stay untouched."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu

EDGE_N = [0, 1, 2, 127, 128, 129, 255, 256, 257]


def _inputs(L, T, H_I, seed):
    wl = W.small(3, L=L, T=T, chunk=T, H_I=H_I, dtype="bf16", seed=5000 + seed)
    k = W.shared_keys(wl)
    q, w = W.shared_queries(wl, 0, T)
    g = np.random.default_rng(seed)
    n = g.integers(0, L + 1, size=T).astype(np.int32)
    e = [x for x in EDGE_N + [L - 1, L] if x <= L]
    n[: min(T, len(e))] = e[: min(T, len(e))]
    return k, q, w, n, g


def _heads(g, T, H_I, h):
    return np.stack([g.choice(H_I, h, replace=False) for _ in range(T)]).astype(np.int32)


def _run(L_, k, q, w, n, heads):
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    out = torch.full((q.shape[0], k.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
    hd = None if heads is None else dev(heads, torch.int32)
    L_.misa_token_scores(qd, wd, kd, nd, hd, out=out)
    return host(out)


def _check(k, q, w, n, heads, got, rows=None):
    o = oracle.get()
    L = k.shape[0]
    rows = range(q.shape[0]) if rows is None else rows
    sel = np.asarray(list(rows))
    want = o.scores(q[sel], w[sel], k, 0, n[sel], heads=None if heads is None else heads[sel], ld=L)
    for i, t in enumerate(sel.tolist()):
        nt = int(n[t])
        assert np.all(np.isnan(got[t][nt:])), f"t={t}: entries at s >= n_t were written"
        if nt == 0:
            continue
        tol = P.score_tol(q[t], w[t], k, nt, None if heads is None else heads[t])
        P.check_close(got[t][:nt], want[i][:nt], tol, f"t={t} n={nt}")


@pytest.mark.parametrize("L,T,H_I,h", [
    (4099, 100, 64, 8),     # 8 rows per query, 4 query blocks (the last partial)
    (1000, 33, 64, 5),      # 5 heads padded to 8
    (1000, 40, 64, 9),      # padded to 16
    (1000, 20, 64, 17),     # padded to 32
    (1000, 10, 64, None),   # dense: 64 rows per query
    (600, 6, 128, 128),     # 128 rows per query, two queries per block
    (130, 3, 64, 8),        # fewer queries than a block, two key tiles
])
def test_shared_cache_scores_match_the_oracle(L, T, H_I, h):
    L_ = lib()
    k, q, w, n, g = _inputs(L, T, H_I, seed=L + T + H_I)
    heads = None if h is None else _heads(g, T, H_I, h)
    got = _run(L_, k, q, w, n, heads)
    _check(k, q, w, n, heads, got)
    L_.misa_device_check()


def test_call_split_over_launches():
    """128 rows per query: 2 queries per block and at most 4096 queries per launch, so 4100
    queries take two launches; rows on both sides of the split are checked."""
    L_ = lib()
    L, T, H_I = 300, 4100, 128
    k, q, w, n, g = _inputs(L, T, H_I, seed=7)
    heads = _heads(g, T, H_I, 128)
    got = _run(L_, k, q, w, n, heads)
    rows = sorted(set(range(0, 40)) | set(range(4080, 4100)) | set(g.choice(T, 60, replace=False).tolist()))
    _check(k, q, w, n, heads, got, rows)
    for t in range(T):
        assert np.all(np.isnan(got[t][n[t]:])), f"t={t}: entries at s >= n_t were written"
        assert not np.any(np.isnan(got[t][: n[t]])), f"t={t}: entries below n_t missing"
    L_.misa_device_check()


def test_prefill_chunk_shape():
    """A causal chunk: the last 512 queries of a 6000-key prefix (n_t = L - T + 1 + t)."""
    L_ = lib()
    wl = W.small(3, L=6000, T=512, chunk=512, dtype="bf16", seed=77)
    k = W.shared_keys(wl)
    q, w = W.shared_queries(wl, 0, wl.T)
    n = W.prefix_lengths(wl)
    heads = _heads(np.random.default_rng(3), wl.T, wl.H_I, 8)
    got = _run(L_, k, q, w, n, heads)
    _check(k, q, w, n, heads, got, rows=range(0, wl.T, 7))
    L_.misa_device_check()


def test_all_heads_in_any_order_is_dense_bit_for_bit():
    """Routing every head, listed in a shuffled order, gives the dense scores exactly: the kernel
    sorts each head list, so both sum the same terms in the same order."""
    L_ = lib()
    L, T, H_I = 2000, 50, 64
    k, q, w, n, g = _inputs(L, T, H_I, seed=11)
    heads = _heads(g, T, H_I, H_I)
    a = _run(L_, k, q, w, n, heads)
    b = _run(L_, k, q, w, n, None)
    assert np.array_equal(a, b, equal_nan=True)
    L_.misa_device_check()
