"""misa_hier_rerank_static, the re-rank entry point that allocates nothing.

Callers that cannot allocate device memory (a plugin handed only its input and output buffers
by a host framework that owns the device memory, or a decode loop that must not risk an
allocation or the synchronisation it can bring mid-step) use this variant: its scratch is a
fixed array inside the library.  This file is collected last so that a run stopping at the first
failure has already run every other test; it passes alone in a fresh process too.

Checks, all through the C ABI:
  * two calls in a row on different batches (the second sees the first call's leftovers in the
    shared array): each result agrees with misa_hier_rerank's under the tie-band rule of the
    parity tests, with scores within the score tolerance;
  * the same kind of call against the CPU oracle's re-rank on candidate lists with empty (-1)
    slots, candidates past a query's prefix, prefixes shorter than k and exact ties across the
    k-th value (copies of the boundary key): the selection follows the oracle under the tie-band
    rule and, inside a group of exactly tied candidates, takes the lowest token ids;
  * a request larger than the array is refused with MISA_ERR_WORKSPACE, launching nothing.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _batch(L, T, seed):
    wl = W.small(4, L=L, n_seq=T, T=T, seed=7000 + seed)
    k, q, w, n, _ = W.decode_batch(wl)
    return wl, k, q, w, n


def _static_call(M, q, w, k, n, cand, topk):
    T, H_I, d = q.shape
    L = k.shape[1]
    idx = torch.full((T, topk), -7, dtype=torch.int32, device="cuda")
    vals = torch.full((T, topk), float("nan"), dtype=torch.float32, device="cuda")
    st = M.library().misa_hier_rerank_static(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(k.data_ptr()), L * d,
        ctypes.c_void_p(n.data_ptr()), ctypes.c_void_p(cand.data_ptr()), T, L, H_I, d, cand.shape[1], topk,
        M.BF16, ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(vals.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, idx, vals


def _dense_by_id(F_cand, cand, n):
    """Oracle dense scores indexed by token id (NaN where the token is not a valid candidate)."""
    v = np.full(n, np.nan)
    ok = (cand >= 0) & (cand < n)
    v[cand[ok]] = F_cand[ok]
    return v


def test_static_scratch_rerank_matches_workspace_rerank():
    M = lib()
    for call, (L, T, kp, topk) in enumerate(((20000, 8, 8192, 2048), (9000, 5, 4096, 1000))):
        wl, k, q, w, n = _batch(L, T, call)
        kd, qd = dev(k, torch.bfloat16), dev(q, torch.bfloat16)
        wd, nd = dev(w, torch.float32), dev(n, torch.int32)
        heads, _ = M.misa_route(qd, wd, kd, M.misa_pool_keys(kd, wl.B), nd, wl.B, wl.h)
        cand, _ = M.misa_score_topk(qd, wd, kd, nd, heads, kp, want_vals=False)
        ref_idx, ref_vals = M.misa_hier_rerank(qd, wd, kd, nd, cand, topk)
        st, idx, vals = _static_call(M, qd, wd, kd, nd, cand, topk)
        assert st == M.OK, M.library().misa_status_str(st)
        ri, rv, gi, gv, ch = host(ref_idx), host(ref_vals), host(idx), host(vals), host(cand)
        F = oracle.get().dense_scores_at(q, w, k, L * 128, n, ch)
        for t in range(T):
            nt = int(n[t])
            values = _dense_by_id(F[t], ch[t], nt)
            tol = np.where(np.isnan(values), np.inf, P.score_tol(q[t], w[t], k[t], nt, None))
            # two selection kernels may break fp32 near-ties differently: both must respect the band
            order_r = np.argsort(-values[ri[t][ri[t] >= 0]], kind="stable")
            P.check_selection(gi[t], ri[t][ri[t] >= 0][order_r], values, tol, topk, f"call {call} query {t}")
            sel = gi[t][gi[t] >= 0]
            P.check_close(gv[t][: len(sel)], values[sel], tol[sel], f"call {call} query {t} scores")


def _tie_case(seed, L, T, kp, topk):
    """Candidate lists with empty slots, ids past the prefix and ties copied onto the boundary key."""
    wl, k, q, w, n = _batch(L, T, 10 + seed)
    rng = np.random.default_rng(seed)
    n = np.array([L, L - 3000, topk + 37, topk // 2, 8191 % L][:T], np.int32)
    cand = np.stack([rng.choice(L, kp, replace=False) for _ in range(T)]).astype(np.int32)
    cand[:, rng.choice(kp, kp // 16, replace=False)] = -1  # empty slots
    o = oracle.get()
    groups = []
    for t in range(T):
        nt = int(n[t])
        ids, _ = o.rerank(q[t], w[t], k[t], nt, cand[t], topk)
        valid = cand[t][(cand[t] >= 0) & (cand[t] < nt)]
        if len(valid) <= topk:
            groups.append(np.zeros(0, np.int64))
            continue
        s_k = int(ids[topk - 1])  # the boundary token; copy its key onto six unselected candidates
        others = np.setdiff1d(valid, ids[ids >= 0])
        lo, hi = others[others < s_k], others[others > s_k]
        pick = np.concatenate([lo[:3], hi[-3:]])
        k[t][pick] = k[t][s_k]
        groups.append(np.sort(np.concatenate([pick, [s_k]])))
    return wl, k, q, w, n, cand, groups


def test_static_scratch_rerank_against_the_oracle():
    """Two calls in a row (the second on another batch and another k') against the oracle."""
    M = lib()
    o = oracle.get()
    for call, (L, T, kp, topk) in enumerate(((9000, 5, 4096, 1024), (16384, 4, 8192, 2048))):
        wl, k, q, w, n, cand, groups = _tie_case(call, L, T, kp, topk)
        kd, qd = dev(k, torch.bfloat16), dev(q, torch.bfloat16)
        wd, nd, cd = dev(w, torch.float32), dev(n, torch.int32), dev(cand, torch.int32)
        st, idx, vals = _static_call(M, qd, wd, kd, nd, cd, topk)
        assert st == M.OK, M.library().misa_status_str(st)
        gi, gv = host(idx), host(vals)
        F = o.dense_scores_at(q, w, k, L * 128, n, cand)
        for t in range(T):
            nt = int(n[t])
            ids, _ = o.rerank(q[t], w[t], k[t], nt, cand[t], topk)
            values = _dense_by_id(F[t], cand[t], nt)
            tol = np.where(np.isnan(values), np.inf, P.score_tol(q[t], w[t], k[t], nt, None))
            what = f"call {call} query {t} (n_t {nt})"
            P.check_selection(gi[t], ids, values, tol, topk, what)
            sel = gi[t][gi[t] >= 0]
            assert np.all(sel < nt), f"{what}: a candidate past the prefix was selected"
            P.check_close(gv[t][: len(sel)], values[sel], tol[sel], f"{what} scores")
            g = groups[t]
            if len(g):
                taken = np.intersect1d(sel, g)
                assert len(taken) >= 1, f"{what}: the boundary group lost every member"
                assert np.array_equal(taken, g[: len(taken)]), \
                    f"{what}: exact ties must go to the lowest ids ({taken} of {g})"


def test_static_scratch_rejects_oversized_requests():
    M = lib()
    T, kp, topk = 129, 8192, 2048  # 129 * 8192 floats > 1 << 20
    q = torch.zeros((T, 64, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((T, 64), dtype=torch.float32, device="cuda")
    k = torch.zeros((T, 8192, 128), dtype=torch.bfloat16, device="cuda")
    n = torch.full((T,), 8192, dtype=torch.int32, device="cuda")
    cand = torch.zeros((T, kp), dtype=torch.int32, device="cuda")
    st, idx, _ = _static_call(M, q, w, k, n, cand, topk)
    assert st == M.ERR_WORKSPACE
    assert torch.all(idx == -7), "nothing launched on a refused call"
