"""misa_hier_rerank_static, the re-rank entry point that allocates nothing.

Callers that cannot allocate device memory (a plugin handed only its input and output buffers
by a host framework that owns the device memory, or a decode loop that must not risk an
allocation or the synchronisation it can bring mid-step) use this variant: its scratch is a
fixed array inside the library.  This file is collected last so that a run stopping at the first
failure has already run every other test; it passes alone in a fresh process too.

Checks: called through the C ABI twice in a row on different batches (the second call sees the
first call's leftovers in the shared array), each result must equal misa_hier_rerank's (same
selected set, scores within the score tolerance of the parity tests); a request larger than the
array is refused with MISA_ERR_WORKSPACE.
"""
import ctypes

import numpy as np
import pytest
import torch

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
        ri, rv, gi, gv = host(ref_idx), host(ref_vals), host(idx), host(vals)
        for t in range(T):
            assert set(gi[t].tolist()) == set(ri[t].tolist()), f"call {call} query {t}: selected sets differ"
            order_g, order_r = np.argsort(gi[t]), np.argsort(ri[t])
            tol = P.score_tol(q[t], w[t], k[t], int(n[t]), None)[ri[t][order_r]]
            P.check_close(gv[t][order_g], rv[t][order_r], tol, f"call {call} query {t} scores")


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
