"""The MISA-dagger re-rank on the tensor cores (gathered candidate rows, all H_I heads) against the
oracle: candidate counts that are not multiples of the 128-row tile, every head-pool size the
tensor-core path takes (H_I = 16 .. 128 in steps of 16) and one it leaves to the warp-level path
(H_I = 24), many short queries (a CTA's range spans several queries, so head rows are staged many
times), empty slots and ids past the prefix, per-query and shared caches."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(T, L, H_I, kp, topk, shared, seed):
    rng = np.random.default_rng(seed)
    wl = W.small(2, L=L, n_seq=T, T=T, H_I=H_I, seed=5000 + seed)
    k, q, w, _, _ = W.decode_batch(wl)
    if shared:
        k = k[:1]
    n = rng.integers(max(1, L // 2), L + 1, size=T).astype(np.int32)
    n[0] = L
    cand = np.stack([rng.choice(L, kp, replace=False) for _ in range(T)]).astype(np.int32)
    cand[:, ::17] = -1  # empty slots; ids >= n_t are empty too
    return k, q, w, n, cand


@pytest.mark.parametrize("T,L,H_I,kp,topk,shared", [
    (8, 20000, 64, 8192, 2048, False),
    (5, 9000, 64, 1000, 300, False),
    (300, 4096, 64, 256, 64, False),
    (4, 6000, 16, 640, 100, False),
    (4, 6000, 48, 640, 100, False),
    (3, 6000, 128, 2000, 500, False),
    (4, 6000, 24, 640, 100, False),
    (64, 8000, 32, 1024, 256, True),
])
def test_rerank_matches_oracle(T, L, H_I, kp, topk, shared):
    L_ = lib()
    k, q, w, n, cand = _case(T, L, H_I, kp, topk, shared, T * 7 + H_I)
    kd = dev(k[0] if shared else k, torch.bfloat16)
    qd, wd, nd, cd = dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32), dev(cand, torch.int32)
    idx, vals = L_.misa_hier_rerank(qd, wd, kd, nd, cd, topk)
    L_.misa_device_check()
    gi, gv = host(idx), host(vals)
    o = oracle.get()
    kf = np.broadcast_to(k, (T,) + k.shape[1:]) if shared else k
    stride = 0 if shared else L * 128
    F = o.dense_scores_at(q, w, k[0] if shared else k, stride, n, cand)
    for t in range(T):
        nt = int(n[t])
        ids, _ = o.rerank(q[t], w[t], kf[t], nt, cand[t], topk)
        vals_by_id = np.full(nt, np.nan)
        ok = (cand[t] >= 0) & (cand[t] < nt)
        vals_by_id[cand[t][ok]] = F[t][ok]
        tol = np.where(np.isnan(vals_by_id), np.inf, P.score_tol(q[t], w[t], kf[t], nt, None))
        P.check_selection(gi[t], ids, vals_by_id, tol, topk, f"rerank q{t}")
        sel = gi[t][gi[t] >= 0]
        P.check_close(gv[t][: len(sel)], vals_by_id[sel], tol[sel], f"rerank q{t} scores")
