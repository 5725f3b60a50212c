"""The bounds-checked build (libmisa_checked.so, MISA_CHECKED) on the GPU: ids outside their range
are skipped exactly as in the normal build, and counted by kind on the device.

A child process loads the checked library (MISA_LIBRARY=checked) and makes calls with host-made bad
inputs: a candidate list with ids past the prefix and negative ids other than the empty marker -1,
a page table with an out-of-pool page inside a prefix, routed-head lists with ids outside [0, H_I).
Each call's counts are read with misa_bad_index_counts; a clean call must leave them at zero, and
misa_device_check must report MISA_ERR_BAD_INDEX after a bad call.  The re-rank with bad ids must
select what the oracle selects when those ids are empty slots.  No kernel is made to fault: the
bad ids are exactly the ones every build already skips.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _child():
    """Runs in the child process (checked library loaded); prints one JSON line."""
    import torch

    import oracle
    import parity as P
    from gpu_common import dev, host
    from long_context_sparse_mean_b200 import build
    from long_context_sparse_mean_b200 import workloads as W

    build.build(checked=True)
    from long_context_sparse_mean_b200 import binding as M
    out = {"checked": M.checked_build()}
    M.misa_bad_index_counts()  # start from zero

    # re-rank with 5 ids past the prefix and 2 negative ids other than -1 in query 0
    L, T, kp, topk = 4096, 2, 1024, 256
    wl = W.small(2, L=L, n_seq=T, T=T, seed=9100)
    k, q, w, n, _ = W.decode_batch(wl)
    n = np.array([4000, 4096], np.int32)
    rng = np.random.default_rng(5)
    cand = np.stack([rng.choice(4000, kp, replace=False) for _ in range(T)]).astype(np.int32)
    cand[0, :10] = -1
    cand[0, 10:15] = 4000 + np.arange(5)
    cand[0, 15:17] = -7
    kd, qd, wd, nd = dev(k, torch.bfloat16), dev(q, torch.bfloat16), dev(w, torch.float32), dev(n, torch.int32)
    idx, _ = M.misa_hier_rerank(qd, wd, kd, nd, dev(cand, torch.int32), topk)
    out["rerank_counts"] = M.misa_bad_index_counts()
    o = oracle.get()
    F = o.dense_scores_at(q, w, k, L * 128, n, cand)
    gi = host(idx)
    for t in range(T):
        nt = int(n[t])
        ids, _ = o.rerank(q[t], w[t], k[t], nt, cand[t], topk)
        vals = np.full(nt, np.nan)
        ok = (cand[t] >= 0) & (cand[t] < nt)
        vals[cand[t][ok]] = F[t][ok]
        tol = np.where(np.isnan(vals), np.inf, P.score_tol(q[t], w[t], k[t], nt, None))
        P.check_selection(gi[t], ids, vals, tol, topk, f"checked re-rank q{t}")
    out["rerank_matches_oracle"] = True

    # the same re-rank with clean candidates: no counts, device check ok
    M.misa_hier_rerank(qd, wd, kd, nd, dev(np.abs(cand) % 4000, torch.int32), topk)
    out["clean_counts"] = M.misa_bad_index_counts()
    M.misa_device_check()

    # a bad call, then misa_device_check reports it
    M.misa_hier_rerank(qd, wd, kd, nd, dev(cand, torch.int32), topk)
    try:
        M.misa_device_check()
        out["device_check"] = "ok"
    except M.MisaError as e:
        out["device_check"] = e.status

    # paged scoring with one out-of-pool page (page 3 of sequence 1) inside the prefix
    ps, lp = 64, L // 64
    pool = torch.zeros((T * lp, ps, 128), dtype=torch.bfloat16, device="cuda")
    perm = torch.randperm(T * lp, generator=torch.Generator().manual_seed(3)).cuda()
    pool[perm] = kd.reshape(T * lp, ps, 128)
    table = perm.reshape(T, lp).to(torch.int32).contiguous()
    table[1, 3] = T * lp + 5
    heads = dev(np.tile(np.arange(8, dtype=np.int32), (T, 1)), torch.int32)
    M.misa_score_topk_paged(qd, wd, pool, table, nd, heads, topk, L=L)
    out["paged_counts"] = M.misa_bad_index_counts()

    # routed heads outside [0, H_I) in the block filter's head list
    bad_heads = np.tile(np.arange(8, dtype=np.int32), (T, 1))
    bad_heads[0, 2] = 64
    bad_heads[1, 5] = -3
    kbar = M.misa_pool_keys(kd, wl.B)
    M.misa_block_filter_topk(qd, wd, kd, kbar, nd, dev(bad_heads, torch.int32), wl.B, 4, topk)
    out["head_counts"] = M.misa_bad_index_counts()
    print(json.dumps(out))


def test_checked_build_counts_skipped_ids():
    env = dict(os.environ, MISA_LIBRARY="checked")
    code = ("import sys; sys.path[:0] = [%r, %r]; import test_gpu_checked as t; t._child()" % (ROOT, HERE))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["checked"] is True
    assert out["rerank_counts"] == [0, 7, 0], out
    assert out["rerank_matches_oracle"]
    assert out["clean_counts"] == [0, 0, 0], out
    assert out["device_check"] == 6, "MISA_ERR_BAD_INDEX after a bad call"
    assert out["paged_counts"] == [0, 0, 64], "one out-of-pool page of 64 keys inside a prefix"
    assert out["head_counts"][0] >= 2 and out["head_counts"][1:] == [0, 0], out
