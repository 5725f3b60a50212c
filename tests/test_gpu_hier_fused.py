"""The one-call MISA-dagger decode (misa_hier_topk_fused) against the oracle.

The routed heads are the oracle's, so what is under test is the routed scoring, the sampled cut, the
dense scores kept while the keys are read, the top-k' by the routed score and the top-k by the dense
score.  The GPU's candidate set is its exact top-k' with those heads (misa_score_topk); where it
equals the oracle's (it differs only inside the routed score's tie band, which the parity tests
count), the final selection must be the oracle's top-k of the dense score up to that score's tie
band, and the returned values must be the dense scores.

Cases: the 32 x 131072 decode batch of the MISA-dagger workload (every row takes the dense lists);
prefixes of mixed lengths around the list cap (16384) and below k' and k (rows without lists are
answered exactly from their score rows); exact ties at both cuts and a row whose keys are all equal
(its list overflows); head pools of 32 and 128 with h = 4 and h = 8; k' = k and k' = 16384."""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib, report
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(name, k, q, w, n, B, h, kp, topk, max_skipped=0):
    L_ = lib()
    o = oracle.get()
    T, L, d = k.shape
    kd, qd = dev(k, torch.bfloat16), dev(q, torch.bfloat16)
    wd, nd = dev(w, torch.float32), dev(n, torch.int32)
    orc = o.indexer(oracle.MODE_DAGGER, q, w, k, L * d, n, B, h, topk, kp=kp)
    oh = dev(orc["heads"], torch.int32)
    fi, fv = L_.misa_hier_topk_fused(qd, wd, kd, nd, oh, kp, topk)
    L_.misa_device_check()
    fi, fv = host(fi), host(fv)
    cand_g = host(L_.misa_score_topk(qd, wd, kd, nd, oh, kp, want_vals=False)[0])
    F = o.dense_scores_at(q, w, k, L * d, n, orc["cand"])
    swaps = skipped = 0
    for t in range(T):
        nt = int(n[t])
        oc = orc["cand"][t]
        ok = (oc >= 0) & (oc < nt)
        gc = cand_g[t][cand_g[t] >= 0]
        if set(gc.tolist()) != set(oc[ok].tolist()):
            skipped += 1
            continue
        Fv = np.full(nt, np.nan)
        Fv[oc[ok]] = F[t][ok]
        tol = np.where(np.isnan(Fv), np.inf, P.score_tol(q[t], w[t], k[t], nt, None))
        rep = P.check_selection(fi[t], orc["idx"][t], Fv, tol, topk, f"{name} q{t} fused MISA-dagger")
        swaps += rep.swaps
        sel = fi[t][fi[t] >= 0]
        assert np.all(fi[t][len(sel):] == -1), f"{name} q{t}: -1 padding not at the end"
        P.check_close(fv[t][: len(sel)], Fv[sel], tol[sel], f"{name} q{t} fused dense scores")
    assert skipped <= max_skipped, f"{name}: {skipped} rows with a candidate set outside the oracle's"
    report(name, checked_queries=T - skipped, skipped_cand_band=skipped, final_swaps=swaps)


def test_decode_128k_batch():
    wl = W.WORKLOADS[4]
    k, q, w, n, _ = W.decode_batch(wl)
    _run("hier_fused_cfg4", k, q, w, n, wl.B, wl.h, wl.kp, wl.topk)


def test_mixed_lengths_around_the_cap():
    wl = W.small(4, L=40000, n_seq=8, T=8, needles=None)
    k, q, w, _, _ = W.decode_batch(wl)
    n = np.array([40000, 31000, 16385, 16384, 12000, 5000, 1500, 100], np.int32)
    _run("hier_fused_lengths", k, q, w, n, wl.B, wl.h, 4096, 1024)


def test_ties_and_an_overflowing_list():
    wl = W.small(4, L=24000, n_seq=4, T=4, needles=None)
    k, q, w, n, _ = W.decode_batch(wl)
    rng = np.random.default_rng(11)
    k[0, :] = k[0, 7]  # every key equal: every score ties, the list overflows
    protos = k[1, rng.choice(wl.L, 3, replace=False)].copy()
    k[1] = protos[rng.integers(0, 3, wl.L)]  # three distinct keys: exact ties at both cuts
    k[2, ::5] = k[2, 3]  # a fifth of the row shares one key
    _run("hier_fused_ties", k, q, w, n, wl.B, wl.h, 4096, 1000)


@pytest.mark.parametrize("H_I,h", [(32, 4), (128, 8)])
def test_head_pools(H_I, h):
    wl = W.small(4, H_I=H_I, h=h, L=30000, n_seq=3, T=3, needles=None)
    k, q, w, n, _ = W.decode_batch(wl)
    _run(f"hier_fused_H{H_I}_h{h}", k, q, w, n, wl.B, h, 8192, 2048)


@pytest.mark.parametrize("kp,topk", [(2048, 2048), (16384, 2048)])
def test_candidate_counts(kp, topk):
    wl = W.small(4, L=50000, n_seq=3, T=3, needles=None)
    k, q, w, n, _ = W.decode_batch(wl)
    _run(f"hier_fused_kp{kp}", k, q, w, n, wl.B, wl.h, kp, topk)
