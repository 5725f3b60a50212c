"""CUDA path against the CPU oracle on the five workloads, at full size.

The GPU runs every workload whole, in the launch configuration the benchmark uses.  The oracle
checks every query of the decode workloads (configs 1, 2, 4 and 5, the dense indexer on every
sequence too) and, in prefill, every query of the first and last 128-query tile of the first and
last chunk plus block and chunk edges and seeded queries spread over every chunk.  A few queries
sharing one 128K cache (the multi-query decode regime on the tensor cores) run the whole
MISA-dagger path.  On the 128K MISA-dagger workload the planted needles must all be in the GPU's
dense top-k.

Per sampled query:
  * pooled keys, router scores and routed heads against the oracle (tie band on r);
  * stage-wise: the GPU scores every prefix token with the ORACLE's routed heads (oracle -> GPU
    only) and its top-k is compared with the oracle's under the tie-band rule;
  * end-to-end: the GPU's own routed pass against the oracle's, for queries whose routed head
    sets agree (queries whose head sets differ inside the tie band are counted and reported);
  * MISA-dagger: the GPU re-ranks the ORACLE's candidate set and must keep the oracle's final
    tokens (tie band on the dense score); end-to-end final sets are compared when the candidate
    sets agree, and the token recovery (IoU) against the dense indexer is reported;
  * the dense indexer (h = H_I) against the oracle's dense top-k.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, kdtype, lib, report
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _iou(a, b):
    a = set(np.asarray(a)[np.asarray(a) >= 0].tolist())
    b = set(np.asarray(b)[np.asarray(b) >= 0].tolist())
    return len(a & b) / max(1, len(a | b))


def _check_query(name, wl, i, q, w, kseq, n, gpu, orc, stats, dag=None):
    """Checks of one query; gpu and orc are dicts of per-query arrays."""
    B, h = wl.B, wl.h
    # pooled keys (decode caches: the whole cache is pooled)
    if "kbar" in gpu:
        kb_o = oracle.get().pool_keys(kseq, B, n)
        P.check_close(gpu["kbar"][: kb_o.shape[0]].ravel(), kb_o.ravel(), P.pool_tol(kseq, n, B, kb_o).ravel(),
                      f"{name} q{i} kbar")
    # router
    rt = P.router_tol(q, w, kseq, n, B)
    P.check_close(gpu["r"], orc["r"], rt, f"{name} q{i} router scores")
    rep = P.check_selection(gpu["heads"], orc["heads"], orc["r"], rt, h, f"{name} q{i} routed heads")
    stats["head_swaps"] += rep.swaps
    heads_same = set(gpu["heads"].tolist()) == set(orc["heads"].tolist())
    # stage-wise scoring with the oracle's heads
    st = P.score_tol(q, w, kseq, n, orc["heads"])
    I_o = orc["I"][:n]
    P.check_close(gpu["I_oh"][:n], I_o, st, f"{name} q{i} token scores")
    kk = wl.kp if dag is not None else wl.topk
    rep = P.check_selection(gpu["idx_oh"], orc["top_I"], I_o, st, kk, f"{name} q{i} top-k (oracle heads)")
    stats["token_swaps"] += rep.swaps
    # end-to-end routed pass
    if heads_same:
        rep = P.check_selection(gpu["sel"], orc["top_I"], I_o, st, kk, f"{name} q{i} top-k end-to-end")
        stats["e2e_token_swaps"] += rep.swaps
    else:
        stats["e2e_skipped_head_band"] += 1
    if dag is not None:
        # MISA-dagger fine stage on the oracle's candidates
        cand = orc["top_I"]
        F_c = dag["F_cand"]
        Fv = np.full(n, np.nan)
        Fv[cand[cand >= 0]] = F_c[cand >= 0]
        ft = np.full(n, np.inf)
        ct = P.score_tol(q, w, kseq, n, None)
        ft[cand[cand >= 0]] = ct[cand[cand >= 0]]
        rep = P.check_selection(gpu["fin_oc"], dag["fin"], Fv, ft, wl.topk, f"{name} q{i} re-rank (oracle cand)")
        stats["rerank_swaps"] += rep.swaps
        sel = gpu["fin_oc"][gpu["fin_oc"] >= 0]
        P.check_close(gpu["fin_oc_v"][: len(sel)], Fv[sel], ct[sel], f"{name} q{i} re-rank scores")
        if heads_same and set(gpu["sel"].tolist()) == set(cand.tolist()):
            rep = P.check_selection(gpu["fin"], dag["fin"], Fv, ft, wl.topk, f"{name} q{i} MISA-dagger end-to-end")
            stats["e2e_final_swaps"] += rep.swaps
        else:
            stats["e2e_final_skipped_cand_band"] += 1


def _decode_case(name, wl, check_seqs, dense_seqs=(), run_dagger=None):
    L_ = lib()
    run_dagger = wl.kp is not None if run_dagger is None else run_dagger
    k, q, w, n, needles = W.decode_batch(wl)
    S, L, d = k.shape
    dt = kdtype(wl)
    kd, qd = dev(k, dt), dev(q, dt)
    wd, nd = dev(w, torch.float32), dev(n, torch.int32)
    B, h = wl.B, wl.h
    kbar = L_.misa_pool_keys(kd, B)
    heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    kk = wl.kp if run_dagger else wl.topk
    sel, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, kk)
    fin = None
    if run_dagger:
        fin, _ = L_.misa_hier_rerank(qd, wd, kd, nd, sel, wl.topk)
    gdense = L_.dsa_dense_topk(qd, wd, kd, nd, wl.topk)[0] if dense_seqs else None

    sel_i = np.array(check_seqs)
    mode = oracle.MODE_DAGGER if run_dagger else oracle.MODE_MISA
    orc = oracle.get().indexer(mode, q[sel_i], w[sel_i], k[sel_i], L * d, n[sel_i], B, h, wl.topk,
                               kp=wl.kp or 0)
    top_I = orc["cand"] if run_dagger else orc["idx"]
    # stage-wise GPU runs fed with oracle outputs
    qs, ws_, ns_ = qd[sel_i], wd[sel_i], nd[sel_i]
    ks = kd[sel_i].contiguous()
    oh = dev(orc["heads"], torch.int32)
    I_oh = host(L_.misa_token_scores(qs, ws_, ks, ns_, oh))
    idx_oh, _ = L_.misa_score_topk(qs, ws_, ks, ns_, oh, kk)
    I_o = oracle.get().scores(q[sel_i], w[sel_i], k[sel_i], L * d, n[sel_i], heads=orc["heads"], ld=L)
    fin_oc = fin_oc_v = F_cand = None
    if run_dagger:
        oc = dev(orc["cand"], torch.int32)
        fo, fv = L_.misa_hier_rerank(qs, ws_, ks, ns_, oc, wl.topk)
        fin_oc, fin_oc_v = host(fo), host(fv)
        F_cand = oracle.get().dense_scores_at(q[sel_i], w[sel_i], k[sel_i], L * d, n[sel_i], orc["cand"])
    stats = dict(head_swaps=0, token_swaps=0, e2e_token_swaps=0, e2e_skipped_head_band=0, rerank_swaps=0,
                 e2e_final_swaps=0, e2e_final_skipped_cand_band=0)
    kbar_h, r_h, heads_h, sel_h = host(kbar), host(r), host(heads), host(sel)
    fin_h = host(fin) if fin is not None else None
    idx_oh_h = host(idx_oh)
    for a, s in enumerate(check_seqs):
        gpu = {"kbar": kbar_h[s], "r": r_h[s], "heads": heads_h[s], "I_oh": I_oh[a], "idx_oh": idx_oh_h[a],
               "sel": sel_h[s]}
        o = {"r": orc["r"][a], "heads": orc["heads"][a], "I": I_o[a], "top_I": top_I[a]}
        dag = None
        if run_dagger:
            gpu.update(fin_oc=fin_oc[a], fin_oc_v=fin_oc_v[a], fin=fin_h[s])
            dag = {"F_cand": F_cand[a], "fin": orc["idx"][a]}
        _check_query(name, wl, s, q[s], w[s], k[s], int(n[s]), gpu, o, stats, dag)
    extra = {}
    if needles[0] is not None:
        final = fin_h if run_dagger else sel_h
        extra["needle_recall_gpu"] = float(np.mean([len(set(needles[s]) & set(final[s])) / len(needles[s])
                                                    for s in range(S)]))
    if dense_seqs:
        di = np.array(dense_seqs)
        od = oracle.get().indexer(oracle.MODE_DSA, q[di], w[di], k[di], L * d, n[di], B, h, wl.topk)
        F_all = oracle.get().scores(q[di], w[di], k[di], L * d, n[di], ld=L)
        gd = host(gdense)
        ious = []
        for a, s in enumerate(dense_seqs):
            ft = P.score_tol(q[s], w[s], k[s], int(n[s]), None)
            rep = P.check_selection(gd[s], od["idx"][a], F_all[a], ft, wl.topk, f"{name} q{s} dense top-k")
            stats["token_swaps"] += rep.swaps
            ious.append(_iou(fin_h[s] if run_dagger else sel_h[s], gd[s]))
        extra["iou_vs_dense"] = float(np.mean(ious))
        if needles[0] is not None:
            rec = [len(set(needles[s]) & set(gd[s])) / len(needles[s]) for s in dense_seqs]
            extra["needle_recall_dense_gpu"] = float(np.mean(rec))
            # the planted needles outscore every background key under the dense indexer
            assert min(rec) == 1.0, f"{name}: dense top-k misses planted needles (recall {rec})"
            if run_dagger:
                extra["needle_recall_misa_gpu"] = float(np.mean(
                    [len(set(needles[s]) & set(sel_h[s])) / len(needles[s]) for s in range(S)]))
    report(name, checked_queries=len(check_seqs), **stats, **extra)
    return stats


def test_config1_tiny_fp32():
    wl = W.WORKLOADS[1]
    L_ = lib()
    inp = W.shared_inputs(wl)
    dt = kdtype(wl)
    kd, qd = dev(inp.k, dt), dev(inp.q, dt)
    wd, nd = dev(inp.w, torch.float32), dev(inp.n, torch.int32)
    B, h, kk, kp = wl.B, wl.h, wl.topk, 4 * wl.topk
    kbar = L_.misa_pool_keys(kd, B)
    heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    sel, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, kp)
    fin, _ = L_.misa_hier_rerank(qd, wd, kd, nd, sel, kk)
    sel_k, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, kk)
    gd, _ = L_.dsa_dense_topk(qd, wd, kd, nd, kk)
    o = oracle.get()
    orc = o.indexer(oracle.MODE_DAGGER, inp.q, inp.w, inp.k, 0, inp.n, B, h, kk, kp=kp)
    orc_m = o.indexer(oracle.MODE_MISA, inp.q, inp.w, inp.k, 0, inp.n, B, h, kk)
    orc_d = o.indexer(oracle.MODE_DSA, inp.q, inp.w, inp.k, 0, inp.n, B, h, kk)
    oh = dev(orc["heads"], torch.int32)
    I_oh = host(L_.misa_token_scores(qd, wd, kd, nd, oh))
    idx_oh, _ = L_.misa_score_topk(qd, wd, kd, nd, oh, kp)
    fo, fv = L_.misa_hier_rerank(qd, wd, kd, nd, dev(orc["cand"], torch.int32), kk)
    I_o = o.scores(inp.q, inp.w, inp.k, 0, inp.n, heads=orc["heads"], ld=wl.L)
    F_all = o.scores(inp.q, inp.w, inp.k, 0, inp.n, ld=wl.L)
    kb = host(kbar)
    kb_o = o.pool_keys(inp.k, B)
    P.check_close(kb.ravel(), kb_o.ravel(), P.pool_tol(inp.k, wl.L, B, kb_o).ravel(), "cfg1 kbar")
    stats = dict(head_swaps=0, token_swaps=0, e2e_token_swaps=0, e2e_skipped_head_band=0, rerank_swaps=0,
                 e2e_final_swaps=0, e2e_final_skipped_cand_band=0)
    hh, rr, ss, ff, iohh, fo_h, fv_h = (host(x) for x in (heads, r, sel, fin, idx_oh, fo, fv))
    sk, gdh = host(sel_k), host(gd)
    for t in range(wl.T):
        n = int(inp.n[t])
        gpu = {"r": rr[t], "heads": hh[t], "I_oh": I_oh[t], "idx_oh": iohh[t], "sel": ss[t], "fin_oc": fo_h[t],
               "fin_oc_v": fv_h[t], "fin": ff[t]}
        og = {"r": orc["r"][t], "heads": orc["heads"][t], "I": I_o[t], "top_I": orc["cand"][t]}
        F_c = np.where(orc["cand"][t] >= 0, F_all[t][np.maximum(orc["cand"][t], 0)], 0.0)
        _check_query("cfg1", wl, t, inp.q[t], inp.w[t], inp.k, n, gpu, og, stats,
                     {"F_cand": F_c, "fin": orc["idx"][t]})
        st = P.score_tol(inp.q[t], inp.w[t], inp.k, n, orc["heads"][t])
        if set(hh[t].tolist()) == set(orc["heads"][t].tolist()):
            P.check_selection(sk[t], orc_m["idx"][t], I_o[t][:n], st, kk, f"cfg1 q{t} MISA top-k")
        ft = P.score_tol(inp.q[t], inp.w[t], inp.k, n, None)
        P.check_selection(gdh[t], orc_d["idx"][t], F_all[t][:n], ft, kk, f"cfg1 q{t} dense top-k")
        for res in (sk[t], ff[t], gdh[t]):
            assert set(inp.needle_pos.tolist()) <= set(res.tolist()), "planted needles selected"
        assert set(inp.needle_heads.tolist()) <= set(hh[t].tolist()), "needle heads routed"
    report("cfg1_tiny_fp32", checked_queries=wl.T, **stats)


def test_config2_decode_32k():
    wl = W.WORKLOADS[2]
    every = list(range(wl.n_seq))
    _decode_case("cfg2_decode_32k", wl, every, dense_seqs=every, run_dagger=False)


def test_config4_misa_dagger_128k():
    wl = W.WORKLOADS[4]
    every = list(range(wl.n_seq))
    _decode_case("cfg4_misa_dagger_128k", wl, every, dense_seqs=every)


def test_config5_glm5_128k():
    wl = W.WORKLOADS[5]
    every = list(range(wl.n_seq))
    _decode_case("cfg5_glm5_128k", wl, every, dense_seqs=every, run_dagger=False)


def _prefill_sample(wl):
    """Every query of the first and the last 128-query tile of the first and the last chunk, block
    and chunk edges, and seeded queries spread over the whole prefill."""
    ch = wl.chunk
    tiles = []
    for c0 in (0, wl.T - ch):
        tiles += list(range(c0, c0 + 128)) + list(range(c0 + ch - 128, c0 + ch))
    fixed = [0, 1, 2, 63, 64, 127, 128, 129, 255, 256, 4095, 4096, 4097, 8191, 32767, 32768, 65407, 65408,
             65534, 65535]
    rng = np.random.default_rng(3)
    extra = rng.choice(wl.T, 64, replace=False).tolist()
    return sorted(set(t for t in tiles + fixed + extra if t < wl.T))


def test_config3_prefill_64k():
    wl = W.WORKLOADS[3]
    L_ = lib()
    k = W.shared_keys(wl)
    kd = dev(k, kdtype(wl))
    B, h, kk, ch = wl.B, wl.h, wl.topk, wl.chunk
    kbar = L_.misa_pool_keys(kd, B)
    sample = _prefill_sample(wl)
    want = {}
    scores_buf = torch.empty((ch, wl.L), dtype=torch.float32, device="cuda")
    for c0 in range(0, wl.T, ch):
        q, w = W.shared_queries(wl, c0, c0 + ch)
        n = W.prefix_lengths(wl, c0, c0 + ch)
        qd, wd, nd = dev(q, kdtype(wl)), dev(w, torch.float32), dev(n, torch.int32)
        heads, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
        sel, _ = L_.misa_score_topk(qd, wd, kd, nd, heads, kk, scores_full=scores_buf)
        for t in sample:
            if c0 <= t < c0 + ch:
                a = t - c0
                want[t] = dict(q=q[a], w=w[a], n=int(n[a]), r=host(r[a]), heads=host(heads[a]), sel=host(sel[a]))
    ts = sorted(want)
    q = np.stack([want[t]["q"] for t in ts])
    w = np.stack([want[t]["w"] for t in ts])
    n = np.array([want[t]["n"] for t in ts], np.int32)
    o = oracle.get()
    orc = o.indexer(oracle.MODE_MISA, q, w, k, 0, n, B, h, kk)
    qd, wd, nd = dev(q, kdtype(wl)), dev(w, torch.float32), dev(n, torch.int32)
    oh = dev(orc["heads"], torch.int32)
    I_oh = host(L_.misa_token_scores(qd, wd, kd, nd, oh))
    idx_oh = host(L_.misa_score_topk(qd, wd, kd, nd, oh, kk)[0])
    I_o = o.scores(q, w, k, 0, n, heads=orc["heads"], ld=wl.L)
    stats = dict(head_swaps=0, token_swaps=0, e2e_token_swaps=0, e2e_skipped_head_band=0, rerank_swaps=0,
                 e2e_final_swaps=0, e2e_final_skipped_cand_band=0)
    for a, t in enumerate(ts):
        gpu = {"r": want[t]["r"], "heads": want[t]["heads"], "I_oh": I_oh[a], "idx_oh": idx_oh[a],
               "sel": want[t]["sel"]}
        og = {"r": orc["r"][a], "heads": orc["heads"][a], "I": I_o[a], "top_I": orc["idx"][a]}
        _check_query("cfg3", wl, t, q[a], w[a], k, int(n[a]), gpu, og, stats)
    report("cfg3_prefill_64k", checked_queries=len(ts), **stats)


def test_shared_cache_few_queries_128k_misa_dagger():
    """Four queries on one shared 131072-key bf16 cache (speculative or multi-token decode) through
    the whole MISA-dagger path: router, routed scores on the tensor cores, top-k', dense re-rank."""
    wl = W.small(3, name="shared_L131072_T4", L=131072, T=4, chunk=None, kp=8192)
    L_ = lib()
    inp = W.shared_inputs(wl)
    dt = kdtype(wl)
    kd, qd = dev(inp.k, dt), dev(inp.q, dt)
    wd, nd = dev(inp.w, torch.float32), dev(inp.n, torch.int32)
    B, h, kk, kp = wl.B, wl.h, wl.topk, wl.kp
    kbar = L_.misa_pool_keys(kd, B)
    res = L_.misa_indexer(qd, wd, kd, kbar, nd, B, h, kk, kp=kp)
    _, r = L_.misa_route(qd, wd, kd, kbar, nd, B, h, want_r=True)
    o = oracle.get()
    orc = o.indexer(oracle.MODE_DAGGER, inp.q, inp.w, inp.k, 0, inp.n, B, h, kk, kp=kp)
    oh = dev(orc["heads"], torch.int32)
    I_oh = host(L_.misa_token_scores(qd, wd, kd, nd, oh))
    idx_oh, _ = L_.misa_score_topk(qd, wd, kd, nd, oh, kp)
    fo, fv = L_.misa_hier_rerank(qd, wd, kd, nd, dev(orc["cand"], torch.int32), kk)
    I_o = o.scores(inp.q, inp.w, inp.k, 0, inp.n, heads=orc["heads"], ld=wl.L)
    F_c = o.dense_scores_at(inp.q, inp.w, inp.k, 0, inp.n, orc["cand"])
    stats = dict(head_swaps=0, token_swaps=0, e2e_token_swaps=0, e2e_skipped_head_band=0, rerank_swaps=0,
                 e2e_final_swaps=0, e2e_final_skipped_cand_band=0)
    hh, rr, cc, ff = host(res["heads"]), host(r), host(res["cand"]), host(res["idx"])
    iohh, fo_h, fv_h = host(idx_oh), host(fo), host(fv)
    for t in range(wl.T):
        gpu = {"r": rr[t], "heads": hh[t], "I_oh": I_oh[t], "idx_oh": iohh[t], "sel": cc[t], "fin_oc": fo_h[t],
               "fin_oc_v": fv_h[t], "fin": ff[t]}
        og = {"r": orc["r"][t], "heads": orc["heads"][t], "I": I_o[t], "top_I": orc["cand"][t]}
        _check_query("shared_L131072_T4", wl, t, inp.q[t], inp.w[t], inp.k, int(inp.n[t]), gpu, og, stats,
                     {"F_cand": F_c[t], "fin": orc["idx"][t]})
    report("shared_L131072_T4_misa_dagger", checked_queries=wl.T, **stats)
