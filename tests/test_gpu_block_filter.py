"""The token-axis block filter composed with MISA on the GPU against the oracle ("HISA: Efficient
Hierarchical Indexing for Fine-Grained Sparse Attention", abstract: pooled block representatives
scored, the best blocks kept, the indexer run on their tokens only).

Stage-wise: the GPU is given the oracle's routed heads, so nothing flows from the GPU into the
oracle.  Block scores are compared element by element (parity.block_tol), the kept blocks and the
selected tokens with the tie-band rule; when the kept block sets agree, the token selection is
checked against the oracle's over the same kept tokens.  Cases: per-query caches and one shared
cache, bf16 and fp32, ragged prefixes (partial last blocks, prefixes shorter than a block, empty),
m below, at and above the number of blocks, B = 1, all heads routed.
"""
import numpy as np
import pytest
import torch

import oracle
import parity as P
from gpu_common import dev, host, lib, report
from long_context_sparse_mean_b200 import workloads as W

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}
SENTINEL = -7.0


def _inputs(shared, dtype, L, T, H_I, seed):
    if shared:
        wl = W.small(3, L=L, T=T, chunk=T, H_I=H_I, dtype=dtype, seed=2000 + seed)
        k = W.shared_keys(wl)
        q, w = W.shared_queries(wl, 0, wl.T)
        return k, q, w, 0
    wl = W.small(2, L=L, n_seq=T, T=T, H_I=H_I, dtype=dtype, seed=2000 + seed)
    k, q, w, _, _ = W.decode_batch(wl)
    return k, q, w, L * 128


def _run_case(name, shared, dtype, L, H_I, B, h, m, topk, ns, seed=0):
    L_ = lib()
    ns = np.asarray(ns, np.int32)
    T = len(ns)
    k, q, w, kss = _inputs(shared, dtype, L, T, H_I, seed)
    q, w = q[:T], w[:T]
    kt = (lambda t: k) if shared else (lambda t: k[t])
    o = oracle.get()
    _, oh = o.route_batch(q, w, k, kss, ns, B, h)
    orc = o.block_filter(q, w, k, kss, ns, B, h, m, topk, heads_in=oh)
    I_o = o.scores(q, w, k, kss, ns, heads=oh, ld=L)

    kd, qd = dev(k, DT[dtype]), dev(q, DT[dtype])
    wd, nd, hd = dev(w, torch.float32), dev(ns, torch.int32), dev(oh, torch.int32)
    kbar = L_.misa_pool_keys(kd, B)
    M = -(-L // B)
    S_d = torch.full((T, M), SENTINEL, dtype=torch.float32, device="cuda")
    res = L_.misa_block_filter_topk(qd, wd, kd, kbar, nd, hd, B, m, topk, block_scores=S_d)
    torch.cuda.synchronize()
    S_g, bl, idx, vals = host(S_d), host(res["blocks"]), host(res["idx"]), host(res["vals"])
    L_.misa_device_check()

    block_swaps = token_swaps = compared = 0
    for t in range(T):
        nt = int(ns[t])
        Mt = -(-nt // B)
        tag = f"{name} q{t} n={nt}"
        assert np.all(S_g[t][Mt:] == SENTINEL), f"{tag}: block scores written past M_t"
        if nt == 0:
            assert np.all(bl[t] == -1) and np.all(idx[t] == -1), f"{tag}: empty prefix selects nothing"
            continue
        bt = P.block_tol(q[t], w[t], kt(t), nt, B, oh[t])
        P.check_close(S_g[t][:Mt], orc["S"][t][:Mt], bt, f"{tag} block scores")
        block_swaps += P.check_selection(bl[t], orc["blocks"][t], orc["S"][t][:Mt], bt, m, f"{tag} blocks").swaps
        if set(bl[t][bl[t] >= 0].tolist()) != set(orc["blocks"][t][orc["blocks"][t] >= 0].tolist()):
            continue
        compared += 1
        kept = np.zeros(nt, bool)
        for b in orc["blocks"][t][orc["blocks"][t] >= 0]:
            kept[b * B:min((b + 1) * B, nt)] = True
        vals_o = np.where(kept, I_o[t][:nt], np.nan)
        st = np.where(kept, P.score_tol(q[t], w[t], kt(t), nt, oh[t]), np.inf)
        token_swaps += P.check_selection(idx[t], orc["idx"][t], vals_o, st, topk, f"{tag} tokens").swaps
        sel = idx[t][idx[t] >= 0]
        assert np.all(kept[sel]), f"{tag}: selected token outside the kept blocks"
        P.check_close(vals[t][:len(sel)], I_o[t][sel], st[sel], f"{tag} selected scores")
    assert compared > 0, f"{name}: no query with matching kept blocks"
    report(name, block_swaps=block_swaps, token_swaps=token_swaps, queries=T, compared=compared)


@pytest.mark.parametrize("m", [1, 8, 64, 100])
def test_per_query_caches(m):
    """Eight decode-style caches of 8192 keys (B = 128, 64 blocks): full, partial-block and
    short prefixes; m = 64 keeps every block of a full prefix, m = 100 more blocks than exist."""
    ns = [8192, 8191, 8000, 5000, 129, 128, 64, 0]
    _run_case(f"block filter per-query m={m}", False, "bf16", 8192, 64, 128, 8, m, 512, ns, seed=m)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shared_cache_ragged(dtype):
    """One shared cache of 3001 keys, prefixes around block boundaries (B = 64)."""
    ns = [0, 1, 2, 15, 63, 64, 65, 1000, 2999, 3001]
    _run_case(f"block filter shared {dtype}", True, dtype, 3001, 64, 64, 8, 12, 256, ns, seed=7)


def test_every_block_kept_is_misa():
    """m >= M_t keeps every block: the selection must be MISA's (oracle MISA top-k, tie band)."""
    L_ = lib()
    L, B, h, topk = 4096, 64, 8, 256
    ns = np.array([4096, 4000, 700, 64], np.int32)
    k, q, w, kss = _inputs(False, "bf16", L, len(ns), 64, seed=11)
    q, w = q[:len(ns)], w[:len(ns)]
    o = oracle.get()
    _, oh = o.route_batch(q, w, k, kss, ns, B, h)
    misa = o.indexer(oracle.MODE_MISA, q, w, k, kss, ns, B, h, topk, heads_in=oh)
    I_o = o.scores(q, w, k, kss, ns, heads=oh, ld=L)
    kd, qd = dev(k, torch.bfloat16), dev(q, torch.bfloat16)
    res = L_.misa_block_filter_topk(qd, dev(w, torch.float32), kd, L_.misa_pool_keys(kd, B), dev(ns, torch.int32),
                                    dev(oh, torch.int32), B, L // B, topk)
    idx, bl = host(res["idx"]), host(res["blocks"])
    for t, nt in enumerate(ns.tolist()):
        Mt = -(-nt // B)
        assert sorted(bl[t][:Mt].tolist()) == list(range(Mt)) and np.all(bl[t][Mt:] == -1), f"q{t}: every block"
        st = P.score_tol(q[t], w[t], k[t], nt, oh[t])
        P.check_selection(idx[t], misa["idx"][t], I_o[t][:nt], st, topk, f"q{t} every block kept")


def test_one_key_blocks():
    """B = 1: every key is its own block (its pooled key is the key itself)."""
    ns = [2000, 1999, 333, 1]
    _run_case("block filter B=1", False, "bf16", 2000, 64, 1, 8, 300, 100, ns, seed=13)


def test_all_heads_routed():
    """h = H_I (the block filter on the dense indexer), H_I = 32 and 128 (64 KB of staged q rows)."""
    ns = [4096, 3000, 130]
    _run_case("block filter h=H_I=32", False, "bf16", 4096, 32, 128, 32, 6, 300, ns, seed=17)
    _run_case("block filter h=H_I=128", False, "bf16", 4096, 128, 128, 128, 6, 300, ns, seed=19)


def test_end_to_end_with_router():
    """misa_indexer(m=...): the GPU router's heads feed the block filter; checked against the
    oracle where the routed sets agree."""
    L_ = lib()
    L, B, h, m, topk = 8192, 128, 8, 16, 512
    ns = np.array([8192, 6000, 4097, 300], np.int32)
    k, q, w, kss = _inputs(False, "bf16", L, len(ns), 64, seed=23)
    q, w = q[:len(ns)], w[:len(ns)]
    kd, qd = dev(k, torch.bfloat16), dev(q, torch.bfloat16)
    res = L_.misa_indexer(qd, dev(w, torch.float32), kd, L_.misa_pool_keys(kd, B), dev(ns, torch.int32), B, h, topk,
                          m=m)
    o = oracle.get()
    orc = o.block_filter(q, w, k, kss, ns, B, h, m, topk)
    heads, bl, idx = host(res["heads"]), host(res["blocks"]), host(res["idx"])
    agree = 0
    for t, nt in enumerate(ns.tolist()):
        rt = P.router_tol(q[t], w[t], k[t], nt, B)
        P.check_selection(heads[t], orc["heads"][t], orc["r"][t], rt, h, f"q{t} heads")
        if set(heads[t].tolist()) != set(orc["heads"][t].tolist()):
            continue
        Mt = -(-nt // B)
        bt = P.block_tol(q[t], w[t], k[t], nt, B, orc["heads"][t])
        P.check_selection(bl[t], orc["blocks"][t], orc["S"][t][:Mt], bt, m, f"q{t} blocks")
        if set(bl[t].tolist()) == set(orc["blocks"][t].tolist()):
            agree += 1
            sel = set(idx[t][idx[t] >= 0].tolist())
            assert all(any(b * B <= s < (b + 1) * B for b in orc["blocks"][t]) for s in sel), f"q{t} outside blocks"
    assert agree > 0
