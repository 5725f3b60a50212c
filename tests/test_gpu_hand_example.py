"""The hand-computed fixture (tests/golden/hand_example.json) run through the CUDA path.

The 2-dimensional example is zero-padded to d = 128 and to H_I = 8 heads (padding heads have
q = 0 and w = 0, hence router score 0); all values are small integers, exact in bf16 and fp32,
so every GPU output must equal the hand-computed value exactly.
"""
import json
import os

import numpy as np
import pytest
import torch

from gpu_common import dev, host, lib

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_example.json")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_hand_example_on_gpu(dtype):
    L_ = lib()
    g = json.load(open(GOLDEN))
    k = np.zeros((5, 128), np.float32)
    k[:, :2] = g["keys"]
    q1 = np.zeros((8, 128), np.float32)
    q1[:3, :2] = g["q"]
    w1 = np.zeros(8, np.float32)
    w1[:3] = g["w"]
    ns = [qc["n"] for qc in g["queries"]]
    T = len(ns)
    kd = dev(k, dtype)
    qd = dev(np.stack([q1] * T), dtype)
    wd = dev(np.stack([w1] * T), torch.float32)
    nd = dev(np.array(ns, np.int32), torch.int32)
    B = g["B"]

    kbar = host(L_.misa_pool_keys(kd, B))
    assert np.array_equal(kbar[:, :2], np.array(g["queries"][0]["kbar"], np.float32))
    assert np.all(kbar[:, 2:] == 0)

    heads, r = L_.misa_route(qd, wd, kd, L_.misa_pool_keys(kd, B), nd, B, 1, want_r=True)
    r = host(r)
    for t, qc in enumerate(g["queries"]):
        assert np.array_equal(r[t, :3], np.array(qc["r"], np.float32)), (t, r[t])
        assert np.all(r[t, 3:] == 0)
        assert host(heads)[t].tolist() == qc["h1"]["heads"]

    I = host(L_.misa_token_scores(qd, wd, kd, nd, heads))
    for t, qc in enumerate(g["queries"]):
        assert np.array_equal(I[t, :qc["n"]], np.array(qc["h1"]["I"], np.float32))
    idx, vals = L_.misa_score_topk(qd, wd, kd, nd, heads, 2)
    for t, qc in enumerate(g["queries"]):
        assert sorted(host(idx)[t].tolist()) == sorted(qc["h1"]["top2"])

    q0 = g["queries"][0]
    one = dev(np.array([q0["n"]], np.int32), torch.int32)
    h2, _ = L_.misa_route(qd[:1], wd[:1], kd, L_.misa_pool_keys(kd, B), one, B, 2)
    assert host(h2)[0].tolist() == q0["h2"]["heads"]
    I2 = host(L_.misa_token_scores(qd[:1], wd[:1], kd, one, h2))[0]
    assert np.array_equal(I2, np.array(q0["h2"]["I"], np.float32))
    for kk, key in ((2, "top2"), (4, "top4")):
        idx2, _ = L_.misa_score_topk(qd[:1], wd[:1], kd, one, h2, kk)
        assert sorted(host(idx2)[0].tolist()) == sorted(q0["h2"][key])
        dix, dv = L_.dsa_dense_topk(qd[:1], wd[:1], kd, one, kk)
        assert sorted(host(dix)[0].tolist()) == sorted(q0["dense"][key])
    F = host(L_.misa_token_scores(qd[:1], wd[:1], kd, one, None))[0]
    assert np.array_equal(F, np.array(q0["dense"]["F"], np.float32))

    res = L_.misa_indexer(qd[:1], wd[:1], kd, L_.misa_pool_keys(kd, B), one, B, 1, 2, kp=3)
    assert sorted(host(res["cand"])[0].tolist()) == sorted(q0["dagger_h1_kp3"]["cand"])
    assert sorted(host(res["idx"])[0].tolist()) == sorted(q0["dagger_h1_kp3"]["top2"])
