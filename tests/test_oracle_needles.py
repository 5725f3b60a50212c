"""The planted needles of the 128K MISA-dagger decode workload are a real pin of the dense indexer.

"MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference", "Experimental
Results", "Needle-in-a-Haystack": retrieval stays complete up to 128K tokens.  The synthetic
stand-in plants 64 needle keys per sequence whose dense score provably exceeds every background
key's (the generator's sign and norm conditions), so the oracle's dense top-k must hold all of
them.  The oracle's MISA and MISA-dagger recalls are computed alongside; they depend on the
router and are reported by the GPU parity test, not asserted.
"""
import numpy as np

import oracle
from long_context_sparse_mean_b200 import workloads as W


def test_oracle_dense_top_k_holds_every_planted_needle():
    wl = W.WORKLOADS[4]
    seqs = [0, 17]
    k, q, w, n, needles = W.decode_batch(wl, seqs)
    L, d = k.shape[1], k.shape[2]
    o = oracle.get()
    dense = o.indexer(oracle.MODE_DSA, q, w, k, L * d, n, wl.B, wl.h, wl.topk)
    for a in range(len(seqs)):
        got = set(dense["idx"][a].tolist())
        missing = sorted(set(needles[a].tolist()) - got)
        assert not missing, f"sequence {seqs[a]}: needles {missing[:5]} not in the dense top-k"
        # the needles are the 64 largest dense scores: every needle beats every other selected key
        v = dict(zip(dense["idx"][a].tolist(), dense["idx_v"][a].tolist()))
        low = min(v[p] for p in needles[a].tolist())
        others = [x for p, x in v.items() if p not in set(needles[a].tolist())]
        assert low > max(others)


def test_needle_keys_meet_their_sign_conditions():
    """Every needle key has a negative dot product with each negative-weight head and a larger
    weighted projection on some positive head than any background key can score."""
    wl = W.small(4, L=8192, n_seq=3, T=3)
    for s in range(3):
        seq = W.decode_sequence(wl, s)
        q = seq.q.astype(np.float64)
        w = seq.w.astype(np.float64)
        mask = np.ones(wl.L, bool)
        mask[seq.needle_pos] = False
        kmax = np.linalg.norm(seq.k[mask].astype(np.float64), axis=1).max()
        S = (w[w > 0] * np.linalg.norm(q[w > 0], axis=1)).sum() * kmax
        for p in seq.needle_pos:
            kp = seq.k[p].astype(np.float64)
            assert np.all(q[w < 0] @ kp < 0)
            assert np.max(w[w > 0] * (q[w > 0] @ kp)) > 2 * S
