"""Top-k selection of score rows (one CTA per row; for a few long rows the candidates are first
gathered across the GPU), against a stable sort of the same float32 values.  With exact ties going
to the lower index the selected set is unique, so the sets must be equal.  Row kinds cover the
sampled cut, the exact fallback when the sample's candidate list is short or overflows, rows whose
boundary bucket overflows shared memory (all scores equal), heavy ties, negative rows, prefixes up
to k (all taken) and short rows (list only), and row strides that break 16-byte alignment."""
import numpy as np
import pytest
import torch

from gpu_common import host, lib

pytestmark = pytest.mark.gpu


def _rows(T, L, seed):
    g = np.random.default_rng(seed)
    v = np.empty((T, L), np.float32)
    n = g.integers(0, L + 1, size=T).astype(np.int32)
    for t in range(T):
        kind = t % 8
        if kind == 0:
            v[t] = g.standard_normal(L)
        elif kind == 1:
            v[t] = 0.5                                   # one value: every boundary is a tie
        elif kind == 2:
            v[t] = g.integers(0, 5, size=L)              # five levels
        elif kind == 3:
            v[t] = 1.0
            v[t, g.choice(L, 100, replace=False)] = g.uniform(2, 3, 100)
        elif kind == 4:
            v[t] = -np.abs(g.standard_normal(L)) - 1.0   # negative scores
        elif kind == 5:
            v[t] = g.standard_normal(L)
            n[t] = g.integers(0, 2049)                   # at most k: all taken
        elif kind == 6:
            v[t] = g.standard_normal(L) * 1e-3
            n[t] = g.integers(2049, 8193)                # exact path
        else:
            v[t] = np.sort(g.standard_normal(L))         # ascending: the best keys at the end
    v[v == 0] = 0.0
    return v, n


@pytest.mark.parametrize("T,L,pad", [
    (320, 40000, 0),   # many rows: 2 CTAs of 512 threads per SM
    (320, 40000, 1),   # row stride not a multiple of 16 bytes
    (12, 40000, 0),    # a few long rows: candidates gathered across the GPU, then one CTA per row
    (12, 40000, 1),
    (40, 20000, 0),    # a few rows just longer than the 16384-entry list
])
def test_rows_match_stable_sort(T, L, pad):
    L_ = lib()
    k = 2048
    v, n = _rows(T, L, seed=pad + 1 + T)
    buf = torch.zeros((T, L + pad), dtype=torch.float32)
    buf[:, :L] = torch.from_numpy(v)
    sd = buf.cuda()
    nd = torch.from_numpy(n).cuda()
    ws = L_.Workspace(sd.device)
    idx, vals = L_.misa_topk_select(sd, nd, k, L=L, ws=ws)
    idx, vals = host(idx), host(vals)
    for t in range(T):
        nt = int(n[t])
        want = np.argsort(-v[t][:nt].astype(np.float64), kind="stable")[:k]
        got = idx[t]
        m = min(k, nt)
        assert np.all(got[m:] == -1), f"row {t}: padding"
        assert sorted(got[:m].tolist()) == sorted(want.tolist()), f"row {t} (kind {t % 8}, n={nt})"
        assert np.array_equal(vals[t][:m], v[t][got[:m]]), f"row {t}: values"
    L_.misa_device_check()
