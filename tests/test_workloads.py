"""The seeded input generator: determinism, shapes, bf16 rounding and planted structure."""
import numpy as np
import torch

from long_context_sparse_mean_b200 import workloads as W


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    x[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]  # exact ties round to even
    ours = W.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_deterministic_and_independent_sequences():
    wl = W.small(4, L=2048, n_seq=3, T=3)
    a = W.decode_sequence(wl, 1)
    b = W.decode_sequence(wl, 1)
    c = W.decode_sequence(wl, 2)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.q, b.q) and np.array_equal(a.w, b.w)
    assert not np.array_equal(a.k, c.k)
    assert a.k.dtype == np.float32 and np.array_equal(W.round_bf16(a.k), a.k)
    assert len(a.needle_pos) == 64 and len(set(a.needle_pos.tolist())) == 64


def test_shared_inputs_chunks_regenerate():
    wl = W.small(3, L=1024, T=1024, chunk=256)
    full = W.shared_inputs(wl)
    part = W.shared_inputs(wl, 512, 768)
    assert np.array_equal(full.q[512:768], part.q) and np.array_equal(full.w[512:768], part.w)
    assert np.array_equal(full.n, np.arange(1, 1025))
    assert np.array_equal(part.n, np.arange(513, 769))


def test_tiny_workload_shape_and_needles():
    wl = W.WORKLOADS[1]
    inp = W.shared_inputs(wl)
    assert inp.k.shape == (4096, 128) and inp.q.shape == (16, 64, 128) and inp.w.shape == (16, 64)
    assert list(inp.n) == list(range(4081, 4097))
    assert np.all(inp.w[:, inp.needle_heads] == 1.0)
    assert inp.needle_pos.max() < 4081
