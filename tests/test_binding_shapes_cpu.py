"""The Python binding checks tensor shapes against the sizes it passes to the C library before any
device check: a tensor smaller than those sizes would be read or written past its end on the GPU.
On a machine without a GPU, well-shaped host tensors get past the shape checks and stop at the
device check; a wrong shape stops at its own check first."""
import pytest
import torch

from long_context_sparse_mean_b200 import binding as M

T, H_I, D, L, B = 3, 16, 128, 100, 8
MB = -(-L // B)


def _t(*shape, dtype=torch.float32):
    return torch.zeros(shape, dtype=dtype)


def _base(per_query=False):
    k = _t(T, L, D, dtype=torch.bfloat16) if per_query else _t(L, D, dtype=torch.bfloat16)
    kbar = _t(T, MB, D) if per_query else _t(MB, D)
    return dict(q=_t(T, H_I, D, dtype=torch.bfloat16), w=_t(T, H_I), k=k, kbar=kbar, n=_t(T, dtype=torch.int32),
                heads=_t(T, 4, dtype=torch.int32), cand=_t(T, 50, dtype=torch.int32))


def _device_check_only(fn):
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn()


def _shape_error(fn, what):
    with pytest.raises(ValueError, match=what):
        fn()


@pytest.mark.parametrize("per_query", [False, True])
def test_well_shaped_calls_reach_the_device_check(per_query):
    a = _base(per_query)
    q, w, k, kbar, n, heads, cand = (a[x] for x in ("q", "w", "k", "kbar", "n", "heads", "cand"))
    _device_check_only(lambda: M.misa_pool_keys(k, B))
    _device_check_only(lambda: M.misa_pool_keys(k, B, kbar=kbar))
    _device_check_only(lambda: M.misa_route(q, w, k, kbar, n, B, 4, heads=heads, r=_t(T, H_I)))
    _device_check_only(lambda: M.misa_token_scores(q, w, k, n, heads, out=_t(T, L + 4)))
    _device_check_only(lambda: M.misa_topk_select(_t(T, L), n, 10, idx=_t(T, 10, dtype=torch.int32)))
    _device_check_only(lambda: M.misa_score_topk(q, w, k, n, heads, 10, scores_full=_t(T + 1, L)))
    _device_check_only(lambda: M.misa_hier_rerank(q, w, k, n, cand, 10, idx=_t(T, 10, dtype=torch.int32)))
    _device_check_only(lambda: M.misa_hier_rerank_static(q, w, k, n, cand, 10))
    _device_check_only(lambda: M.dsa_dense_topk(q, w, k, n, 10, vals=_t(T, 10)))
    _device_check_only(lambda: M.misa_block_filter_topk(q, w, k, kbar, n, heads, B, 4, 10,
                                                        blocks=_t(T, 4, dtype=torch.int32),
                                                        block_scores=_t(T, MB)))
    if per_query:
        _device_check_only(lambda: M.misa_hier_topk_fused(q, w, k, n, heads, 50, 10, vals=_t(T, 10)))


def test_wrong_shapes_are_rejected_first():
    a = _base()
    q, w, k, kbar, n, heads, cand = (a[x] for x in ("q", "w", "k", "kbar", "n", "heads", "cand"))
    i32 = torch.int32
    _shape_error(lambda: M.misa_route(q[0], w, k, kbar, n, B, 4), "q must be")
    _shape_error(lambda: M.misa_route(q, w[:, :8], k, kbar, n, B, 4), "w must be")
    _shape_error(lambda: M.misa_route(q, w, k, kbar, n[:2], B, 4), "n must be")
    _shape_error(lambda: M.misa_route(q, w, k[:, :64], kbar, n, B, 4), "k rows have")
    _shape_error(lambda: M.misa_route(q, w, k, kbar[:5], n, B, 4), "kbar must be")
    _shape_error(lambda: M.misa_route(q, w, k, _t(T, MB, D), n, B, 4), "kbar must be")  # per-query pooled keys
    _shape_error(lambda: M.misa_route(q, w, k, kbar, n, B, 4, heads=_t(T, 3, dtype=i32)), "heads must be")
    _shape_error(lambda: M.misa_route(q, w, k, kbar, n, B, 4, r=_t(T, 8)), "r must be")
    _shape_error(lambda: M.misa_pool_keys(k, B, kbar=_t(MB + 1, D)), "kbar must be")
    _shape_error(lambda: M.misa_token_scores(q, w, k, n, heads, out=_t(T, L - 1)), "out must be")
    _shape_error(lambda: M.misa_token_scores(q, w, k, n, heads[:2]), "heads must be")
    _shape_error(lambda: M.misa_topk_select(_t(T, L), n, 10, idx=_t(T, 9, dtype=i32)), "idx must be")
    _shape_error(lambda: M.misa_topk_select(_t(T, L), n, 10, vals=_t(T - 1, 10)), "vals must be")
    _shape_error(lambda: M.misa_topk_select(_t(T, L), n[:1], 10), "n must be")
    _shape_error(lambda: M.misa_score_topk(q, w, k, n, heads, 10, scores_full=_t(T, L + 1)), "scores_full must be")
    _shape_error(lambda: M.misa_score_topk(q, w, k, n, heads, 10, idx=_t(T, 11, dtype=i32)), "idx must be")
    _shape_error(lambda: M.misa_hier_rerank(q, w, k, n, cand[:1], 10), "cand must be")
    _shape_error(lambda: M.misa_hier_rerank_static(q, w, k, n, cand, 10, vals=_t(T, 5)), "vals must be")
    _shape_error(lambda: M.dsa_dense_topk(q, w, k, n, 10, idx=_t(1, 10, dtype=i32)), "idx must be")
    _shape_error(lambda: M.misa_block_filter_topk(q, w, k, kbar, n, heads, B, 4, 10,
                                                  blocks=_t(T, 3, dtype=i32)), "blocks must be")
    _shape_error(lambda: M.misa_block_filter_topk(q, w, k, kbar, n, heads, B, 4, 10,
                                                  block_scores=_t(T, MB - 1)), "block_scores must be")
    _shape_error(lambda: M.misa_block_filter_topk(q, w, k, kbar, n, heads, 4, 4, 10), "kbar must be")  # B mismatch
    kq = _t(T, L, D, dtype=torch.bfloat16)
    _shape_error(lambda: M.misa_hier_topk_fused(q, w, k, n, heads, 50, 10), "per-query caches")  # a shared cache
    _shape_error(lambda: M.misa_hier_topk_fused(q, w, kq, n, heads[:2], 50, 10), "heads must be")
    _shape_error(lambda: M.misa_hier_topk_fused(q, w, kq, n, heads, 50, 10, idx=_t(T, 9, dtype=i32)), "idx must be")


def test_device_check_rejects_a_tensor_on_another_gpu(monkeypatch):
    """The library launches on the current device, so a tensor on another GPU is refused before
    its pointer reaches a kernel."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)

    class OnGpu:
        def __init__(self, index):
            self.index = index
            self.device = f"cuda:{index}"

        def get_device(self):
            return self.index

    M._on_device(OnGpu(0), None, OnGpu(0))
    with pytest.raises(ValueError, match="current device cuda:0"):
        M._on_device(OnGpu(0), OnGpu(1))


def test_default_workspaces_are_per_stream(monkeypatch):
    """Calls given no Workspace share the default one of their device and stream only."""
    class FakeStream:
        def __init__(self, handle):
            self.cuda_stream = handle

    current = FakeStream(11)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: current)
    monkeypatch.setattr(M, "_default_ws", {})
    a = M._ws(None, "cpu")
    assert M._ws(None, "cpu") is a, "one stream: one default workspace"
    assert M._ws(None, "cpu", FakeStream(11)) is a, "the same stream given explicitly"
    b = M._ws(None, "cpu", FakeStream(12))
    assert b is not a, "another stream gets its own"
    current = FakeStream(12)
    assert M._ws(None, "cpu") is b
    mine = M.Workspace("cpu")
    assert M._ws(mine, "cpu") is mine, "a caller's Workspace is used as given"


def test_workspace_buffers_belong_to_the_stream_that_uses_them(monkeypatch):
    """A workspace buffer is allocated on the stream of the call that grows it, and a call on
    another stream marks it as used there (so the allocator recycles it only after that stream's
    work), except while a CUDA graph is being captured."""
    import contextlib

    class FakeStream:
        def __init__(self, handle):
            self.cuda_stream = handle

    class FakeBuf:
        def __init__(self, n):
            self.n, self.uses = n, []

        def numel(self):
            return self.n

        def record_stream(self, st):
            self.uses.append(st.cuda_stream)

    entered = []

    @contextlib.contextmanager
    def fake_stream_ctx(st):
        entered.append(st.cuda_stream)
        yield

    capturing = [False]
    monkeypatch.setattr(torch.cuda, "stream", fake_stream_ctx)
    monkeypatch.setattr(torch.cuda, "is_current_stream_capturing", lambda: capturing[0])
    monkeypatch.setattr(torch.cuda, "current_stream", lambda device=None: FakeStream(5))
    monkeypatch.setattr(torch, "empty", lambda n, **kw: FakeBuf(n))
    ws = M.Workspace("cpu")
    assert ws.get(0) is None
    b1 = ws.get(64)
    assert entered == [5] and b1.numel() == 64, "allocated on the current stream"
    assert ws.get(32, FakeStream(5)) is b1 and b1.uses == [], "same stream: no record"
    assert ws.get(32, FakeStream(9)) is b1 and b1.uses == [9], "another stream is recorded"
    capturing[0] = True
    ws.get(32, FakeStream(10))
    assert b1.uses == [9], "no record_stream while capturing"
    capturing[0] = False
    b2 = ws.get(128, FakeStream(9))
    assert b2 is not b1 and entered == [5, 9], "a larger buffer is allocated on the calling stream"
    ws.release()
    assert ws.buf is None
    monkeypatch.setattr(M, "_default_ws", {"x": ws})
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    M.release_default_workspaces()
    assert M._default_ws == {}
