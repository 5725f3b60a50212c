"""Python binding of libmisa.so: argument marshalling only.

Each function has the name of the C entry point it calls (include/misa.h) and passes torch
tensors' device pointers and the current CUDA stream through ctypes.  Every step of the indexer
runs in the library's CUDA kernels; there is no fallback.  If libmisa.so is missing the import
of this module fails.

Workspaces: a call given no Workspace uses a default buffer of its device and stream, shared only by
calls ordered on that stream, so calls on different streams never share scratch.  A Workspace passed
explicitly must likewise serve one stream at a time.  Default buffers are kept for the life of the
process, each as large as the largest call made on its stream; release_default_workspaces() frees
them.

Tensor conventions (all on one CUDA device, contiguous):
  q [T, H_I, 128] bf16 or fp32, w [T, H_I] fp32, n [T] int32 (prefix lengths),
  k [L, 128] (one cache shared by all queries) or [T, L, 128] (cache t for query t), same dtype as q,
  kbar [M, 128] or [T, M, 128] fp32 with M = ceil(L / B).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
# MISA_LIBRARY=checked selects the bounds-checked build (libmisa_checked.so, misa.h).
LIB_PATH = os.path.join(PKG, "libmisa_checked.so" if os.environ.get("MISA_LIBRARY") == "checked" else "libmisa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_BAD_INDEX = range(7)
BF16, F32 = 0, 1
(OP_ROUTE, OP_SCORE_TOPK, OP_RERANK, OP_DENSE_TOPK, OP_TOPK_SELECT, OP_BLOCK_FILTER, OP_ROUTE_PAGED,
 OP_SCORE_TOPK_PAGED, OP_RERANK_PAGED, OP_SCORE_TOPK_FUSED, OP_HIER_FUSED) = range(11)
MAX_KP = 16384

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -m long_context_sparse_mean_b200.build`")


class MisaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {_lib.misa_status_str(status).decode()} (status {status})")
        self.status = status


def _setup(lib):
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sigs = {
        "misa_version": ([], i32),
        "misa_device_check": ([], i32),
        "misa_checked_build": ([], i32),
        "misa_bad_index_counts": ([P], i32),
        "misa_status_str": ([i32], ctypes.c_char_p),
        "misa_workspace_bytes": ([i32, i32, i32, i32, i32, i32, i32, i32], sz),
        "misa_pool_keys": ([P, i64, i32, i32, i32, i32, i32, P, i64, i32, i32, P], i32),
        "misa_route": ([P, P, P, i64, P, i64, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz, P], i32),
        "misa_token_scores": ([P, P, P, i64, P, P, i32, i32, i32, i32, i32, i32, P, i64, i32, P, sz, P], i32),
        "misa_topk_select": ([P, i64, P, i32, i32, i32, P, P, P, sz, i32, P], i32),
        "misa_score_topk": ([P, P, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, sz, P], i32),
        "misa_hier_rerank": ([P, P, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz, P], i32),
        "dsa_dense_topk": ([P, P, P, i64, P, i32, i32, i32, i32, i32, i32, P, P, P, sz, P], i32),
        "misa_block_filter_topk": ([P, P, P, i64, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, i32, i32, P,
                                    i64, P, P, P, P, sz, P], i32),
        "misa_pool_keys_paged": ([P, i64, i32, P, i64, i32, i32, i32, i32, i32, P, i64, i32, i32, P], i32),
        "misa_route_paged": ([P, P, P, i64, i32, P, i64, P, i64, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz,
                              P], i32),
        "misa_score_topk_paged": ([P, P, P, i64, i32, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz,
                                   P], i32),
        "misa_hier_rerank_paged": ([P, P, P, i64, i32, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz,
                                    P], i32),
        "misa_score_topk_fused": ([P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz, P], i32),
        "misa_hier_topk_fused": ([P, P, P, i64, P, P, i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, sz, P], i32),
    }
    for name, (args, res) in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _setup(ctypes.CDLL(LIB_PATH))


def library() -> ctypes.CDLL:
    return _lib


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != OK:
        raise MisaError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q/k must be bfloat16 or float32, got {t.dtype}")


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _need_opt(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is not None:
        _need(t, name, dtype)


def _on_device(*ts):
    """Every given tensor is on the current CUDA device, where the library launches."""
    cur = torch.cuda.current_device()
    for t in ts:
        if t is not None and t.get_device() != cur:
            raise ValueError(f"every tensor must be on the current device cuda:{cur}; one is on {t.device}")


def _cache_geometry(k: torch.Tensor, T: int):
    """(L, d, k_seq_stride) of a shared [L, d] or per-query [T, L, d] key cache."""
    s = k.shape
    if len(s) == 2:
        return s[0], s[1], 0
    if len(s) == 3:
        if s[0] != T:
            raise ValueError(f"per-query cache needs k.shape[0] == T ({T}), got {s[0]}")
        return s[1], s[2], s[1] * s[2]
    raise ValueError("k must be [L, d] or [T, L, d]")


# Shape checks.  The C library sees only pointers and sizes, so a tensor smaller than the sizes
# passed with it would be read or written past its end; these run before any device check.
def _matrix(t, name: str, rows: int, cols: Optional[int] = None, min_cols: Optional[int] = None):
    """t is 2-D with at least `rows` rows and exactly `cols` (or at least `min_cols`) columns."""
    s = t.shape
    if len(s) != 2 or s[0] < rows or (cols is not None and s[1] != cols) or \
            (min_cols is not None and s[1] < min_cols):
        c = cols if cols is not None else (f">= {min_cols}" if min_cols is not None else "*")
        raise ValueError(f"{name} must be [>= {rows}, {c}], got {tuple(t.shape)}")


def _queries(q, w, n):
    """(T, H_I, d) of a query batch q [T, H_I, d] with w [>= T, H_I] and n [>= T]."""
    s = q.shape
    if len(s) != 3:
        raise ValueError(f"q must be [T, H_I, d], got {tuple(s)}")
    T, H_I, d = s
    _matrix(w, "w", T, H_I)
    ns = n.shape
    if len(ns) != 1 or ns[0] < T:
        raise ValueError(f"n must be [>= {T}], got {tuple(ns)}")
    return T, H_I, d


def _cache(k, T: int, d: int):
    """(L, k_seq_stride) of the key cache of a query batch whose vectors have d elements."""
    L, dk, kss = _cache_geometry(k, T)
    if dk != d:
        raise ValueError(f"k rows have {dk} elements, q rows {d}")
    return L, kss


def _pooled(kbar, k, T: int, L: int, B: int):
    """kbar matches the cache: [>= ceil(L/B), d] for a shared cache, [>= T, >= ceil(L/B), d] for
    per-query caches.  Returns the pooled caches' stride in floats (0 when shared)."""
    M = -(-L // B)
    ks, bs = k.shape, kbar.shape
    d = ks[-1]
    if not (len(bs) == len(ks) and bs[-2] >= M and bs[-1] == d and (len(bs) == 2 or bs[0] >= T)):
        want = f"[{M}, {d}]" if len(ks) == 2 else f"[{T}, {M}, {d}]"
        raise ValueError(f"kbar must be {want} for this cache and B = {B}, got {tuple(bs)}")
    return 0 if len(bs) == 2 else bs[1] * bs[2]


def _outputs(T: int, topk: int, idx, vals):
    """Caller-provided selection outputs hold [>= T, topk]."""
    if idx is not None:
        _matrix(idx, "idx", T, topk)
    if vals is not None:
        _matrix(vals, "vals", T, topk)


def misa_device_check() -> None:
    """Waits for the device, then raises MisaError if a tensor-core kernel stopped early on a
    wait that ran out since the last check (its outputs are then incomplete)."""
    _check("misa_device_check", _lib.misa_device_check())


def misa_bad_index_counts():
    """Counts of skipped out-of-range ids since the last read, (heads, candidates, pages); all zero
    unless the bounds-checked library is loaded.  Waits for the device; clears the counts."""
    out = (ctypes.c_uint * 3)()
    _check("misa_bad_index_counts", _lib.misa_bad_index_counts(out))
    return tuple(int(x) for x in out)


def checked_build() -> bool:
    return bool(_lib.misa_checked_build())


def misa_workspace_bytes(op: int, T: int, L: int, H_I: int, B: int = 1, h: int = 0, topk: int = 0,
                         kp: int = 0) -> int:
    return int(_lib.misa_workspace_bytes(op, T, L, H_I, B, h, topk, kp))


class Workspace:
    """A reusable, 256-byte aligned device scratch buffer (grown on demand).  One Workspace serves
    calls that are ordered on one stream; give each stream that may overlap another its own.

    The buffer is allocated on the stream of the call that needs it, so the caching allocator
    hands its memory to no other tensor while that stream's kernels may still use it.  A call on
    another stream marks the buffer as used there too (record_stream, outside graph capture), so
    a buffer that is replaced later returns to the allocator only after the work of every stream
    that used it."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None
        self._home = None  # raw handle of the stream the buffer was allocated on

    def get(self, nbytes: int, stream=None) -> Optional[torch.Tensor]:
        if nbytes <= 0:
            return None
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if self.buf is None or self.buf.numel() < nbytes:
            with torch.cuda.stream(st):
                self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device or "cuda")
            self._home = int(st.cuda_stream)
        elif int(st.cuda_stream) != self._home and not torch.cuda.is_current_stream_capturing():
            self.buf.record_stream(st)
        return self.buf

    def release(self) -> None:
        """Drop the buffer (its memory goes back to torch's caching allocator)."""
        self.buf = None
        self._home = None


_default_ws = {}


def _ws(ws: Optional[Workspace], device, stream=None) -> Workspace:
    """The caller's Workspace, or the default one of (device, stream): calls ordered on one stream
    share it, calls on different streams never do.  Default workspaces stay allocated (each as
    large as the largest call made on its stream) until release_default_workspaces()."""
    if ws is not None:
        return ws
    st = stream if stream is not None else torch.cuda.current_stream(device)
    key = (str(device), int(st.cuda_stream))
    w = _default_ws.get(key)
    if w is None:
        w = _default_ws[key] = Workspace(device)
    return w


def release_default_workspaces() -> None:
    """Free every default workspace (for example after a run on many external streams, whose
    handles could otherwise be reused by unrelated streams that then inherit a large buffer).
    Synchronises the device first, so no kernel still uses them."""
    if _default_ws:
        torch.cuda.synchronize()
    _default_ws.clear()


def misa_pool_keys(k: torch.Tensor, B: int, kbar: Optional[torch.Tensor] = None, block_begin: int = 0,
                   block_end: Optional[int] = None, stream=None) -> torch.Tensor:
    """Block means of every cache: k [L,d] or [S,L,d] -> kbar [M,d] or [S,M,d] (fp32)."""
    if k.dim() not in (2, 3):
        raise ValueError(f"k must be [L, d] or [S, L, d], got {tuple(k.shape)}")
    shared = k.dim() == 2
    S = 1 if shared else k.shape[0]
    L, d = k.shape[-2], k.shape[-1]
    M = -(-L // B)
    if kbar is not None and tuple(kbar.shape) != ((M, d) if shared else (S, M, d)):
        raise ValueError(f"kbar must be {[M, d] if shared else [S, M, d]}, got {tuple(kbar.shape)}")
    _need(k, "k")
    if kbar is None:
        kbar = torch.empty((M, d) if shared else (S, M, d), dtype=torch.float32, device=k.device)
    _need(kbar, "kbar", torch.float32)
    _on_device(k, kbar)
    block_end = M if block_end is None else block_end
    _check("misa_pool_keys", _lib.misa_pool_keys(
        _p(k), 0 if shared else L * d, S, L, d, B, _dtype_code(k), _p(kbar), 0 if shared else M * d,
        block_begin, block_end, _stream(stream)))
    return kbar


def misa_route(q, w, k, kbar, n, B: int, h: int, heads=None, r=None, ws: Optional[Workspace] = None,
               want_r: bool = False, stream=None):
    """Routed heads [T, h] (descending router score) and, if asked, router scores r [T, H_I]."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    kbss = _pooled(kbar, k, T, L, B)
    if heads is not None:
        _matrix(heads, "heads", T, h)
    if r is not None:
        _matrix(r, "r", T, H_I)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(kbar, "kbar", torch.float32)
    _need_opt(heads, "heads", torch.int32)
    _need_opt(r, "r", torch.float32)
    _on_device(q, k, w, n, kbar, heads, r)
    if heads is None:
        heads = torch.empty((T, h), dtype=torch.int32, device=q.device)
    if r is None and want_r:
        r = torch.empty((T, H_I), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_ROUTE, T, L, H_I, B, h)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_route", _lib.misa_route(
        _p(q), _p(w), _p(k), kss, _p(kbar), kbss, _p(n), T, L, H_I, d, B, h, _dtype_code(q), _p(heads), _p(r),
        _p(buf), nbytes, _stream(stream)))
    return heads, r


def misa_token_scores(q, w, k, n, heads=None, out=None, select_topk: int = 0, select_ws=None, stream=None):
    """Scores [T, L] fp32 (entries s >= n_t untouched); heads None = all heads (dense score).
    With select_topk > 0 and a Workspace, a top-select_topk selection of the scores is prepared in
    that workspace (for one bf16 cache per query: a sampled cut and the candidate list of every
    query) for misa_topk_select(..., ws=<same>, ws_prepared=True)."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    if heads is not None:
        _matrix(heads, "heads", T)
    if out is not None:
        _matrix(out, "out", T, min_cols=L)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need_opt(out, "out", torch.float32)
    h = 0
    if heads is not None:
        _need(heads, "heads", torch.int32)
        h = heads.shape[1]
    _on_device(q, k, w, n, heads, out)
    if out is None:
        out = torch.empty((T, L), dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32)
    buf, nbytes = None, 0
    if select_topk > 0:
        if select_ws is None:
            raise ValueError("select_topk needs select_ws")
        nbytes = misa_workspace_bytes(OP_TOPK_SELECT, T, L, H_I)
        buf = select_ws.get(nbytes, stream)
    _check("misa_token_scores", _lib.misa_token_scores(
        _p(q), _p(w), _p(k), kss, _p(n), _p(heads), T, L, H_I, d, h, _dtype_code(q), _p(out), out.shape[1],
        select_topk, _p(buf), nbytes, _stream(stream)))
    return out


def misa_topk_select(scores, n, topk: int, L: Optional[int] = None, idx=None, vals=None, want_vals=True,
                     ws: Optional[Workspace] = None, ws_prepared: bool = False, stream=None):
    """Top-k per row of scores [T, ld] over entries s < min(n_t, L) -> (idx [T, k], vals [T, k])."""
    if scores.dim() != 2:
        raise ValueError(f"scores must be [T, ld], got {tuple(scores.shape)}")
    T, ld = scores.shape
    if n.dim() != 1 or n.shape[0] < T:
        raise ValueError(f"n must be [>= {T}], got {tuple(n.shape)}")
    if idx is not None:
        _matrix(idx, "idx", T, topk)
    if vals is not None:
        _matrix(vals, "vals", T, topk)
    _need(scores, "scores", torch.float32)
    _need(n, "n", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(scores, n, idx, vals)
    L = ld if L is None else L
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=scores.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=scores.device)
    nbytes = misa_workspace_bytes(OP_TOPK_SELECT, T, L, 8)
    buf = _ws(ws, scores.device, stream).get(nbytes, stream)
    _check("misa_topk_select", _lib.misa_topk_select(
        _p(scores), ld, _p(n), T, L, topk, _p(idx), _p(vals), _p(buf), nbytes, int(ws_prepared), _stream(stream)))
    return idx, vals


def misa_score_topk(q, w, k, n, heads, topk: int, idx=None, vals=None, scores_full=None, want_vals=True,
                    ws: Optional[Workspace] = None, stream=None):
    """Routed scoring + top-k -> (idx [T, k], vals [T, k]); the index order is not specified."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    _matrix(heads, "heads", T)
    _outputs(T, topk, idx, vals)
    if scores_full is not None:
        _matrix(scores_full, "scores_full", T, L)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(heads, "heads", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _need_opt(scores_full, "scores_full", torch.float32)
    _on_device(q, k, w, n, heads, idx, vals, scores_full)
    h = heads.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    op = OP_TOPK_SELECT if scores_full is not None else OP_SCORE_TOPK
    nbytes = misa_workspace_bytes(op, T, L, H_I, 1, h, topk)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_score_topk", _lib.misa_score_topk(
        _p(q), _p(w), _p(k), kss, _p(n), _p(heads), T, L, H_I, d, h, topk, _dtype_code(q), _p(idx), _p(vals),
        _p(scores_full), _p(buf), nbytes, _stream(stream)))
    return idx, vals


def misa_score_topk_fused(q, w, k, n, heads, topk: int, idx=None, vals=None, want_vals=True,
                          ws: Optional[Workspace] = None, stream=None):
    """misa_score_topk for queries sharing one bf16 cache k [L, d], without score rows (sampled cut,
    candidate lists, exact redo of the queries whose list fell short or overflowed) -> (idx, vals)."""
    T, H_I, d = _queries(q, w, n)
    if k.dim() != 2:
        raise ValueError(f"k must be one shared cache [L, d], got {tuple(k.shape)}")
    L, _ = _cache(k, T, d)
    _matrix(heads, "heads", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(heads, "heads", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, k, w, n, heads, idx, vals)
    h = heads.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_SCORE_TOPK_FUSED, T, L, H_I, 0, h, topk)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_score_topk_fused", _lib.misa_score_topk_fused(
        _p(q), _p(w), _p(k), _p(n), _p(heads), T, L, H_I, d, h, topk, BF16, _p(idx), _p(vals), _p(buf), nbytes,
        _stream(stream)))
    return idx, vals


def misa_hier_topk_fused(q, w, k, n, heads, kp: int, topk: int, idx=None, vals=None, want_vals=True,
                         ws: Optional[Workspace] = None, stream=None):
    """MISA-dagger for per-query bf16 caches k [T, L, d] in one call: routed scores, top-k' by them,
    dense scores of those k' kept while the keys are read once, top-k of the dense score ->
    (idx [T, k], vals [T, k])."""
    T, H_I, d = _queries(q, w, n)
    if k.dim() != 3:
        raise ValueError(f"k must be per-query caches [T, L, d], got {tuple(k.shape)}")
    L, kss = _cache(k, T, d)
    _matrix(heads, "heads", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q", torch.bfloat16)
    _need(k, "k", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(heads, "heads", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, k, w, n, heads, idx, vals)
    h = heads.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_HIER_FUSED, T, L, H_I, 0, h, topk, kp)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_hier_topk_fused", _lib.misa_hier_topk_fused(
        _p(q), _p(w), _p(k), kss, _p(n), _p(heads), T, L, H_I, d, h, kp, topk, BF16, _p(idx), _p(vals), _p(buf),
        nbytes, _stream(stream)))
    return idx, vals


def misa_hier_rerank(q, w, k, n, cand, topk: int, idx=None, vals=None, want_vals=True,
                     ws: Optional[Workspace] = None, stream=None):
    """MISA-dagger fine stage: dense re-score of cand [T, k'] -> (idx [T, k], vals [T, k])."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    _matrix(cand, "cand", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(cand, "cand", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, k, w, n, cand, idx, vals)
    kp = cand.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_RERANK, T, L, H_I, 1, 0, topk, kp)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_hier_rerank", _lib.misa_hier_rerank(
        _p(q), _p(w), _p(k), kss, _p(n), _p(cand), T, L, H_I, d, kp, topk, _dtype_code(q), _p(idx), _p(vals),
        _p(buf), nbytes, _stream(stream)))
    return idx, vals


def dsa_dense_topk(q, w, k, n, topk: int, idx=None, vals=None, want_vals=True, ws: Optional[Workspace] = None,
                   stream=None):
    """Dense all-head indexer -> (idx [T, k], vals [T, k]); the index order is not specified."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    _outputs(T, topk, idx, vals)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, k, w, n, idx, vals)
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_DENSE_TOPK, T, L, H_I, 1, 0, topk)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("dsa_dense_topk", _lib.dsa_dense_topk(
        _p(q), _p(w), _p(k), kss, _p(n), T, L, H_I, d, topk, _dtype_code(q), _p(idx), _p(vals), _p(buf), nbytes,
        _stream(stream)))
    return idx, vals


def misa_block_filter_topk(q, w, k, kbar, n, heads, B: int, m: int, topk: int, idx=None, vals=None,
                           blocks=None, block_scores=None, want_vals=True, want_block_scores=False,
                           ws: Optional[Workspace] = None, stream=None):
    """Block filter + routed refinement: block scores with the routed heads, the m best blocks,
    then top-k over their tokens -> dict with idx [T, k], vals [T, k] (or None), blocks [T, m]
    (-1 padded; order not specified) and, if asked, block_scores [T, ceil(L/B)]."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    kbss = _pooled(kbar, k, T, L, B)
    M = -(-L // B)
    _matrix(heads, "heads", T)
    _outputs(T, topk, idx, vals)
    if blocks is not None:
        _matrix(blocks, "blocks", T, m)
    if block_scores is not None:
        _matrix(block_scores, "block_scores", T, min_cols=M)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(kbar, "kbar", torch.float32)
    _need(heads, "heads", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _need_opt(blocks, "blocks", torch.int32)
    _need_opt(block_scores, "block_scores", torch.float32)
    _on_device(q, k, w, n, kbar, heads, idx, vals, blocks, block_scores)
    h = heads.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    if blocks is None:
        blocks = torch.empty((T, m), dtype=torch.int32, device=q.device)
    if block_scores is None and want_block_scores:
        block_scores = torch.empty((T, M), dtype=torch.float32, device=q.device)
    ld_bs = 0 if block_scores is None else block_scores.shape[1]
    nbytes = misa_workspace_bytes(OP_BLOCK_FILTER, T, L, H_I, B, h, topk, m)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_block_filter_topk", _lib.misa_block_filter_topk(
        _p(q), _p(w), _p(k), kss, _p(kbar), kbss, _p(n), _p(heads), T, L, H_I, d, B, h, m, topk, _dtype_code(q),
        _p(block_scores), ld_bs, _p(blocks), _p(idx), _p(vals), _p(buf), nbytes, _stream(stream)))
    return {"idx": idx, "vals": vals, "blocks": blocks, "block_scores": block_scores}


def misa_indexer(q, w, k, kbar, n, B: int, h: int, topk: int, kp: Optional[int] = None,
                 ws: Optional[Workspace] = None, stream=None, m: Optional[int] = None):
    """The whole indexer for one batch: route -> routed scoring -> top-k (MISA), or with kp given
    route -> routed scoring -> top-k' candidates -> dense re-rank -> top-k (MISA-dagger), or with
    m given route -> block filter keeping m blocks -> routed scoring of their tokens -> top-k.
    Returns a dict with idx [T, k], vals [T, k], heads [T, h], (MISA-dagger) cand [T, k'] and
    (block filter) blocks [T, m]."""
    if kp is not None and m is not None:
        raise ValueError("give kp (MISA-dagger) or m (block filter), not both")
    heads, _ = misa_route(q, w, k, kbar, n, B, h, ws=ws, stream=stream)
    if m is not None:
        res = misa_block_filter_topk(q, w, k, kbar, n, heads, B, m, topk, ws=ws, stream=stream)
        return {"idx": res["idx"], "vals": res["vals"], "heads": heads, "blocks": res["blocks"]}
    if kp is None:
        idx, vals = misa_score_topk(q, w, k, n, heads, topk, ws=ws, stream=stream)
        return {"idx": idx, "vals": vals, "heads": heads}
    cand, _ = misa_score_topk(q, w, k, n, heads, kp, want_vals=False, ws=ws, stream=stream)
    idx, vals = misa_hier_rerank(q, w, k, n, cand, topk, ws=ws, stream=stream)
    return {"idx": idx, "vals": vals, "heads": heads, "cand": cand}


_lib.misa_hier_rerank_static.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] + [ctypes.c_void_p] * 2 + \
    [ctypes.c_int] * 7 + [ctypes.c_void_p] * 3
_lib.misa_hier_rerank_static.restype = ctypes.c_int
STATIC_RERANK_SCRATCH_FLOATS = 1 << 20


def misa_hier_rerank_static(q, w, k, n, cand, topk: int, idx=None, vals=None, want_vals=True, stream=None):
    """misa_hier_rerank for callers that cannot allocate device memory: the library's fixed
    scratch array replaces the workspace (T * k' <= STATIC_RERANK_SCRATCH_FLOATS).  Calls that
    overlap on the GPU share that array and must be ordered on one stream."""
    T, H_I, d = _queries(q, w, n)
    L, kss = _cache(k, T, d)
    _matrix(cand, "cand", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q")
    _need(k, "k", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(cand, "cand", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, k, w, n, cand, idx, vals)
    kp = cand.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    _check("misa_hier_rerank_static", _lib.misa_hier_rerank_static(
        _p(q), _p(w), _p(k), kss, _p(n), _p(cand), T, L, H_I, d, kp, topk, _dtype_code(q), _p(idx), _p(vals),
        _stream(stream)))
    return idx, vals


# ---- paged key caches: pool [num_pages, page_size, d], page_table [T, max_pages] int32 ----------

def _paged_geometry(pool, page_table, T: int, d: int, L: Optional[int]):
    """(num_pages, page_size, max_pages, L) of a paged cache; L defaults to what the table covers."""
    if pool.dim() != 3 or pool.shape[2] != d:
        raise ValueError(f"pool must be [num_pages, page_size, {d}], got {tuple(pool.shape)}")
    _matrix(page_table, "page_table", T)
    num_pages, page_size = pool.shape[0], pool.shape[1]
    max_pages = page_table.shape[1]
    L = max_pages * page_size if L is None else L
    if L > max_pages * page_size:
        raise ValueError(f"a table of {max_pages} pages of {page_size} keys cannot hold L = {L}")
    return num_pages, page_size, max_pages, L


def misa_pool_keys_paged(pool, page_table, B: int, L: Optional[int] = None, kbar=None, block_begin: int = 0,
                         block_end: Optional[int] = None, stream=None):
    """Block means of every sequence's logical cache through its page table -> kbar [S, M, d]."""
    S = page_table.shape[0]
    num_pages, page_size, max_pages, L = _paged_geometry(pool, page_table, S, pool.shape[-1], L)
    d = pool.shape[2]
    M = -(-L // B)
    if kbar is not None and tuple(kbar.shape) != (S, M, d):
        raise ValueError(f"kbar must be {[S, M, d]}, got {tuple(kbar.shape)}")
    _need(pool, "pool")
    _need(page_table, "page_table", torch.int32)
    if kbar is None:
        kbar = torch.empty((S, M, d), dtype=torch.float32, device=pool.device)
    _need(kbar, "kbar", torch.float32)
    _on_device(pool, page_table, kbar)
    block_end = M if block_end is None else block_end
    _check("misa_pool_keys_paged", _lib.misa_pool_keys_paged(
        _p(pool), num_pages, page_size, _p(page_table), max_pages, S, L, d, B, _dtype_code(pool), _p(kbar), M * d,
        block_begin, block_end, _stream(stream)))
    return kbar


def misa_route_paged(q, w, pool, page_table, kbar, n, B: int, h: int, L: Optional[int] = None, heads=None, r=None,
                     ws: Optional[Workspace] = None, want_r: bool = False, stream=None):
    """misa_route on paged caches -> (heads [T, h], r [T, H_I] or None)."""
    T, H_I, d = _queries(q, w, n)
    num_pages, page_size, max_pages, L = _paged_geometry(pool, page_table, T, d, L)
    M = -(-L // B)
    if kbar.dim() != 3 or kbar.shape[0] < T or kbar.shape[1] < M or kbar.shape[2] != d:
        raise ValueError(f"kbar must be [{T}, {M}, {d}], got {tuple(kbar.shape)}")
    if heads is not None:
        _matrix(heads, "heads", T, h)
    if r is not None:
        _matrix(r, "r", T, H_I)
    _need(q, "q")
    _need(pool, "pool", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(kbar, "kbar", torch.float32)
    _need(page_table, "page_table", torch.int32)
    _need_opt(heads, "heads", torch.int32)
    _need_opt(r, "r", torch.float32)
    _on_device(q, pool, w, n, kbar, page_table, heads, r)
    if heads is None:
        heads = torch.empty((T, h), dtype=torch.int32, device=q.device)
    if r is None and want_r:
        r = torch.empty((T, H_I), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_ROUTE_PAGED, T, L, H_I, B, h)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_route_paged", _lib.misa_route_paged(
        _p(q), _p(w), _p(pool), num_pages, page_size, _p(page_table), max_pages, _p(kbar),
        kbar.shape[1] * kbar.shape[2], _p(n), T, L, H_I, d, B, h, _dtype_code(q), _p(heads), _p(r), _p(buf), nbytes,
        _stream(stream)))
    return heads, r


def misa_score_topk_paged(q, w, pool, page_table, n, heads, topk: int, L: Optional[int] = None, idx=None, vals=None,
                          want_vals=True, ws: Optional[Workspace] = None, stream=None):
    """misa_score_topk on paged caches -> (idx [T, k], vals [T, k]); logical token indices."""
    T, H_I, d = _queries(q, w, n)
    num_pages, page_size, max_pages, L = _paged_geometry(pool, page_table, T, d, L)
    _matrix(heads, "heads", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q")
    _need(pool, "pool", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(heads, "heads", torch.int32)
    _need(page_table, "page_table", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, pool, w, n, heads, page_table, idx, vals)
    h = heads.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_SCORE_TOPK_PAGED, T, L, H_I, 0, h, topk)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_score_topk_paged", _lib.misa_score_topk_paged(
        _p(q), _p(w), _p(pool), num_pages, page_size, _p(page_table), max_pages, _p(n), _p(heads), T, L, H_I, d, h,
        topk, _dtype_code(q), _p(idx), _p(vals), _p(buf), nbytes, _stream(stream)))
    return idx, vals


def misa_hier_rerank_paged(q, w, pool, page_table, n, cand, topk: int, L: Optional[int] = None, idx=None,
                           vals=None, want_vals=True, ws: Optional[Workspace] = None, stream=None):
    """misa_hier_rerank on paged caches: dense re-score of logical candidates cand [T, k']."""
    T, H_I, d = _queries(q, w, n)
    num_pages, page_size, max_pages, L = _paged_geometry(pool, page_table, T, d, L)
    _matrix(cand, "cand", T)
    _outputs(T, topk, idx, vals)
    _need(q, "q")
    _need(pool, "pool", q.dtype)
    _need(w, "w", torch.float32)
    _need(n, "n", torch.int32)
    _need(cand, "cand", torch.int32)
    _need(page_table, "page_table", torch.int32)
    _need_opt(idx, "idx", torch.int32)
    _need_opt(vals, "vals", torch.float32)
    _on_device(q, pool, w, n, cand, page_table, idx, vals)
    kp = cand.shape[1]
    if idx is None:
        idx = torch.empty((T, topk), dtype=torch.int32, device=q.device)
    if vals is None and want_vals:
        vals = torch.empty((T, topk), dtype=torch.float32, device=q.device)
    nbytes = misa_workspace_bytes(OP_RERANK_PAGED, T, L, H_I, 0, 0, topk, kp)
    buf = _ws(ws, q.device, stream).get(nbytes, stream)
    _check("misa_hier_rerank_paged", _lib.misa_hier_rerank_paged(
        _p(q), _p(w), _p(pool), num_pages, page_size, _p(page_table), max_pages, _p(n), _p(cand), T, L, H_I, d, kp,
        topk, _dtype_code(q), _p(idx), _p(vals), _p(buf), nbytes, _stream(stream)))
    return idx, vals


def misa_indexer_paged(q, w, pool, page_table, kbar, n, B: int, h: int, topk: int, kp: Optional[int] = None,
                       L: Optional[int] = None, ws: Optional[Workspace] = None, stream=None):
    """misa_indexer on paged caches (MISA, or MISA-dagger with kp given)."""
    heads, _ = misa_route_paged(q, w, pool, page_table, kbar, n, B, h, L=L, ws=ws, stream=stream)
    if kp is None:
        idx, vals = misa_score_topk_paged(q, w, pool, page_table, n, heads, topk, L=L, ws=ws, stream=stream)
        return {"idx": idx, "vals": vals, "heads": heads}
    cand, _ = misa_score_topk_paged(q, w, pool, page_table, n, heads, kp, L=L, want_vals=False, ws=ws,
                                    stream=stream)
    idx, vals = misa_hier_rerank_paged(q, w, pool, page_table, n, cand, topk, L=L, ws=ws, stream=stream)
    return {"idx": idx, "vals": vals, "heads": heads, "cand": cand}
