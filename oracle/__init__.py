"""CPU oracle for the MISA indexer (plain C, double accumulation) and its Python wrapper.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the CPU-baseline leg of
the benchmark are the only callers.  The CUDA library does not import, link or execute anything
here, and nothing here imports the CUDA library.

Every function follows "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
Inference" (gist.science/paper/2605.07363), "Technical Summary": "Methodology: MISA" (the
block-pooled router and the sparse token scoring), "Hierarchical Variant (MISA-dagger)" and
"Problem Statement" (the dense DSA indexer).  The block filter composed with MISA follows "HISA:
Efficient Hierarchical Indexing for Fine-Grained Sparse Attention" (arXiv 2603.28458), abstract.
The C source states the formulas and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "misa_oracle.c")
LIBRARY = os.path.join(HERE, "libmisa_oracle.so")

MODE_MISA, MODE_DAGGER, MODE_DSA = 0, 1, 2


def compile_oracle(src: str = SOURCE, out: str = LIBRARY, force: bool = False) -> str:
    """Compile an oracle source with gcc (-O2 -fopenmp) if the library is missing or stale."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, src, "-lm"],
                       check=True)
        os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    return compile_oracle(force=force)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        lib.orc_num_threads.restype = i32
        lib.orc_topk.argtypes = [P, P, i64, i64, P, P]
        lib.orc_topk.restype = i64
        lib.orc_pool_keys.argtypes = [P, i64, i32, i32, P]
        lib.orc_route.argtypes = [P, P, P, i64, i32, i32, i32, i32, P, P]
        lib.orc_token_scores.argtypes = [P, P, P, i32, P, i64, i32, P]
        lib.orc_rerank.argtypes = [P, P, i32, P, i64, i32, P, i64, i64, P, P]
        lib.orc_indexer_batch.argtypes = [i32, P, P, P, i64, P, i32, i32, i32, i32, i32, i64, i64,
                                          P, P, P, P, P, P]
        lib.orc_scores_batch.argtypes = [P, P, P, i64, P, i32, i32, i32, P, i32, P, i64]
        lib.orc_dense_scores_at.argtypes = [P, P, P, i64, P, i32, i32, i32, P, i64, P]
        lib.orc_route_batch.argtypes = [P, P, P, i64, P, i32, i32, i32, i32, i32, P, P]
        lib.orc_pool_batch.argtypes = [P, i64, i32, i64, i32, i32, P]
        lib.orc_paged_gather.argtypes = [P, i64, i32, i32, P, i64, P, i32, i64, P]
        lib.orc_paged_gather.restype = i64
        lib.orc_block_scores.argtypes = [P, P, P, i32, P, i64, i32, i32, P]
        lib.orc_block_filter.argtypes = [P, P, P, i32, P, i64, i32, i32, i64, i64, P, P, P, P]
        lib.orc_block_filter_batch.argtypes = [P, P, P, i64, P, i32, i32, i32, i32, i32, i64, i64, P, P,
                                               P, P, i64, P, P, P]
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return int(self.lib.orc_num_threads())

    def topk(self, v, k, ids=None):
        """Top-k of v (descending; exact ties to the lower id; ids < 0 skipped) -> (ids[k], vals[k])."""
        v = np.ascontiguousarray(v, dtype=np.float64)
        ids = None if ids is None else _i32(ids)
        out = np.empty(k, np.int32)
        out_v = np.empty(k, np.float64)
        self.lib.orc_topk(_p(v), _p(ids), v.shape[0], k, _p(out), _p(out_v))
        return out, out_v

    def pool_keys(self, k, B, n=None):
        """Block means of the first n keys of k[L,d] -> kbar[ceil(n/B), d] (double)."""
        k = _f32(k)
        n = k.shape[0] if n is None else n
        out = np.empty((-(-n // B), k.shape[1]), np.float64)
        self.lib.orc_pool_keys(_p(k), n, k.shape[1], B, _p(out))
        return out

    def pool_batch(self, k, k_seq_stride, n_seq, L, d, B):
        k = _f32(k)
        out = np.empty((n_seq, -(-L // B), d), np.float64)
        self.lib.orc_pool_batch(_p(k), k_seq_stride, n_seq, L, d, B, _p(out))
        return out

    def route(self, q, w, k, n, B, h):
        """Router for one query: q[H_I,d], w[H_I], k[>=n,d] -> (r[H_I], heads[h] by descending r)."""
        q, w, k = _f32(q), _f32(w), _f32(k)
        H_I, d = q.shape
        r = np.empty(H_I, np.float64)
        heads = np.empty(h, np.int32)
        self.lib.orc_route(_p(q), _p(w), _p(k), n, H_I, d, B, h, _p(r), _p(heads))
        return r, heads

    def token_scores(self, q, w, heads, k, n):
        """I[s] for s < n of one query with the given heads (summed in ascending head index)."""
        q, w, k, heads = _f32(q), _f32(w), _f32(k), _i32(heads)
        out = np.empty(n, np.float64)
        self.lib.orc_token_scores(_p(q), _p(w), _p(heads), heads.shape[0], _p(k), n, q.shape[1], _p(out))
        return out

    def rerank(self, q, w, k, n, cand, topk_):
        """MISA-dagger fine stage for one query -> (ids[topk], dense scores[topk])."""
        q, w, k, cand = _f32(q), _f32(w), _f32(k), _i32(cand)
        out = np.empty(topk_, np.int32)
        out_v = np.empty(topk_, np.float64)
        self.lib.orc_rerank(_p(q), _p(w), q.shape[0], _p(k), n, q.shape[1], _p(cand), cand.shape[0], topk_,
                            _p(out), _p(out_v))
        return out, out_v

    def indexer(self, mode, q, w, k, k_seq_stride, n, B, h, topk_, kp=0, heads_in=None):
        """Batched MISA / MISA-dagger / DSA over T queries (layouts as in the C driver).

        Returns a dict with idx[T,k], idx_v[T,k] and, for the routed modes, r[T,H_I],
        heads[T,h] and (MISA-dagger) cand[T,k']."""
        q, w, k, n = _f32(q), _f32(w), _f32(k), _i32(n)
        T, H_I, d = q.shape
        out = {"idx": np.empty((T, topk_), np.int32), "idx_v": np.empty((T, topk_), np.float64)}
        r = heads = cand = None
        if mode != MODE_DSA:
            r = out["r"] = np.empty((T, H_I), np.float64)
            heads = out["heads"] = np.empty((T, h), np.int32)
            if mode == MODE_DAGGER:
                cand = out["cand"] = np.empty((T, kp), np.int32)
        hin = None if heads_in is None else _i32(heads_in)
        self.lib.orc_indexer_batch(mode, _p(q), _p(w), _p(k), k_seq_stride, _p(n), T, H_I, d, B, h, topk_, kp,
                                   _p(hin), _p(r), _p(heads), _p(cand), _p(out["idx"]), _p(out["idx_v"]))
        return out

    def scores(self, q, w, k, k_seq_stride, n, heads=None, ld=None):
        """I[T, ld] (double) with heads[T,h] (None: all heads); entries s >= n_t are NaN."""
        q, w, k, n = _f32(q), _f32(w), _f32(k), _i32(n)
        T, H_I, d = q.shape
        ld = int(n.max()) if ld is None else ld
        out = np.full((T, ld), np.nan, np.float64)
        hh = None if heads is None else _i32(heads)
        nh = 0 if heads is None else hh.shape[1]
        self.lib.orc_scores_batch(_p(q), _p(w), _p(k), k_seq_stride, _p(n), T, H_I, d, _p(hh), nh, _p(out), ld)
        return out

    def dense_scores_at(self, q, w, k, k_seq_stride, n, ids):
        """All-head scores F[T, m] of the listed token ids[T, m] (invalid ids give 0)."""
        q, w, k, n, ids = _f32(q), _f32(w), _f32(k), _i32(n), _i32(ids)
        T, H_I, d = q.shape
        out = np.empty(ids.shape, np.float64)
        self.lib.orc_dense_scores_at(_p(q), _p(w), _p(k), k_seq_stride, _p(n), T, H_I, d, _p(ids), ids.shape[1],
                                     _p(out))
        return out

    def route_batch(self, q, w, k, k_seq_stride, n, B, h):
        q, w, k, n = _f32(q), _f32(w), _f32(k), _i32(n)
        T, H_I, d = q.shape
        r = np.empty((T, H_I), np.float64)
        heads = np.empty((T, h), np.int32)
        self.lib.orc_route_batch(_p(q), _p(w), _p(k), k_seq_stride, _p(n), T, H_I, d, B, h, _p(r), _p(heads))
        return r, heads

    def paged_caches(self, pool, page_table, n, L):
        """Logical caches [T, L, d] of sequences stored in pages: pool [num_pages, page_size, d],
        page_table [T, max_pages] (physical page of each logical page), n [T].  Keys past each
        prefix are zero.  Raises if a page id inside a prefix is out of range."""
        pool, page_table, n = _f32(pool), _i32(page_table), _i32(n)
        num_pages, page_size, d = pool.shape
        T, max_pages = page_table.shape
        out = np.empty((T, L, d), np.float32)
        bad = self.lib.orc_paged_gather(_p(pool), num_pages, page_size, d, _p(page_table), max_pages, _p(n), T, L,
                                        _p(out))
        if bad:
            raise ValueError(f"{bad} keys inside a prefix map to a page id outside the pool")
        return out

    def block_scores(self, q, w, heads, k, n, B):
        """Block-filter scores of one query: S[ceil(n/B)] with the given heads."""
        q, w, k, heads = _f32(q), _f32(w), _f32(k), _i32(heads)
        out = np.empty(-(-n // B), np.float64)
        self.lib.orc_block_scores(_p(q), _p(w), _p(heads), heads.shape[0], _p(k), n, q.shape[1], B, _p(out))
        return out

    def block_filter(self, q, w, k, k_seq_stride, n, B, h, m, topk_, heads_in=None):
        """Batched MISA with the token-axis block filter (route, keep m blocks, top-k inside them).

        Returns r[T,H_I], heads[T,h], S[T,ceil(max n/B)] (NaN past each query's blocks),
        blocks[T,m] (descending S, -1 padded), idx[T,k] and idx_v[T,k]."""
        q, w, k, n = _f32(q), _f32(w), _f32(k), _i32(n)
        T, H_I, d = q.shape
        ldS = max(1, -(-int(n.max(initial=0)) // B))
        out = {"r": np.empty((T, H_I), np.float64), "heads": np.empty((T, h), np.int32),
               "S": np.full((T, ldS), np.nan, np.float64), "blocks": np.empty((T, m), np.int32),
               "idx": np.empty((T, topk_), np.int32), "idx_v": np.empty((T, topk_), np.float64)}
        hin = None if heads_in is None else _i32(heads_in)
        self.lib.orc_block_filter_batch(_p(q), _p(w), _p(k), k_seq_stride, _p(n), T, H_I, d, B, h, m, topk_,
                                        _p(hin), _p(out["r"]), _p(out["heads"]), _p(out["S"]), ldS,
                                        _p(out["blocks"]), _p(out["idx"]), _p(out["idx_v"]))
        return out


_default = None
_lock = threading.Lock()


def get() -> Oracle:
    """The oracle compiled from this directory's source (built on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default
