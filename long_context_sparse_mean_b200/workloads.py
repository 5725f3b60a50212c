"""Seeded synthetic inputs for the MISA indexer (shared by the tests, the bench and the oracle runs).

This module draws random numbers and nothing else: it holds none of the indexer's arithmetic
(no pooling, no router, no token scores, no selection).  Both the CUDA path and the CPU oracle
consume exactly the arrays produced here, so the two sides see identical input bits.

Shapes follow the workloads described on "MISA: Mixture of Indexer Sparse Attention for
Long-Context LLM Inference" (gist.science/paper/2605.07363), "Experimental Results":
DeepSeek-V3.2 (H_I = 64 indexer heads) and GLM-5 (H_I = 32), h = 8 routed heads, an enlarged
candidate set k' = 8192 (section "Hierarchical Variant (MISA-dagger)"), contexts up to 128K.
The pages measure on LongBench and Needle-in-a-Haystack with trained models; neither the
datasets nor the weights exist here, so seeded synthetic tensors with the same shapes stand
in for them (planted "needle" keys play the part of the NIAH needles).

Value distributions
-------------------
* ``gaussian``  : q, k ~ N(0, 1) (fp32, not rounded), w ~ N(0, 1) / sqrt(H_I).
* ``clustered`` : 16 centres c_i uniform on the unit sphere S^{d-1}; every key picks a centre
  uniformly, k_s = c_z + 0.5 * xi / sqrt(d) with xi ~ N(0, I) (0.5 is the scale of the noise
  *norm*); every head j has a fixed preferred set P_j of 1-3 centres and
  q_{t,j} = normalize(sum_{i in P_j} u_i c_i) + 0.5 * xi / sqrt(d) with u_i ~ U(0.5, 1.5);
  w ~ N(0, 1) / sqrt(H_I).  q and k are rounded once to bfloat16 (round to nearest even).
* needles (config 1): two seeded heads j1, j2 get w = +1 for every query and
  q_{t,j} = 4 u_j + xi; four keys (two per head) at seeded positions inside every query's
  prefix are k = 40 u_j.
* needles (config 4): 64 keys per sequence at seeded distinct positions.  Needle p points along
  a direction u_p that has a positive component along q_{j*} for a seeded head j* among the
  query's heads with the larger positive weights, and a negative one along every head with a
  negative weight (u_p is q_{j*} with its projection on those heads' span removed, plus a small
  step against each of them).  Its length alpha_p makes w_{j*} (q_{j*} . k_p) at least 3 x
  S = 3 x (sum over heads with w_j > 0 of w_j |q_j|) x (largest background key norm); alpha_p is
  also at least 4 x that largest key norm.  After bf16 rounding the generator asserts both sign
  conditions on the stored key.  These are sign and norm conditions on the inputs, not index
  scores: every term of a needle's dense score with a negative weight is then zero and the term
  of head j* alone exceeds 2 S, while no background key can score above S, so the dense top-k
  (k >= 64) holds every needle.

Every generator is keyed by (config seed, stream name, index) through numpy's SeedSequence, so
one sequence or one query chunk can be regenerated on its own.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

N_CLUSTERS = 16
SEED_BASE = 20261200

_STREAMS = {"centres": 1, "prefs": 2, "keys": 3, "queries": 4, "needles": 5, "extra": 6}


@dataclass(frozen=True)
class Workload:
    """One synthetic indexer workload (sizes in the pages' notation)."""

    cid: int
    name: str
    H_I: int
    d: int
    dtype: str  # "f32" or "bf16": the type of q and k handed to the indexer
    L: int  # key-cache length per sequence
    T: int  # number of queries
    n_seq: int  # number of key caches (1 = all queries share one cache)
    B: int  # router block size
    h: int  # routed heads
    topk: int  # k
    kp: Optional[int] = None  # k' (MISA-dagger candidate count) or None
    dist: str = "clustered"
    needles: Optional[str] = None
    chunk: Optional[int] = None  # prefill query-chunk size
    dense_too: bool = False  # also run the dense all-head indexer on the same inputs
    seed: int = field(default=0)

    @property
    def shared_cache(self) -> bool:
        return self.n_seq == 1 and self.T > 1

    @property
    def M(self) -> int:
        return -(-self.L // self.B)


def _wl(cid, **kw):
    return Workload(cid=cid, seed=SEED_BASE + cid, **kw)


WORKLOADS = {
    1: _wl(1, name="tiny_misa_fp32_L4096", H_I=64, d=128, dtype="f32", L=4096, T=16, n_seq=1,
           B=64, h=8, topk=256, dist="gaussian", needles="heads2"),
    2: _wl(2, name="decode_dsv32_L32768_b8", H_I=64, d=128, dtype="bf16", L=32768, T=8, n_seq=8,
           B=128, h=8, topk=2048),
    3: _wl(3, name="prefill_chunked_L65536", H_I=64, d=128, dtype="bf16", L=65536, T=65536, n_seq=1,
           B=128, h=8, topk=2048, chunk=4096),
    4: _wl(4, name="misa_dagger_decode_L131072_b32", H_I=64, d=128, dtype="bf16", L=131072, T=32,
           n_seq=32, B=128, h=8, topk=2048, kp=8192, needles="uniform64"),
    5: _wl(5, name="glm5_decode_L131072_b64", H_I=32, d=128, dtype="bf16", L=131072, T=64,
           n_seq=64, B=256, h=8, topk=2048, dense_too=True),
}


def small(cid: int, **over) -> Workload:
    """A reduced copy of a workload (same distribution, smaller sizes) for fast parity runs."""
    base = WORKLOADS[cid]
    kw = {f: getattr(base, f) for f in base.__dataclass_fields__}
    kw.update(over)
    return Workload(**kw)


def _rng(wl: Workload, stream: str, index: int = 0) -> np.random.Generator:
    return np.random.default_rng([wl.seed, _STREAMS[stream], int(index)])


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even).

    Returns float32 values that are exactly representable in bfloat16, so a later
    float32 -> bfloat16 conversion is exact.  Inputs are finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # finite inputs stay below 0xff800000, so adding at most 0x8000 cannot wrap in 32 bits
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _finish(wl: Workload, x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return round_bf16(x) if wl.dtype == "bf16" else x


def _unit_rows(a: np.ndarray) -> np.ndarray:
    return a / np.linalg.norm(a, axis=-1, keepdims=True)


def centres(wl: Workload) -> np.ndarray:
    g = _rng(wl, "centres")
    return _unit_rows(g.standard_normal((N_CLUSTERS, wl.d)))


def head_prefs(wl: Workload) -> list:
    g = _rng(wl, "prefs")
    out = []
    for _ in range(wl.H_I):
        m = int(g.integers(1, 4))
        out.append(np.sort(g.choice(N_CLUSTERS, size=m, replace=False)))
    return out


def _clustered_keys(wl: Workload, g: np.random.Generator, n: int, C: np.ndarray) -> np.ndarray:
    z = g.integers(0, N_CLUSTERS, size=n)
    xi = g.standard_normal((n, wl.d), dtype=np.float32)
    xi *= np.float32(0.5 / math.sqrt(wl.d))
    xi += C.astype(np.float32)[z]
    return xi


def _clustered_queries(wl: Workload, g: np.random.Generator, nq: int, C: np.ndarray, prefs) -> np.ndarray:
    q = np.empty((nq, wl.H_I, wl.d), dtype=np.float64)
    for j, P in enumerate(prefs):
        u = g.uniform(0.5, 1.5, size=(nq, len(P)))
        q[:, j, :] = _unit_rows(u @ C[P])
    q += (0.5 / math.sqrt(wl.d)) * g.standard_normal((nq, wl.H_I, wl.d))
    return q.astype(np.float32)


# --- config-1 style planted heads (gaussian, shared cache) ------------------------------------

def _needle_heads(wl: Workload):
    g = _rng(wl, "needles", 0)
    j = g.choice(wl.H_I, size=2, replace=False)
    u = _unit_rows(g.standard_normal((2, wl.d)))
    min_n = wl.L - wl.T + 1
    pos = g.choice(min_n, size=4, replace=False)
    return j, u, pos


@dataclass
class SharedInputs:
    """Queries that all read one key cache (configs 1 and 3): k[L,d], q[T,H_I,d], w[T,H_I], n[T]."""

    k: np.ndarray
    q: np.ndarray
    w: np.ndarray
    n: np.ndarray
    needle_pos: Optional[np.ndarray] = None  # [P] token positions
    needle_heads: Optional[np.ndarray] = None


def shared_keys(wl: Workload) -> np.ndarray:
    g = _rng(wl, "keys", 0)
    if wl.dist == "gaussian":
        k = g.standard_normal((wl.L, wl.d), dtype=np.float32)
    else:
        k = _clustered_keys(wl, g, wl.L, centres(wl))
    if wl.needles == "heads2":
        j, u, pos = _needle_heads(wl)
        for a in range(4):
            k[pos[a]] = 40.0 * u[a % 2]
    return _finish(wl, k)


def prefix_lengths(wl: Workload, t0: int = 0, t1: Optional[int] = None) -> np.ndarray:
    """Causal prefix lengths n_t.  Shared cache: the T queries are the last T positions of the
    cache (n_t = L - T + 1 + t), which for T = L is the full causal prefill n_t = t + 1.
    Separate caches (decode): every query sees its whole cache, n_t = L."""
    t1 = wl.T if t1 is None else t1
    t = np.arange(t0, t1, dtype=np.int64)
    if wl.n_seq == 1:
        return (wl.L - wl.T + 1 + t).astype(np.int32)
    return np.full(t1 - t0, wl.L, dtype=np.int32)


def shared_queries(wl: Workload, t0: int, t1: int):
    """q[t1-t0, H_I, d] and w[t1-t0, H_I] for queries t0..t1-1 of a shared-cache workload.

    Queries are drawn in chunks of ``wl.chunk`` (or all at once) so that any chunk can be
    regenerated alone; t0 and t1 must fall on chunk boundaries."""
    ch = wl.chunk or wl.T
    assert t0 % ch == 0 and (t1 % ch == 0 or t1 == wl.T), "query ranges follow the chunk grid"
    qs, ws = [], []
    for c in range(t0 // ch, -(-t1 // ch)):
        a, b = c * ch, min((c + 1) * ch, wl.T)
        g = _rng(wl, "queries", c)
        if wl.dist == "gaussian":
            q = g.standard_normal((b - a, wl.H_I, wl.d), dtype=np.float32)
        else:
            q = _clustered_queries(wl, g, b - a, centres(wl), head_prefs(wl))
        w = (g.standard_normal((b - a, wl.H_I)) / math.sqrt(wl.H_I)).astype(np.float32)
        if wl.needles == "heads2":
            j, u, _ = _needle_heads(wl)
            for a2 in range(2):
                w[:, j[a2]] = 1.0
                q[:, j[a2], :] = 4.0 * u[a2] + g.standard_normal((b - a, wl.d))
        qs.append(q)
        ws.append(w)
    return _finish(wl, np.concatenate(qs)), np.ascontiguousarray(np.concatenate(ws), dtype=np.float32)


def shared_inputs(wl: Workload, t0: int = 0, t1: Optional[int] = None) -> SharedInputs:
    t1 = wl.T if t1 is None else t1
    q, w = shared_queries(wl, t0, t1)
    out = SharedInputs(k=shared_keys(wl), q=q, w=w, n=prefix_lengths(wl, t0, t1))
    if wl.needles == "heads2":
        j, _, pos = _needle_heads(wl)
        out.needle_pos = np.sort(pos)
        out.needle_heads = np.sort(j)
    return out


# --- separate caches (decode) ------------------------------------------------------------------

@dataclass
class DecodeSequence:
    """One decode sequence: its key cache k[L,d], its query q[H_I,d], w[H_I], n = L."""

    k: np.ndarray
    q: np.ndarray
    w: np.ndarray
    n: int
    needle_pos: Optional[np.ndarray] = None


def decode_sequence(wl: Workload, s: int) -> DecodeSequence:
    assert wl.n_seq > 1 and 0 <= s < wl.n_seq
    C = centres(wl)
    g = _rng(wl, "queries", s)
    q = _finish(wl, _clustered_queries(wl, g, 1, C, head_prefs(wl))[0])
    w = (g.standard_normal(wl.H_I) / math.sqrt(wl.H_I)).astype(np.float32)
    gk = _rng(wl, "keys", s)
    k = _finish(wl, _clustered_keys(wl, gk, wl.L, C))
    pos = None
    if wl.needles == "uniform64":
        gn = _rng(wl, "needles", s)
        pos = np.sort(gn.choice(wl.L, size=64, replace=False))
        k[pos] = _needle_keys(wl, gn, q, w, k, len(pos))
    return DecodeSequence(k=k, q=q, w=w, n=wl.L, needle_pos=pos)


def _needle_keys(wl: Workload, g: np.random.Generator, q: np.ndarray, w: np.ndarray, k: np.ndarray,
                 count: int) -> np.ndarray:
    """Keys of `count` planted needles for one decode query (module docstring, config 4).

    Only signs and norms of the inputs are used: the direction of needle p is orthogonal to, then
    stepped against, the query vectors of the heads with negative weight, and its length follows
    from the weights, the query norms and the largest background key norm."""
    q64 = q.astype(np.float64)
    w64 = w.astype(np.float64)
    qn = np.linalg.norm(q64, axis=1)
    kmax = float(np.sqrt(np.einsum("ij,ij->i", k, k, dtype=np.float64).max()))
    pos_w = np.nonzero(w64 > 0)[0]
    strong = pos_w[w64[pos_w] >= np.median(w64[pos_w])]
    neg = np.nonzero(w64 < 0)[0]
    S = float((w64[pos_w] * qn[pos_w]).sum()) * kmax
    N = q64[neg]  # [m, d]
    basis = np.linalg.qr(N.T)[0] if len(neg) else np.zeros((wl.d, 0))
    out = np.empty((count, wl.d), np.float32)
    for a in range(count):
        j = int(g.choice(strong))
        u = q64[j] - basis @ (basis.T @ q64[j])  # no component along any negative head
        un = np.linalg.norm(u)
        if len(neg):
            # a step against every negative head: N u = -0.02 |q_j'| |u| for each of them
            u = u + np.linalg.lstsq(N, -0.02 * qn[neg] * un, rcond=None)[0]
        u /= np.linalg.norm(u)
        proj = float(q64[j] @ u)
        alpha = max(3.0 * S / (w64[j] * proj), 4.0 * kmax)
        key = _finish(wl, (alpha * u)[None, :])[0]
        kd = key.astype(np.float64)
        if len(neg) and not np.all(N @ kd < 0.0):
            raise RuntimeError("needle key projects positively on a negative-weight head")
        if not w64[j] * float(q64[j] @ kd) > 2.0 * S:
            raise RuntimeError("needle key too short")
        out[a] = key
    return out


def decode_batch(wl: Workload, seqs=None):
    """Stack sequences: k[S,L,d], q[S,H_I,d], w[S,H_I], n[S] (query s reads cache s)."""
    seqs = range(wl.n_seq) if seqs is None else seqs
    parts = [decode_sequence(wl, s) for s in seqs]
    k = np.stack([p.k for p in parts])
    q = np.stack([p.q for p in parts])
    w = np.stack([p.w for p in parts])
    n = np.array([p.n for p in parts], dtype=np.int32)
    needles = [p.needle_pos for p in parts]
    return k, q, w, n, needles
