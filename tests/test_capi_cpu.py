"""The C ABI on a machine without a GPU: the library loads, exports every function that
include/misa.h declares, sizes workspaces, and rejects bad arguments on the host before any
launch (these calls never reach the CUDA runtime)."""
import ctypes
import os
import re

import pytest

from long_context_sparse_mean_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "misa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA, DEVICE_TIMEOUT, BAD_INDEX = range(7)
BF16, F32 = 0, 1
P = ctypes.c_void_p


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:misa_status|size_t|int|const char\s*\*)\s*(\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    path = build.build()
    lib = ctypes.CDLL(path)
    from long_context_sparse_mean_b200 import binding  # sets the argtypes
    return binding.library()


def test_header_declares_the_indexer_calls():
    names = declared_functions()
    for want in ("misa_pool_keys", "misa_route", "misa_token_scores", "misa_topk_select", "misa_score_topk",
                 "misa_hier_rerank", "dsa_dense_topk", "misa_workspace_bytes", "misa_status_str", "misa_version",
                 "misa_device_check", "misa_block_filter_topk", "misa_pool_keys_paged", "misa_route_paged",
                 "misa_score_topk_paged", "misa_hier_rerank_paged"):
        assert want in names, want


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in misa.h but not exported"


def test_status_strings_and_version(lib):
    assert lib.misa_version() >= 100
    for code in range(7):
        assert lib.misa_status_str(code) != b"unknown status"
    assert lib.misa_status_str(99) == b"unknown status"


def _al(x):
    return (x + 255) // 256 * 256


def test_workspace_sizes(lib):
    ws = lib.misa_workspace_bytes
    # router: [T,128] partial-block means + [T, ceil(ceil(L/B)/64), H_I] tile sums + [T] counters
    # + [3, ceil(L/B), 128] bf16 parts of the pooled keys
    assert ws(0, 32, 131072, 64, 128, 8, 0, 0) == 32 * 128 * 4 + 32 * 16 * 64 * 4 + 256 + 3 * 1024 * 128 * 2
    # top-k select: candidate-list state per query: count and cut key [2, T] in one piece, the redo
    # flags [T] and the list [T, 16384] of (key, token) pairs, each piece 256-byte aligned
    def sel(T):
        return _al(T * 8) + _al(T * 4) + _al(T * 16384 * 8)
    assert ws(4, 32, 131072, 64, 0, 0, 2048, 0) == sel(32)
    assert ws(4, 32, 7, 64, 0, 0, 2048, 0) == sel(32), "independent of the row length"
    # scoring + top-k: [T, ceil4(L)] scores in front of the select workspace
    assert ws(1, 32, 131072, 64, 128, 8, 8192, 0) == 32 * 131072 * 4 + sel(32)
    assert ws(3, 32, 131072, 64, 0, 0, 2048, 0) == 32 * 131072 * 4 + sel(32)
    assert ws(1, 3, 1001, 64, 1, 8, 10, 0) == _al(3 * 1004 * 4) + sel(3)
    # re-rank: [T, k'] dense scores + the select workspace
    assert ws(2, 32, 0, 64, 0, 0, 2048, 8192) == 32 * 8192 * 4 + sel(32)
    assert ws(1, 0, 100, 64, 1, 8, 10, 0) == 0
    # block filter (m in the last slot): [T, ceil4(M)] block scores, [T] block counts, [T, m*B] token
    # ids and [T, m*B] their scores, then the select workspace
    P, M = 128 * 128, 1024
    assert ws(5, 32, 131072, 64, 128, 8, 2048, 128) == (32 * M * 4 + 256 + 2 * 32 * P * 4 + sel(32))
    assert ws(5, 3, 1001, 64, 7, 8, 10, 5) == (_al(3 * 144 * 4) + 256 + 2 * _al(3 * 35 * 4) + sel(3))
    assert ws(5, 32, 131072, 64, 128, 8, 2048, 129) == 0  # m * B above the candidate-list limit
    assert ws(5, 32, 131072, 64, 128, 8, 2048, 0) == 0


FAKE = P(0x10000)        # never dereferenced: every call below fails validation first
MISALIGNED = P(0x10008)


def route(lib, **kw):
    a = dict(q=FAKE, w=FAKE, k=FAKE, kss=0, kbar=FAKE, kbss=0, n=FAKE, T=4, L=1000, H_I=64, d=128, B=64, h=8,
             dt=BF16, heads=FAKE, r=None, ws=FAKE, wsb=1 << 30, s=None)
    a.update(kw)
    return lib.misa_route(a["q"], a["w"], a["k"], a["kss"], a["kbar"], a["kbss"], a["n"], a["T"], a["L"], a["H_I"],
                          a["d"], a["B"], a["h"], a["dt"], a["heads"], a["r"], a["ws"], a["wsb"], a["s"])


def test_router_argument_checks(lib):
    assert route(lib, d=64) == UNSUPPORTED
    assert route(lib, H_I=12) == UNSUPPORTED
    assert route(lib, H_I=136) == UNSUPPORTED
    assert route(lib, dt=7) == UNSUPPORTED
    assert route(lib, h=0) == INVALID
    assert route(lib, h=65) == INVALID
    assert route(lib, B=0) == INVALID
    assert route(lib, L=0) == INVALID
    assert route(lib, T=-1) == INVALID
    assert route(lib, q=None) == INVALID
    assert route(lib, kbar=None) == INVALID
    assert route(lib, heads=None) == INVALID
    assert route(lib, kss=1000 * 128 - 1) == INVALID
    assert route(lib, ws=None) == WORKSPACE
    assert route(lib, wsb=100) == WORKSPACE
    assert route(lib, ws=MISALIGNED) == WORKSPACE
    assert route(lib, T=0, q=None, w=None, k=None, n=None, heads=None) == OK


def test_scoring_and_selection_argument_checks(lib):
    st = lib.misa_score_topk(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 8, 0, BF16, FAKE, None, None, FAKE,
                             1 << 30, None)
    assert st == INVALID  # topk < 1
    st = lib.misa_score_topk(FAKE, FAKE, FAKE, 0, FAKE, None, 4, 1000, 64, 128, 8, 10, BF16, FAKE, None, None, FAKE,
                             1 << 30, None)
    assert st == INVALID  # no heads
    st = lib.misa_score_topk(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 8, 10, BF16, FAKE, None, None, FAKE,
                             16, None)
    assert st == WORKSPACE
    st = lib.misa_token_scores(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 8, BF16, FAKE, 999, 0, None, 0,
                               None)
    assert st == INVALID  # ld < L
    st = lib.misa_token_scores(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 8, BF16, FAKE, 1000, 0, FAKE,
                               1 << 30, None)
    assert st == INVALID  # a selection workspace without a k
    st = lib.misa_token_scores(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 8, BF16, FAKE, 1000, 10, FAKE, 64,
                               None)
    assert st == WORKSPACE
    st = lib.misa_topk_select(FAKE, 999, FAKE, 4, 1000, 10, FAKE, None, FAKE, 1 << 30, 0, None)
    assert st == INVALID
    st = lib.misa_topk_select(FAKE, 1000, FAKE, 4, 1000, 0, FAKE, None, FAKE, 1 << 30, 0, None)
    assert st == INVALID
    st = lib.misa_topk_select(FAKE, 1000, FAKE, 4, 1000, 10, FAKE, None, FAKE, 64, 0, None)
    assert st == WORKSPACE
    st = lib.misa_hier_rerank(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 1000, 64, 128, 100, 200, BF16, FAKE, None, FAKE,
                              1 << 30, None)
    assert st == INVALID  # k' < k
    st = lib.misa_hier_rerank(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 4, 100000, 64, 128, 16385, 200, BF16, FAKE, None, FAKE,
                              1 << 30, None)
    assert st == UNSUPPORTED  # k' above the shared-memory limit
    st = lib.dsa_dense_topk(FAKE, FAKE, FAKE, 0, FAKE, 4, 1000, 64, 128, 10, BF16, FAKE, None, MISALIGNED, 1 << 30,
                            None)
    assert st == WORKSPACE
    st = lib.misa_pool_keys(FAKE, 0, 1, 1000, 64, 64, BF16, FAKE, 0, 0, 16, None)
    assert st == UNSUPPORTED
    st = lib.misa_pool_keys(FAKE, 1000, 2, 1000, 128, 64, BF16, FAKE, 16 * 128, 0, 16, None)
    assert st == INVALID  # caches overlap
    assert lib.misa_pool_keys(FAKE, 0, 0, 1000, 128, 64, BF16, FAKE, 0, 0, 16, None) == OK
    assert lib.misa_pool_keys(FAKE, 0, 1, 1000, 128, 64, BF16, FAKE, 0, 16, 16, None) == OK  # empty range


def block_filter(lib, **kw):
    a = dict(q=FAKE, w=FAKE, k=FAKE, kss=0, kbar=FAKE, kbss=0, n=FAKE, heads=FAKE, T=4, L=1000, H_I=64, d=128,
             B=64, h=8, m=4, topk=100, dt=BF16, S=None, ldS=0, blocks=FAKE, idx=FAKE, vals=None, ws=FAKE,
             wsb=1 << 30, s=None)
    a.update(kw)
    return lib.misa_block_filter_topk(*(a[x] for x in ("q", "w", "k", "kss", "kbar", "kbss", "n", "heads", "T", "L",
                                                       "H_I", "d", "B", "h", "m", "topk", "dt", "S", "ldS",
                                                       "blocks", "idx", "vals", "ws", "wsb", "s")))


def test_block_filter_argument_checks(lib):
    assert block_filter(lib, d=64) == UNSUPPORTED
    assert block_filter(lib, H_I=12) == UNSUPPORTED
    assert block_filter(lib, m=0) == INVALID
    assert block_filter(lib, topk=0) == INVALID
    assert block_filter(lib, h=0) == INVALID
    assert block_filter(lib, h=65) == INVALID
    assert block_filter(lib, B=0) == INVALID
    assert block_filter(lib, m=257) == UNSUPPORTED  # 257 * 64 tokens above the candidate-list limit
    assert block_filter(lib, kbss=16 * 128 - 4) == INVALID  # pooled caches overlap
    assert block_filter(lib, kbss=16 * 128 + 2) == INVALID  # rows not 16-byte aligned
    assert block_filter(lib, S=FAKE, ldS=15) == INVALID  # block-score rows shorter than ceil(L/B)
    assert block_filter(lib, kbar=None) == INVALID
    assert block_filter(lib, kbar=MISALIGNED) == INVALID
    assert block_filter(lib, heads=None) == INVALID
    assert block_filter(lib, blocks=None) == INVALID
    assert block_filter(lib, idx=None) == INVALID
    assert block_filter(lib, ws=None) == WORKSPACE
    assert block_filter(lib, wsb=1000) == WORKSPACE
    assert block_filter(lib, ws=MISALIGNED) == WORKSPACE
    assert block_filter(lib, T=0, q=None, w=None, k=None, n=None, kbar=None, heads=None) == OK


def test_paged_workspaces_and_argument_checks(lib):
    ws = lib.misa_workspace_bytes
    # route: the contiguous router's workspace plus [T, 128] partial-block means
    assert ws(6, 32, 131072, 64, 128, 8, 0, 0) == ws(0, 32, 131072, 64, 128, 8, 0, 0) + 32 * 128 * 4
    # scoring + top-k: [T, L] physical rows and [T] row counts in front of the contiguous layout
    assert ws(7, 32, 131072, 64, 0, 8, 8192, 0) == 32 * 131072 * 4 + 256 + ws(1, 32, 131072, 64, 0, 8, 8192, 0)
    # re-rank: [T, k'] physical rows and [T] row counts in front of the contiguous layout
    assert ws(8, 32, 0, 64, 0, 0, 2048, 8192) == 32 * 8192 * 4 + 256 + ws(2, 32, 0, 64, 0, 0, 2048, 8192)

    def score(**kw):
        a = dict(q=FAKE, w=FAKE, pool=FAKE, num_pages=100, ps=64, table=FAKE, max_pages=20, n=FAKE, heads=FAKE, T=4,
                 L=1000, H_I=64, d=128, h=8, topk=10, dt=BF16, idx=FAKE, vals=None, ws=FAKE, wsb=1 << 30, s=None)
        a.update(kw)
        return lib.misa_score_topk_paged(*(a[x] for x in ("q", "w", "pool", "num_pages", "ps", "table", "max_pages",
                                                          "n", "heads", "T", "L", "H_I", "d", "h", "topk", "dt",
                                                          "idx", "vals", "ws", "wsb", "s")))
    assert score(L=1281) == INVALID           # 20 pages of 64 keys hold 1280
    assert score(table=None) == INVALID
    assert score(pool=None) == INVALID
    assert score(ps=0) == INVALID
    assert score(num_pages=1 << 26) == UNSUPPORTED  # pool rows past int32
    assert score(heads=None) == INVALID
    assert score(wsb=1000) == WORKSPACE
    assert score(T=0, q=None, w=None, pool=None, n=None, heads=None, table=None) == OK
    st = lib.misa_hier_rerank_paged(FAKE, FAKE, FAKE, 100, 64, FAKE, 20, FAKE, FAKE, 4, 1000, 64, 128, 100, 200, BF16,
                                    FAKE, None, FAKE, 1 << 30, None)
    assert st == INVALID  # k' < k
    st = lib.misa_route_paged(FAKE, FAKE, FAKE, 100, 64, FAKE, 20, FAKE, 0, FAKE, 4, 1000, 64, 128, 64, 8, BF16, FAKE,
                              None, FAKE, 1 << 30, None)
    assert st == INVALID  # queries need their own pooled caches
    st = lib.misa_pool_keys_paged(FAKE, 100, 64, FAKE, 20, 2, 1000, 128, 64, BF16, FAKE, 16 * 128 - 1, 0, 16, None)
    assert st == INVALID  # pooled caches overlap
    assert lib.misa_pool_keys_paged(FAKE, 100, 64, FAKE, 20, 2, 1000, 128, 64, BF16, FAKE, 16 * 128, 16, 16,
                                    None) == OK  # empty block range


def test_binding_rejects_host_tensors():
    import torch
    from long_context_sparse_mean_b200 import binding
    with pytest.raises(ValueError):
        binding.misa_pool_keys(torch.zeros(10, 128, dtype=torch.bfloat16), 4)


def test_device_check_reports_without_a_device(lib):
    """misa_device_check synchronises and reads the device status word: without a usable device
    the synchronisation fails and the call says so; with one, nothing has timed out."""
    import torch
    want = OK if torch.cuda.is_available() else CUDA
    assert lib.misa_device_check() == want
    assert lib.misa_status_str(DEVICE_TIMEOUT) != b"unknown status"


def test_a_c_program_compiles_links_and_calls_the_library(tmp_path):
    """include/misa.h is plain C (C99, no C++ names): a C program includes it, links libmisa.so and
    calls entry points that need no GPU (version, status text, workspace sizes, argument checks)."""
    import subprocess
    lib_path = build.build()
    src = tmp_path / "use_misa.c"
    src.write_text(r"""
#include <stdio.h>
#include "misa.h"
int main(void) {
  if (misa_version() < 100) return 1;
  if (misa_workspace_bytes(MISA_OP_SCORE_TOPK, 0, 100, 64, 1, 8, 10, 0) != 0) return 2;
  if (misa_workspace_bytes(MISA_OP_RERANK, 4, 0, 64, 0, 0, 10, 100) == 0) return 3;
  /* d = 64 is refused on the host, before any launch */
  misa_status st = misa_route((const void*)0x10000, (const float*)0x10000, (const void*)0x10000, 0,
                              (const float*)0x10000, 0, (const int32_t*)0x10000, 4, 1000, 64, 64, 64, 8,
                              MISA_BF16, (int32_t*)0x10000, NULL, (void*)0x10000, 1u << 30, NULL);
  if (st != MISA_ERR_UNSUPPORTED) return 4;
  printf("%s\n", misa_status_str(st));
  return 0;
}
""")
    exe = tmp_path / "use_misa"
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(lib_path)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-L", libdir, "-lmisa",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "unsupported configuration"


def test_bounds_checked_build_exports_the_same_calls():
    """libmisa_checked.so (MISA_CHECKED) exports every call misa.h declares and says it is the checked
    build; the normal library says it is not, and both refuse a null count buffer on the host."""
    checked = ctypes.CDLL(build.build(checked=True))
    for name in declared_functions():
        assert hasattr(checked, name), f"{name} missing from the checked build"
    checked.misa_checked_build.restype = ctypes.c_int
    checked.misa_bad_index_counts.argtypes = [P]
    checked.misa_bad_index_counts.restype = ctypes.c_int
    assert checked.misa_checked_build() == 1
    assert checked.misa_bad_index_counts(None) == INVALID
    normal = ctypes.CDLL(build.build())
    normal.misa_checked_build.restype = ctypes.c_int
    assert normal.misa_checked_build() == 0


def test_fused_prefill_workspace_and_argument_checks(lib):
    """misa_score_topk_fused: workspace = candidate-list state (counts and cut keys [2, T], redo flags
    [T], lists [T, 4k] of (key, token) pairs) + the cut [T] + the sample's largest score [T] + the
    packed sample [T, ceil(ceil(L/128)/32) * 128] + score rows [T, ceil4(L)] for the queries that are
    redone; k above 4096 (lists over 16384 entries) and fp32 inputs are unsupported."""
    ws = lib.misa_workspace_bytes
    T, L, k = 4096, 65536, 2048
    cols = -(-(-(-L // 128)) // 32) * 128
    want = (_al(T * 8) + _al(T * 4) + _al(T * 4 * k * 8) + 2 * _al(T * 4) + _al(T * cols * 4) +
            _al(T * (-(-L // 4) * 4) * 4))
    assert ws(9, T, L, 64, 128, 8, k, 0) == want
    assert ws(9, 3, 1001, 64, 128, 8, 10, 0) == (_al(24) + _al(12) + _al(3 * 40 * 8) + 2 * _al(12) + _al(3 * 128 * 4) +
                                                 _al(3 * 1004 * 4))
    assert ws(9, T, L, 64, 128, 8, 4097, 0) == 0, "lists of more than 16384 entries"
    f = lib.misa_score_topk_fused
    st = f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1000, 64, 128, 8, 10, F32, FAKE, None, FAKE, 1 << 30, None)
    assert st == UNSUPPORTED  # fp32 inputs take the unfused calls
    st = f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1000, 64, 128, 8, 4097, BF16, FAKE, None, FAKE, 1 << 30, None)
    assert st == UNSUPPORTED
    st = f(FAKE, FAKE, FAKE, FAKE, None, 4, 1000, 64, 128, 8, 10, BF16, FAKE, None, FAKE, 1 << 30, None)
    assert st == INVALID  # no heads
    st = f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1000, 64, 128, 65, 10, BF16, FAKE, None, FAKE, 1 << 30, None)
    assert st == INVALID  # h > H_I
    st = f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1000, 64, 128, 8, 10, BF16, FAKE, None, FAKE, 64, None)
    assert st == WORKSPACE
    st = f(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 1000, 64, 128, 8, 10, BF16, FAKE, None, MISALIGNED, 1 << 30, None)
    assert st == WORKSPACE
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1000, 64, 128, 8, 10, BF16, FAKE, None, None, 0, None) == OK


def test_hier_fused_workspace_and_argument_checks(lib):
    """misa_hier_topk_fused: workspace = score rows [T, ceil4(L)] + list counts and cuts [2, T] +
    dense lists [T, 16384] of (key, token) pairs and their dense scores + the k' candidates [T, k']
    of rows the lists cannot answer; shared caches, fp32 inputs and k' above 16384 are unsupported."""
    ws = lib.misa_workspace_bytes
    T, L, kp, k = 32, 131072, 8192, 2048
    cap = 16384
    want = _al(T * L * 4) + 2 * _al(T * 4) + _al(T * cap * 8) + _al(T * cap * 4) + _al(T * kp * 4)
    assert ws(10, T, L, 64, 0, 8, k, kp) == want
    assert ws(10, 3, 1001, 64, 0, 8, 10, 20) == (_al(3 * 1004 * 4) + 2 * _al(12) + _al(3 * cap * 8) +
                                                 _al(3 * cap * 4) + _al(3 * 20 * 4))
    assert ws(10, 0, L, 64, 0, 8, k, kp) == 0
    f = lib.misa_hier_topk_fused
    S = 1000 * 128
    args = lambda **o: dict(dict(q=FAKE, w=FAKE, k=FAKE, kss=S, n=FAKE, heads=FAKE, T=4, L=1000, H=64, d=128, h=8,
                                 kp=40, topk=10, dt=BF16, idx=FAKE, v=None, ws=FAKE, wsb=1 << 30, s=None), **o)
    call = lambda a: f(*a.values())
    assert call(args(dt=F32)) == UNSUPPORTED
    assert call(args(kss=0)) == UNSUPPORTED  # one shared cache
    assert call(args(kp=16385)) == UNSUPPORTED
    assert call(args(kp=9)) == INVALID  # k' < k
    assert call(args(heads=None)) == INVALID
    assert call(args(h=65)) == INVALID
    assert call(args(kss=999 * 128)) == INVALID  # stride below L * d
    assert call(args(wsb=64)) == WORKSPACE
    assert call(args(ws=MISALIGNED)) == WORKSPACE
    assert call(args(T=0, ws=None, wsb=0)) == OK
