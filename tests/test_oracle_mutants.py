"""Plant one plausible mistake at a time in a copy of the oracle and show the pins catch it.

Each mutant is a textual edit of the oracle source (a dropped term, a wrong sign, a wrong index,
a reversed tie rule ...), compiled into a temporary directory; the real oracle is untouched.
"""

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "token score without relu": (
        "acc += (double)w[j] * orc_relu(orc_dot_ff(q + (int64_t)j * d, k + s * d, d));",
        "acc += (double)w[j] * (orc_dot_ff(q + (int64_t)j * d, k + s * d, d));"),
    "router without relu": ("acc += orc_relu(orc_dot_fd(", "acc += (orc_dot_fd("),
    "router ignores head weight": ("r[j] = (double)w[j] * acc;", "r[j] = acc;"),
    "block sum instead of mean": ("for (int i = 0; i < d; ++i) mean[i] /= c;", "(void)c;"),
    "partial block dropped": ("for (int64_t b = 0; b < M; ++b) acc += orc_relu(",
                              "for (int64_t b = 0; b < n / B; ++b) acc += orc_relu("),
    "ties to the higher index": ("if (a->i < b->i) return -1;\n  if (a->i > b->i) return 1;",
                                 "if (a->i < b->i) return 1;\n  if (a->i > b->i) return -1;"),
    "ascending selection": ("if (a->v > b->v) return -1;\n  if (a->v < b->v) return 1;",
                            "if (a->v > b->v) return 1;\n  if (a->v < b->v) return -1;"),
    "relu keeps negatives": ("return x > 0.0 ? x : 0.0;", "return x < 0.0 ? x : 0.0;"),
    "head row stride dropped": ("orc_dot_ff(q + (int64_t)j * d, k + s * d, d)",
                                "orc_dot_ff(q + (int64_t)j, k + s * d, d)"),
    "weight of slot, not of head": ("acc += (double)w[j] * orc_relu(orc_dot_ff(q + (int64_t)j * d, k + s * d, d));",
                                    "acc += (double)w[a] * orc_relu(orc_dot_ff(q + (int64_t)j * d, k + s * d, d));"),
    "batched driver ignores the cache stride": ("    const float* kt = k + (int64_t)t * k_seq_stride;",
                                                "    const float* kt = k;"),
    "batched scores use the first query's prefix": (
        "    const int64_t nt = n[t] > 0 ? n[t] : 0;\n    orc_token_scores(q + (int64_t)t * H_I * d",
        "    const int64_t nt = n[0] > 0 ? n[0] : 0;\n    orc_token_scores(q + (int64_t)t * H_I * d"),
    "block score without relu": (
        "acc += (double)w[j] * orc_relu(orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));",
        "acc += (double)w[j] * (orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));"),
    "block score ignores head weight": (
        "acc += (double)w[j] * orc_relu(orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));",
        "acc += orc_relu(orc_dot_fd(q + (int64_t)j * d, kbar + b * d, d));"),
    "block score with the first heads, not the routed ones": (
        "      const int j = hs[a];\n      acc += (double)w[j] * orc_relu(orc_dot_fd(",
        "      const int j = a;\n      acc += (double)w[j] * orc_relu(orc_dot_fd("),
    "partial last block never kept": ("  const int64_t M = (n + B - 1) / B;\n  orc_block_scores(",
                                      "  const int64_t M = n / B;\n  orc_block_scores("),
    "filter keeps the leading blocks": (
        "  orc_topk(S, NULL, M, m, blocks, NULL);",
        "  for (int64_t a = 0; a < m; ++a) blocks[a] = a < M ? (int32_t)a : -1;"),
    "kept block's tokens taken from the block before": (
        "    const int64_t s0 = (int64_t)blocks[a] * B;",
        "    const int64_t s0 = (int64_t)(blocks[a] > 0 ? blocks[a] - 1 : 0) * B;"),
    "paged gather ignores the page table": (
        "      const int32_t pg = lp < max_pages ? page_table[(int64_t)t * max_pages + lp] : -1;",
        "      const int32_t pg = (int32_t)((t * max_pages + lp) % num_pages);"),
    "paged rows counted from the page's end": (
        "(int64_t)pg * page_size + s % page_size",
        "(int64_t)pg * page_size + (page_size - 1 - s % page_size)"),
    "paged gather reads the page past the row's": (
        "      const int64_t lp = s / page_size;",
        "      const int64_t lp = s / page_size + 1;"),
    "dense re-rank with half the heads": ("      for (int j = 0; j < H_I; ++j)\n        acc += (double)w[j]",
                                          "      for (int j = 0; j < H_I / 2; ++j)\n        acc += (double)w[j]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) >= 1, f"mutation site not found for {name!r}"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = oracle.compile_oracle(str(mutated), str(tmp_path / "libmutant.so"), force=True)
    orc = oracle.Oracle(lib)
    failures = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            failures.append(check.__name__)
    assert failures, f"no pin catches the mutant {name!r}"
