"""The oracle and the CUDA path share no code and do not import each other, and the product
package never reaches the oracle (no CPU fallback)."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_sparse_mean_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(d, exts):
    for dp, _, fns in os.walk(d):
        if "__pycache__" in dp:
            continue
        for f in fns:
            if f.endswith(exts):
                yield os.path.join(dp, f)


def test_package_does_not_reference_the_oracle():
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        src = open(f).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
        assert "misa_oracle" not in src and "orc_" not in src, f


def test_oracle_does_not_reference_the_package():
    for f in _files(ORACLE, (".py", ".c", ".h")):
        src = open(f).read()
        assert "long_context_sparse_mean_b200" not in src, f
        assert "misa.h" not in src and "#include \"" not in src, f


def test_bench_uses_the_oracle_only_for_the_cpu_baseline():
    src = open(os.path.join(ROOT, "bench.py")).read()
    imports = [m.start() for m in re.finditer(r"^\s*import oracle|^\s*from oracle", src, re.M)]
    for pos in imports:
        # every oracle import sits inside a cpu-baseline / reference-arm function
        fn = src.rfind("\ndef ", 0, pos)
        name = src[fn + 5:src.index("(", fn)]
        assert "cpu" in name or "reference" in name, name
