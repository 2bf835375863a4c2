"""The product and the oracle stay apart: the package never imports the oracle (or anything under
a working folder), and the oracle never imports the package; the two share only the seeded
workload generators, which hold none of the verify arithmetic."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sources(d, exts):
    for base, _, files in os.walk(os.path.join(ROOT, d)):
        if "_build" in base or "__pycache__" in base:
            continue
        for f in files:
            if f.endswith(exts):
                yield os.path.join(base, f)


def test_package_does_not_import_the_oracle():
    for p in _sources("tree_speculative_decoding_06_b200", (".py", ".cu", ".cuh", ".h")):
        src = open(p).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", src, flags=re.M), p
        assert "oracle.c" not in src and "orc_" not in src, p
        assert "_work/" not in src, p


def test_oracle_does_not_import_the_package():
    for p in _sources("oracle", (".py", ".c")):
        src = open(p).read()
        assert not re.search(r"^\s*(import|from)\s+tree_speculative_decoding_06_b200\b", src, flags=re.M), p
        assert not re.search(r"CDLL\([^)]*libtsd|dlopen\([^)]*libtsd", src), p


def test_workload_generators_hold_no_verify_kernels():
    src = open(os.path.join(ROOT, "workloads", "__init__.py")).read()
    assert "tree_speculative_decoding_06_b200" not in src and not re.search(r"^\s*import oracle", src, flags=re.M)
