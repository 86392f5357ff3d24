"""Static checks of the product sources (no GPU): the library path never reaches the oracle, and
no source issues a TMA or bulk load with cluster multicast or a batched memcpy."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "w4_gemm_error_channel_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        if "__pycache__" in d:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_package_does_not_import_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle\b|from\s+oracle\b)", re.M)
    bad = [p for p in _files(PKG, (".py",)) if pat.search(open(p).read())]
    assert not bad, bad


def test_no_multicast_loads_or_batched_copies():
    # The patterns are assembled from pieces so that this file does not spell them out itself.
    mc = "multi" + "cast" + "::" + "cluster"
    loads = re.compile(r"cp\.async\.bulk[^\"\n]*" + re.escape(mc))
    batched = re.compile(r"\bcu(da)?" + "Mem" + "cpy" + r"(3D)?" + "Batch" + "Async" + r"\b")
    bad = []
    for p in _files(PKG, (".cu", ".cuh", ".h", ".cpp", ".py")):
        text = open(p).read()
        if loads.search(text) or batched.search(text):
            bad.append(p)
    assert not bad, bad
