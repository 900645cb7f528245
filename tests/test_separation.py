"""The oracle and the CUDA path share no code: the product package never
imports the oracle, the oracle never imports the product, and their C/CUDA
sources include nothing of each other.  (The seeded input generator,
``deltanet_chunkwise_delta_b200/workloads.py``, serves both callers and holds
none of the method's arithmetic; only tests, the smoke check and the
benchmark's CPU arms import both.)"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "deltanet_chunkwise_delta_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(base, exts):
    out = []
    for ext in exts:
        out += glob.glob(os.path.join(base, "**", "*" + ext), recursive=True)
    return [f for f in out if "_build" not in f]


def test_product_never_imports_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)", re.M)
    for f in _files(PKG, [".py"]):
        assert not pat.search(open(f).read()), f


def test_oracle_never_imports_the_product():
    pat = re.compile(r"^\s*(import|from)\s+deltanet_chunkwise_delta_b200\b", re.M)
    for f in _files(ORACLE, [".py"]):
        assert not pat.search(open(f).read()), f


def test_sources_include_nothing_of_each_other():
    inc = re.compile(r'#\s*include\s*[<"]([^>"]+)[>"]')
    for f in _files(PKG, [".cu", ".cuh", ".h"]):
        for name in inc.findall(open(f).read()):
            assert "oracle" not in name, (f, name)
    for f in _files(ORACLE, [".c", ".h"]):
        for name in inc.findall(open(f).read()):
            assert not name.startswith(("dn_", "deltanet")) and "csrc" not in name, (f, name)
