"""The oracle and the CUDA path share no code and never import each other;
the product path never loads the oracle."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _files(d, exts):
    for base, _, names in os.walk(os.path.join(ROOT, d)):
        for n in names:
            if n.endswith(exts) and "_build" not in base:
                yield os.path.join(base, n)


def test_product_does_not_reference_oracle():
    for f in _files("group_scale_search_b200", (".py", ".cu", ".cuh", ".h", ".c")):
        src = open(f).read()
        assert not re.search(r"\boracle\b", src.replace("the oracle", "")), f
        assert "tq_oracle" not in src and "orc_" not in src, f


def test_oracle_does_not_reference_product():
    for f in _files("oracle", (".py", ".c", ".h")):
        src = open(f).read()
        assert "group_scale_search_b200" not in src and "tq.h" not in src and "libtq" not in src, f


def test_input_generators_hold_no_method_arithmetic():
    src = open(os.path.join(ROOT, "synth", "__init__.py")).read()
    for word in ("rint", "round(", "clamp", "argmin", "e4m3", "e2m1", "pack"):
        assert word not in src.lower().replace("round(0.0", "").replace("round(0.001", "").replace(
            "round(0.005", "").replace("round(0.01", "").replace("int(round(n", ""), word
