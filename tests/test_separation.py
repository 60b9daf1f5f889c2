"""The oracle and the product path share no code and never import each
other; the oracle is test infrastructure only."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "token_sparse_attention_sm_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _sources(top, exts):
    for dirpath, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_product_never_references_oracle():
    pat = re.compile(r"\boracle\b")
    for path in _sources(PKG, (".py", ".cu", ".cuh", ".h", ".cpp", ".c")):
        for line in open(path, encoding="utf-8"):
            code = line.split("#")[0] if path.endswith(".py") else line.split("//")[0]
            if "import" in code or "include" in code or "dlopen" in code or "CDLL" in code:
                assert not pat.search(code), f"{path}: {line.strip()}"


def test_oracle_never_references_product():
    for path in _sources(ORACLE, (".py", ".c", ".h")):
        text = open(path, encoding="utf-8").read()
        assert "token_sparse_attention_sm_b200" not in text, path
        assert "sparse_decode" not in text, path
