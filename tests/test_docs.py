"""The documents name only files that exist (CPU only).

README.md point readers to tests, sources, profiles and scripts by path;
a renamed or removed file leaves a dangling reference.  Every backticked path that looks
like a file of this repository must exist.
"""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PREFIXES = ("tests/", "oracle/", "include/", "profiles/", "workloads/", "random_gradient_projection_b200/",
            "csrc/")
SUFFIXES = (".py", ".cu", ".cuh", ".h", ".md", ".json", ".txt")


def _paths(doc):
    text = open(os.path.join(ROOT, doc)).read()
    for tok in re.findall(r"`([^`\s]+)`", text):
        tok = tok.rstrip(".,;:)")
        if tok.startswith(PREFIXES) and tok.endswith(SUFFIXES) and "*" not in tok:
            yield tok


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md"])
def test_every_named_file_exists(doc):
    missing = []
    for p in set(_paths(doc)):
        cands = [os.path.join(ROOT, p)]
        if p.startswith("csrc/"):
            cands.append(os.path.join(ROOT, "random_gradient_projection_b200", p))
        if not any(os.path.exists(c) for c in cands):
            missing.append(p)
    assert not missing, f"{doc} names files that do not exist: {sorted(missing)}"


def test_the_documents_name_some_files():
    assert len(set(_paths("DESIGN.md"))) >= 20
