"""Structural checks on the separation between the product and its test oracle (no GPU):
the package never imports, loads or names the oracle; the oracle never imports the package;
the CUDA sources include no oracle file and the oracle's C file includes no library header;
and nothing committed reaches into the working folder."""
from __future__ import annotations

import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "activation_quantization_block_b200")


def _tracked(*prefixes):
    out = subprocess.run(["git", "ls-files", *prefixes], cwd=ROOT, capture_output=True, text=True)
    if out.returncode != 0:   # not a git checkout: fall back to a walk
        files = []
        for p in prefixes:
            for d, _, fs in os.walk(os.path.join(ROOT, p)):
                files += [os.path.relpath(os.path.join(d, f), ROOT) for f in fs]
        return files
    return [l for l in out.stdout.splitlines() if l]


def _read(rel):
    with open(os.path.join(ROOT, rel), encoding="utf-8", errors="replace") as f:
        return f.read()


def test_the_package_never_reaches_the_oracle():
    for rel in _tracked("activation_quantization_block_b200"):
        if not rel.endswith((".py", ".cu", ".cuh", ".h")):
            continue
        text = _read(rel)
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), rel
        assert "fp4q_oracle" not in text and "orc_" not in text, rel


def test_the_oracle_never_reaches_the_package():
    for rel in _tracked("oracle"):
        if not rel.endswith((".py", ".c", ".h")):
            continue
        text = _read(rel)
        # the seeded input generators are the one shared module, and they hold no quantization arithmetic
        for sub, names in re.findall(r"from\s+activation_quantization_block_b200(\.\w+)?\s+import\s+([\w, ]+)", text):
            used = {sub.lstrip(".")} if sub else {n.strip() for n in names.split(",")}
            assert used <= {"synthetic"}, (rel, used)
        assert not re.search(r"^\s*import\s+activation_quantization_block_b200", text, re.M), rel
        assert "libfp4q.so" not in text and '#include "fp4q' not in text, rel


def test_cuda_sources_include_only_their_own_headers():
    for rel in _tracked("activation_quantization_block_b200/csrc", "include"):
        for inc in re.findall(r'#include\s+"([^"]+)"', _read(rel)):
            assert not inc.startswith("oracle") and "orc" not in inc, (rel, inc)


def test_nothing_committed_uses_the_working_folder():
    for rel in _tracked():
        if rel.startswith("_work/") or rel.endswith(".md") or rel in (".gitignore", "tests/test_independence.py"):
            continue
        assert "_work/" not in _read(rel), rel


def test_profile_summaries_name_committed_commands_only():
    """Each ncu summary under profiles/ gives the command that made it, and that command runs
    committed files (bench.py or the package's kernel_bench), never a working-folder script."""
    for rel in _tracked("profiles"):
        if not rel.endswith(".md"):
            continue
        text = _read(rel)
        assert "_work" not in text, rel
        assert "ncu " in text and ("python bench.py" in text or "activation_quantization_block_b200.kernel_bench" in text), rel
