"""Repository rules that can be checked by reading the files: the product
package never reaches the oracle (no fallback to it), nothing committed runs or
reads the git-ignored scratch folder, and the command in every profile summary
runs only files of the repository."""
import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_attention_bifocal_b200")
SCRATCH = "_" + "work/"  # spelled in two parts so this file does not match itself


def _tracked():
    out = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True)
    if out.returncode != 0:  # not a git checkout: walk the tree instead
        files = []
        for d, dirs, names in os.walk(ROOT):
            dirs[:] = [x for x in dirs if not x.startswith((".", "_"))]
            files += [os.path.relpath(os.path.join(d, n), ROOT) for n in names]
        return files
    return out.stdout.split()


def _text_files(paths):
    for rel in paths:
        if rel.endswith((".py", ".cu", ".cuh", ".h", ".c", ".md", ".txt", ".sh", ".json")):
            p = os.path.join(ROOT, rel)
            if os.path.isfile(p):
                yield rel, open(p, encoding="utf-8", errors="replace").read()


def test_product_package_does_not_import_the_oracle():
    for d, _, names in os.walk(PKG):
        for n in names:
            if n.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(d, n), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), n
                assert "jl_oracle" not in src and "libjloracle" not in src, n


def test_nothing_committed_uses_the_scratch_folder():
    for rel, src in _text_files(_tracked()):
        if rel.startswith(("SURVEY", "BASELINE", "VERDICT", "ADVICE", "DESIGN")):
            continue
        assert SCRATCH not in src, rel


def test_profile_commands_run_committed_files():
    tracked = set(_tracked())
    prof = os.path.join(ROOT, "profiles")
    for n in sorted(os.listdir(prof)):
        src = open(os.path.join(prof, n), encoding="utf-8").read()
        scripts = re.findall(r"\bpython3?\s+(?:-m\s+\S+\s+)?([\w./-]+\.py)\b", src)
        assert scripts, f"{n}: no command found"
        for s in scripts:
            assert not s.startswith(SCRATCH), (n, s)
            assert s in tracked, (n, s)
