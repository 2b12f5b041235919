"""Source hygiene: what committed code may name and import.

- Code and comments name no build-process file or working folder.
- The CUDA package never imports or loads the oracle; the oracle never
  imports the CUDA package.
- The input generators hold neither side.
"""
import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CODE = (".py", ".cu", ".cuh", ".h", ".cpp", ".ini")
HERE = os.path.relpath(os.path.abspath(__file__), ROOT)


def tracked(prefix=""):
    out = subprocess.run(["git", "ls-files", prefix], cwd=ROOT, capture_output=True, text=True)
    if out.returncode != 0:   # not a git checkout: walk the tree
        files = []
        for d, _, names in os.walk(os.path.join(ROOT, prefix)):
            if "/." in d or "_work" in d or "__pycache__" in d:
                continue
            files += [os.path.relpath(os.path.join(d, n), ROOT) for n in names]
        return files
    return out.stdout.split()


def read(path):
    with open(os.path.join(ROOT, path), encoding="utf-8", errors="replace") as f:
        return f.read()


def test_code_names_no_build_process_files():
    # assembled so that this file does not match itself
    words = ["BASE" + "LINE", "north" + "_star", "PAPER" + r"\.md", "SUR" + "VEY", "VER" + "DICT",
             "ADV" + "ICE", "DESIGN" + r"\.md", "gpu" + "run", "_wo" + "rk/", "/ro" + "ot/"]
    pat = re.compile("|".join(words))
    bad = []
    for f in tracked():
        if f.endswith(CODE) and f != HERE:
            for i, line in enumerate(read(f).splitlines(), 1):
                if pat.search(line) and "MEASURED_PEAKS" not in line:
                    bad.append(f"{f}:{i}: {line.strip()[:100]}")
    assert not bad, "\n".join(bad)


def test_cuda_package_never_touches_the_oracle():
    bad = [f for f in tracked("sparse_attention_10_b200") + tracked("include")
           if f.endswith(CODE) and re.search(r"\boracle\b|dsa_oracle", read(f))]
    assert not bad, bad


def test_oracle_never_touches_the_cuda_package():
    bad = [f for f in tracked("oracle")
           if f.endswith(CODE) and re.search(r"sparse_attention_10_b200|libdsa\.so|dsa\.h|csrc", read(f))]
    assert not bad, bad


def test_input_generators_hold_neither_side():
    bad = [f for f in tracked("synth")
           if f.endswith(CODE) and re.search(r"import oracle|from oracle|sparse_attention_10_b200|libdsa",
                                             read(f))]
    assert not bad, bad
