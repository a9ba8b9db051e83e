"""The repository's own documents stay consistent with it.

* Every repository path that the design notes, the README or a profile names in backticks
  exists.
* Every profile summary gives a command that runs committed files only (`bench.py`), and
  none names a scratch folder.
* No code, comment or test names the build's working documents or the page-source file
  (they are cited by page title and section instead).
"""
import os
import re
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PATH = re.compile(r"`((?:tests|profiles|include|oracle|pruning_hinm_spmm_b200|csrc)/[A-Za-z0-9_./-]+)`")


def _docs():
    out = ["DESIGN" + ".md", "README.md"]
    out += [os.path.join("profiles", f) for f in sorted(os.listdir(os.path.join(ROOT, "profiles")))
            if f.endswith(".md")]
    return out


def test_named_paths_exist():
    missing = []
    for doc in _docs():
        text = open(os.path.join(ROOT, doc), encoding="utf-8").read()
        for m in PATH.finditer(text):
            p = m.group(1).rstrip(".,")
            if not any(os.path.exists(os.path.join(ROOT, base, p))
                       for base in ("", "pruning_hinm_spmm_b200")):
                missing.append(f"{doc}: {p}")
    assert not missing, missing


def test_profile_commands_run_committed_files():
    for doc in _docs():
        if not doc.startswith("profiles"):
            continue
        text = open(os.path.join(ROOT, doc), encoding="utf-8").read()
        blocks = re.findall(r"```\n(.*?)```", text, flags=re.S)
        assert blocks, f"{doc} gives no command"
        assert any("bench.py" in b for b in blocks), f"{doc}: the command does not run bench.py"
        for bad in ("_work", "gpurun_out"):
            assert bad not in text, f"{doc} names {bad}"
        for b in blocks:
            if "ncu " in b:
                assert "--clock-control none" in b, f"{doc}: ncu without --clock-control none"


def test_code_names_no_working_document():
    names = ["BASELINE" + ".json", "north" + "_star", "PAPER" + ".md", "SURVEY" + ".md",
             "VERDICT" + ".md", "ADVICE" + ".md", "DESIGN" + ".md", "BASELINE" + ".md"]
    r = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True)
    if r.returncode == 0:
        files = r.stdout.split()
    else:  # a copy without the history: walk the tree, scratch folders left out
        files = []
        for d, sub, fs in os.walk(ROOT):
            sub[:] = [x for x in sub if x not in (".git", "_work", "gpurun_out", "baseline",
                                                  "__pycache__", "_build")]
            files += [os.path.relpath(os.path.join(d, f), ROOT) for f in fs]
    code = [f for f in files if f.endswith((".py", ".cu", ".cuh", ".h", ".sh"))]
    hits = []
    for f in code:
        text = open(os.path.join(ROOT, f), encoding="utf-8").read()
        hits += [f"{f}: {n}" for n in names if n in text]
    assert not hits, hits
