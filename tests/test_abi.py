"""The C-ABI library loads on a machine without a GPU and exports every declared symbol."""
import os
import re
import subprocess

from paged_kv_long_b200 import binding
from paged_kv_long_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    path = build()
    lib = binding.load_library()
    declared = declared_functions()
    assert {"pa_plan", "pa_prefill", "pa_combine"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z0-9_]+)", out))
    assert declared <= exported
    assert set(binding.EXPORTED) <= exported


def test_build_targets_sm100a_only():
    from paged_kv_long_b200 import build as b
    assert b.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_oracle_shares_nothing_with_the_library():
    # the oracle neither includes nor imports the CUDA library's files, and vice versa
    oracle_src = open(os.path.join(ROOT, "oracle", "pa_oracle.c")).read()
    assert "#include \"" not in oracle_src
    oracle_py = open(os.path.join(ROOT, "oracle", "oracle.py")).read()
    assert "paged_kv_long_b200" not in oracle_py
    for dirpath, _, files in os.walk(os.path.join(ROOT, "paged_kv_long_b200")):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, flags=re.M), f
                assert "pa_oracle" not in text and "liboracle" not in text, f
