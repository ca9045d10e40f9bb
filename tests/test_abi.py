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


def test_header_is_c99_and_a_c_program_can_plan(tmp_path):
    """include/pa.h compiles as plain C99, and a C program linked against libpa.so calls the
    host-only entry points (no GPU needed): a plan, the pages' piece cut, a status string."""
    lib = build()
    src = tmp_path / "use_pa.c"
    src.write_text(r"""
#include <stdio.h>
#include "pa.h"
int main(void) {
  pa_plan_t p;
  int st = pa_plan(148, 24, 4, 256, 64, 128, 131072, PA_BF16, 0.0f, 16, PA_POLICY_MAKESPAN, 1,
                   &p);
  int32_t rows[16];
  int n = pa_pieces(2048, 32768, 25, rows, 16);
  printf("%d %d %d %lld %llu %d %d %s\n", st, p.splits, p.ctas_per_unit, (long long)p.units,
         (unsigned long long)p.ws_bytes, n, rows[0], pa_status_string(PA_ERR_WORKSPACE));
  return st != PA_OK;
}
""")
    exe = tmp_path / "use_pa"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lpa", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    st, splits, per, units, ws, n, rows0 = (int(x) for x in out[:7])
    assert (st, splits, per) == (0, 16, 2)
    assert units == 4 * 3 * 16        # 128 rows x G 6 = 6 Q tiles = 3 pair units per KV head
    assert ws == 16 * 128 * 24 * (256 + 1) * 4
    assert (n, rows0) == (4, 512)                    # the pages' 512-row pieces at 32K history
    assert " ".join(out[7:]) == binding.load_library().pa_status_string(-3).decode()
