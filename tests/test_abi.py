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


def test_c_program_plans_decode_batch_and_balanced_items_like_the_binding(tmp_path):
    """A plain C99 program plans a decode step, a batch of sequences and a balanced piece, and
    lists their work items; every field and item equals what the ctypes binding gets from the
    same library (the ABI's structs and arrays read the same from C and from Python)."""
    import numpy as np
    lib = build()
    src = tmp_path / "plan_pa.c"
    src.write_text(r"""
#include <stdio.h>
#include "pa.h"
static void show(const char* tag, const pa_plan_t* p) {
  printf("%s %d %d %d %d %lld %llu %lld\n", tag, p->splits, p->policy, p->batch,
         p->chunk_rows, (long long)p->units, (unsigned long long)p->ws_bytes,
         (long long)p->hist_len);
}
int main(void) {
  pa_plan_t d, b, c;
  int st = pa_decode_plan(148, 16, 2, 256, 16, 32, 32768, PA_F16, 0.0f, 0, &d);
  if (st != PA_OK) return 1;
  show("decode", &d);
  const int32_t q_lens[5] = {300, 1, 0, 2048, 77};
  const int64_t hist[5] = {1000, 40000, 5, 0, 123456};
  st = pa_batch_plan(148, 24, 4, 256, 64, 5, q_lens, hist, PA_BF16, 0.0f, &b);
  if (st != PA_OK) return 2;
  show("batch", &b);
  static int32_t items[4 * 512];
  int n = pa_batch_schedule_items(&b, q_lens, hist, items, 512);
  if (n < 0) return 3;
  printf("batch_items %d", n);
  for (int i = 0; i < 4 * n; ++i) printf(" %d", items[i]);
  printf("\n");
  st = pa_plan(148, 16, 2, 256, 16, 2048, 30720, PA_F16, 0.0f, 0, PA_POLICY_BALANCED, 1, &c);
  if (st != PA_OK) return 4;
  show("piece", &c);
  n = pa_schedule_items(&c, items, 512);
  if (n < 0) return 5;
  printf("piece_items %d", n);
  for (int i = 0; i < 4 * n; ++i) printf(" %d", items[i]);
  printf("\n");
  return 0;
}
""")
    exe = tmp_path / "plan_pa"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lpa", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True,
                           check=True).stdout.splitlines()
    rows = {ln.split()[0]: [int(x) for x in ln.split()[1:]] for ln in lines}

    def fields(p):
        return [p.splits, p.policy, p.batch, p.chunk_rows, p.units, p.ws_bytes, p.hist_len]

    d = binding.decode_plan(16, 2, 256, 16, 32, 32768, "f16", num_sms=148)
    assert rows["decode"] == fields(d)
    q_lens = np.array([300, 1, 0, 2048, 77], dtype=np.int32)
    hist = np.array([1000, 40000, 5, 0, 123456], dtype=np.int64)
    bp = binding.batch_plan(24, 4, 256, 64, q_lens, hist, "bf16", num_sms=148)
    assert rows["batch"] == fields(bp.plan)
    it = binding.batch_schedule_items(bp)
    assert rows["batch_items"][0] == len(it) and rows["batch_items"][1:] == it.ravel().tolist()
    c = binding.plan(16, 2, 256, 16, 2048, 30720, "f16", policy="balanced", num_sms=148)
    assert rows["piece"] == fields(c)
    it = binding.schedule_items(c)
    assert rows["piece_items"][0] == len(it) and rows["piece_items"][1:] == it.ravel().tolist()
    assert len(it) > 0 and (it[:, 3] >= 0).any()       # a balanced piece with cut row blocks
