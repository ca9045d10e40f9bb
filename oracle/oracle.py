"""ctypes wrapper of the fp64 CPU oracle (``pa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the correctness reference for the CUDA path. Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline / reference leg may import it.
It imports nothing from the CUDA package and the CUDA package never imports it.

The oracle computes plain causal GQA attention of a query chunk against its whole history,
reading K/V through the page table (BaseRT issue #51, "Reproduction"; splash PR #33,
"Testing": a CPU reference). See ``pa_oracle.c`` for the formula and the readings taken
where the pages are silent.

Every function here is pinned by ``tests/test_oracle_pins.py`` against brute force in numpy,
torch's fp64 scaled-dot-product attention, closed forms and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pa_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

F16, BF16 = 0, 1
_DTYPE_CODE = {"f16": F16, "bf16": BF16}


def build(force: bool = False, mutant: int = 0, out_path: str | None = None) -> str:
    """Compile the oracle with gcc (OpenMP). ``mutant`` > 0 builds a deliberately broken
    variant for the pin tests; it is never written to the default path."""
    path = out_path or LIB
    if mutant and path == LIB:
        raise ValueError("mutant oracles must not overwrite the real oracle")
    if not force and not mutant and os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(SRC):
        return path
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", f"-DORC_MUTANT={mutant}",
           SRC, "-o", path + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(path + ".tmp", path)
    return path


class _Problem(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("paged", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("num_pages", ctypes.c_int64), ("table_len", ctypes.c_int64), ("hist_len", ctypes.c_int64),
        ("chunk_rows", ctypes.c_int64), ("scale", ctypes.c_double),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p),
    ]


_libs: dict[str, ctypes.CDLL] = {}


def load(path: str | None = None) -> ctypes.CDLL:
    path = path or build()
    lib = _libs.get(path)
    if lib is None:
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(_Problem)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32p = ctypes.POINTER(ctypes.c_int32)
        f64p = ctypes.POINTER(ctypes.c_double)
        lib.orc_attend.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, i64p, i32p,
                                   f64p, f64p, ctypes.c_int]
        lib.orc_attend.restype = ctypes.c_int
        lib.orc_weights.argtypes = [P, ctypes.c_int64, ctypes.c_int32, f64p]
        lib.orc_weights.restype = ctypes.c_int
        lib.orc_merge.argtypes = [ctypes.c_int, ctypes.c_int, f64p, f64p, f64p, f64p]
        lib.orc_merge.restype = None
        lib.orc_decode.argtypes = [ctypes.c_int, ctypes.c_uint16]
        lib.orc_decode.restype = ctypes.c_double
        lib.orc_max_threads.restype = ctypes.c_int
        _libs[path] = lib
    return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


@dataclass
class Problem:
    """One chunk of prefill attention, in the caller's 16-bit bit patterns (uint16 arrays).

    q: [R, Hq, D]; paged: k, v are pools [num_pages, PS, Hkv, D] and page_table int32
    [ceil((H+R)/PS)] (or longer); contiguous: k, v are [H+R, Hkv, D].
    """
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    hist_len: int
    dtype: str
    page_table: np.ndarray | None = None
    scale: float = 0.0
    lib_path: str | None = None
    _keep: list = field(default_factory=list, repr=False)

    def __post_init__(self):
        for name in ("q", "k", "v"):
            a = getattr(self, name)
            assert a.dtype == np.uint16, f"{name} must hold 16-bit patterns as uint16"
            setattr(self, name, np.ascontiguousarray(a))
        if self.page_table is not None:
            self.page_table = np.ascontiguousarray(self.page_table, dtype=np.int32)

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    @property
    def chunk_rows(self) -> int:
        return self.q.shape[0]

    @property
    def n_q_heads(self) -> int:
        return self.q.shape[1]

    @property
    def head_dim(self) -> int:
        return self.q.shape[2]

    @property
    def n_kv_heads(self) -> int:
        return self.k.shape[2] if self.paged else self.k.shape[1]

    def _c(self) -> _Problem:
        p = _Problem()
        p.dtype = _DTYPE_CODE[self.dtype]
        p.paged = 1 if self.paged else 0
        p.page_size = self.k.shape[1] if self.paged else 0
        p.n_q_heads = self.n_q_heads
        p.n_kv_heads = self.n_kv_heads
        p.head_dim = self.head_dim
        p.num_pages = self.k.shape[0] if self.paged else 0
        p.table_len = len(self.page_table) if self.paged else 0
        p.hist_len = self.hist_len
        p.chunk_rows = self.chunk_rows
        p.scale = float(self.scale)
        p.q = self.q.ctypes.data
        p.k = self.k.ctypes.data
        p.v = self.v.ctypes.data
        p.page_table = self.page_table.ctypes.data if self.paged else None
        if not self.paged and self.k.shape[0] < self.hist_len + self.chunk_rows:
            raise ValueError("contiguous K/V must hold H+R positions")
        return p


def attend(pb: Problem, rows=None, heads=None, key_lo: int = 0, key_hi: int | None = None,
           threads: int = 0):
    """fp64 attention output and natural-log LSE for (row, head) samples.

    rows/heads: equal-length int arrays of chunk-relative rows and Q heads; None = every
    (row, head) pair in row-major order. Returns out [n, D] float64 and lse [n] float64.
    """
    if rows is None:
        rr, hh = np.meshgrid(np.arange(pb.chunk_rows), np.arange(pb.n_q_heads), indexing="ij")
        rows, heads = rr.ravel(), hh.ravel()
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    heads = np.ascontiguousarray(heads, dtype=np.int32)
    if key_hi is None:
        key_hi = pb.hist_len + pb.chunk_rows
    n = len(rows)
    out = np.zeros((n, pb.head_dim), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    lib = load(pb.lib_path)
    cp = pb._c()
    rc = lib.orc_attend(ctypes.byref(cp), key_lo, key_hi, n, _ptr(rows, ctypes.c_int64),
                        _ptr(heads, ctypes.c_int32), _ptr(out, ctypes.c_double),
                        _ptr(lse, ctypes.c_double), threads)
    if rc != 0:
        raise RuntimeError(f"oracle attend failed with status {rc}")
    return out, lse


def weights(pb: Problem, row: int, head: int) -> np.ndarray:
    """Normalised softmax weights of one (row, head) over keys 0..H+R-1."""
    w = np.zeros(pb.hist_len + pb.chunk_rows, dtype=np.float64)
    cp = pb._c()
    rc = load(pb.lib_path).orc_weights(ctypes.byref(cp), row, head, _ptr(w, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"oracle weights failed with status {rc}")
    return w


def merge(lse_parts: np.ndarray, o_parts: np.ndarray, lib_path: str | None = None):
    """Log-sum-exp merge of S partials of one (row, head): lse [S], o [S, D]."""
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    S, D = o_parts.shape
    out = np.zeros(D, dtype=np.float64)
    lse = ctypes.c_double(0.0)
    load(lib_path).orc_merge(S, D, _ptr(lse_parts, ctypes.c_double), _ptr(o_parts, ctypes.c_double),
                             _ptr(out, ctypes.c_double), ctypes.byref(lse))
    return out, lse.value


def decode(dtype: str, bits: np.ndarray, lib_path: str | None = None) -> np.ndarray:
    """Exact fp64 value of each 16-bit pattern (the oracle's own decoder)."""
    lib = load(lib_path)
    code = _DTYPE_CODE[dtype]
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([lib.orc_decode(code, int(x)) for x in flat], dtype=np.float64).reshape(np.shape(bits))


def max_threads() -> int:
    return int(load().orc_max_threads())
