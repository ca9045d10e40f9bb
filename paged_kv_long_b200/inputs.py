"""Seeded synthetic inputs for paged-KV prefill attention.

This module only builds inputs: random 16-bit Q/K/V, a shuffled page pool and its page
table. It holds none of the attention arithmetic, and both the CUDA path and the CPU oracle
take their inputs from it.

Workload shapes follow the pages:
  * 16 Q / 2 KV heads, head_dim 256, F16 KV, page-style prompts of 1K..32K tokens
    (BaseRT issue #51, "Model provenance" and "Single-repetition length sweep");
  * 24 Q / 4 KV heads, D256, bf16 KV, a 2048-row chunk cut into 512-row pieces at 32K
    history and 128-row pieces past 128K history (splash PR #33, "attention-sweep" table;
    beellama.cpp issue #163, "Setup").
Values are N(0, 1) in float32 rounded to nearest-even into the 16-bit type. The page table is
the first ceil((H+R)/PS) entries of a seeded permutation of the pool; unused pool slots hold
NaN in parity runs (they must never reach the output) and zero in timing runs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

NAN_BITS = {"f16": 0x7E00, "bf16": 0x7FC0}


@dataclass(frozen=True)
class Workload:
    """One workload: a sequence of pieces (hist_len, rows) over one shared KV cache."""
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    page_size: int
    dtype: str                      # "f16" or "bf16"
    pieces: tuple                   # ((hist_len, rows), ...) in prefill order
    pool_factor: float = 1.25       # pool pages = ceil(needed * factor)
    exact_pool_pages: int = 0       # if > 0, the pool size (overrides pool_factor)
    splits: int = 0                 # split count fixed by the workload (0: the planner picks)
    scale: float = 0.0              # 0: 1/sqrt(head_dim)
    seed_base: int = 0              # seeds: q +1, k +2, v +3, page permutation +4

    @property
    def first_pos(self) -> int:
        return self.pieces[0][0]

    @property
    def total_keys(self) -> int:
        return max(h + r for h, r in self.pieces)

    @property
    def query_rows(self) -> int:
        return sum(r for _, r in self.pieces)

    @property
    def pages_needed(self) -> int:
        return math.ceil(self.total_keys / self.page_size)

    @property
    def pool_pages(self) -> int:
        if self.exact_pool_pages:
            return self.exact_pool_pages
        return math.ceil(self.pages_needed * self.pool_factor)

    def flops(self) -> float:
        """Algorithmic FLOPs: 4*D*Hq per visible (query, key) pair (QK^T and PV, 2 each)."""
        tot = 0
        for h, r in self.pieces:
            tot += r * h + r * (r + 1) // 2
        return 4.0 * self.head_dim * self.n_q_heads * tot

    def kv_bytes(self) -> float:
        """Algorithmic K+V bytes: every visible key's K and V row read once per piece."""
        return float(sum(2 * (h + r) * self.n_kv_heads * self.head_dim * 2 for h, r in self.pieces))


WORKLOADS = {
    # tiny causal prefill: empty history, 128-token chunk, 8 physical pages shuffled by seed
    "c1": Workload("c1 tiny causal prefill 4q/1kv D64 R128 PS16", 4, 1, 64, 16, "f16",
                   ((0, 128),), exact_pool_pages=8, splits=1, scale=1.0 / 8.0, seed_base=1000),
    # BaseRT attention shape, short: 1,024 tokens from an empty cache in one chunk
    "c2": Workload("c2 16q/2kv D256 PS16 f16, 1024-token chunk from empty cache", 16, 2, 256, 16,
                   "f16", ((0, 1024),), seed_base=2000),
    # 2048-row chunk in four 512-row pieces at 32,768-token history, 4 history splits each
    "c3": Workload("c3 24q/4kv D256 PS64 bf16, 4x512-row pieces at 32K history", 24, 4, 256, 64,
                   "bf16", tuple((32768 + 512 * k, 512) for k in range(4)), splits=4,
                   seed_base=3000),
    # 128-row piece at 131,072-token history, 16 history splits
    "c4": Workload("c4 24q/4kv D256 PS64 bf16, 128-row piece at 131072 history", 24, 4, 256, 64,
                   "bf16", ((131072, 128),), splits=16, seed_base=4000),
    # full 32,768-token prefill in 2,048-token chunks (history 0..30,720)
    "c5": Workload("c5 16q/2kv D256 PS16 f16, 32768-token prefill in 2048-token chunks", 16, 2,
                   256, 16, "f16", tuple((2048 * k, 2048) for k in range(16)), seed_base=5000),
}


def to_bits(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 to nearest-even in the 16-bit type; return the bit patterns (uint16)."""
    if dtype == "f16":
        return x32.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch
        t = torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)
    raise ValueError(dtype)


def normal_bits(seed: int, shape, dtype: str) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return to_bits(rng.standard_normal(shape, dtype=np.float32), dtype)


@dataclass
class Inputs:
    """Generated tensors (numpy uint16 bit patterns / int32), host side."""
    wl: Workload
    q: np.ndarray            # [query_rows, Hq, D] for positions first_pos .. total_keys-1
    k_logical: np.ndarray    # [total_keys, Hkv, D]
    v_logical: np.ndarray
    k_pool: np.ndarray       # [pool_pages, PS, Hkv, D]
    v_pool: np.ndarray
    page_table: np.ndarray   # int32 [pages_needed]
    extra: dict = field(default_factory=dict)

    def piece_q(self, idx: int) -> np.ndarray:
        h, r = self.wl.pieces[idx]
        off = h - self.wl.first_pos
        return self.q[off:off + r]


def scatter_to_pool(logical: np.ndarray, page_table: np.ndarray, pool_pages: int, page_size: int,
                    fill_bits: int) -> np.ndarray:
    """Place logical rows [T, Hkv, D] into a pool [pool_pages, PS, Hkv, D] through the table."""
    T, Hkv, D = logical.shape
    pool = np.full((pool_pages, page_size, Hkv, D), fill_bits, dtype=np.uint16)
    n_full = T // page_size
    if n_full:
        pool[page_table[:n_full]] = logical[:n_full * page_size].reshape(n_full, page_size, Hkv, D)
    rem = T - n_full * page_size
    if rem:
        pool[page_table[n_full], :rem] = logical[n_full * page_size:]
    return pool


def generate(wl: Workload | str, poison: bool = True, distribution: str = "normal") -> Inputs:
    """Seeded inputs for a workload. distribution: "normal" (N(0,1)), or "ramp" — N(0,1)
    plus a key-position ramp along one direction, so that the running max grows along the
    history (exercises the rescaling branch of an online softmax)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    T, Hkv, D, Hq = wl.total_keys, wl.n_kv_heads, wl.head_dim, wl.n_q_heads
    s = wl.seed_base
    rows = T - wl.first_pos
    rng_q = np.random.default_rng(s + 1)
    rng_k = np.random.default_rng(s + 2)
    rng_v = np.random.default_rng(s + 3)
    q32 = rng_q.standard_normal((rows, Hq, D), dtype=np.float32)
    k32 = rng_k.standard_normal((T, Hkv, D), dtype=np.float32)
    v32 = rng_v.standard_normal((T, Hkv, D), dtype=np.float32)
    if distribution == "ramp":
        q32[..., 0] = 4.0
        k32[..., 0] += (np.arange(T, dtype=np.float32) * (64.0 / max(T, 1)))[:, None]
    elif distribution != "normal":
        raise ValueError(distribution)
    q = to_bits(q32, wl.dtype)
    del q32
    k = to_bits(k32, wl.dtype)
    del k32
    v = to_bits(v32, wl.dtype)
    del v32
    perm = np.random.default_rng(s + 4).permutation(wl.pool_pages).astype(np.int32)
    table = np.ascontiguousarray(perm[:wl.pages_needed])
    fill = NAN_BITS[wl.dtype] if poison else 0
    k_pool = scatter_to_pool(k, table, wl.pool_pages, wl.page_size, fill)
    v_pool = scatter_to_pool(v, table, wl.pool_pages, wl.page_size, fill)
    return Inputs(wl, q, k, v, k_pool, v_pool, table)


def small_problem(seed: int, R: int, H: int, Hq: int, Hkv: int, D: int, PS: int, dtype: str,
                  pool_extra: int = 2, poison: bool = True):
    """A small random paged problem for brute-force checks. Returns (q, k_pool, v_pool,
    page_table, k_logical, v_logical)."""
    rng = np.random.default_rng(seed)
    T = H + R
    n_pages = max(1, math.ceil(T / PS))
    pool_pages = n_pages + pool_extra
    q = to_bits(rng.standard_normal((R, Hq, D), dtype=np.float32), dtype)
    k = to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), dtype)
    v = to_bits(rng.standard_normal((T, Hkv, D), dtype=np.float32), dtype)
    table = rng.permutation(pool_pages).astype(np.int32)[:n_pages].copy()
    fill = NAN_BITS[dtype] if poison else 0
    k_pool = scatter_to_pool(k, table, pool_pages, PS, fill)
    v_pool = scatter_to_pool(v, table, pool_pages, PS, fill)
    return q, k_pool, v_pool, table, k, v


@dataclass
class DecodeBatch:
    """One batched decode step over a shared page pool (host side, 16-bit patterns / int32).

    Sequence b holds seq_lens[b] keys (its new token's included) on the pages
    block_table[b, :ceil(seq_lens[b]/PS)]; its one query token is q[b]. The pages of different
    sequences are disjoint; table entries past a sequence's pages are -1, and pool slots that
    no sequence owns hold NaN, so neither may reach an output.
    """
    q: np.ndarray            # [B, Hq, D]
    k_pool: np.ndarray       # [pool_pages, PS, Hkv, D]
    v_pool: np.ndarray
    block_table: np.ndarray  # int32 [B, max_pages]
    seq_lens: np.ndarray     # int32 [B]
    dtype: str
    scale: float = 0.0


def decode_batch(seed: int, seq_lens, Hq: int, Hkv: int, D: int, PS: int, dtype: str,
                 pool_factor: float = 1.1, poison: bool = True) -> DecodeBatch:
    """Seeded N(0, 1) Q/K/V for a batch of sequences of the given key counts; the pages of all
    sequences are drawn from one shuffled pool."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    B = len(lens)
    pages = [max(0, math.ceil(int(n) / PS)) for n in lens]
    need = sum(pages)
    pool_pages = max(1, math.ceil(need * pool_factor))
    max_pages = max(1, max(pages))
    rng = np.random.default_rng(seed)
    perm = rng.permutation(pool_pages).astype(np.int32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    fill = NAN_BITS[dtype] if poison else 0
    k_pool = np.full((pool_pages, PS, Hkv, D), fill, dtype=np.uint16)
    v_pool = np.full((pool_pages, PS, Hkv, D), fill, dtype=np.uint16)
    q = to_bits(rng.standard_normal((B, Hq, D), dtype=np.float32), dtype)
    at = 0
    for b in range(B):
        n, p = int(lens[b]), pages[b]
        table[b, :p] = perm[at:at + p]
        at += p
        if n:
            k = to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
            v = to_bits(rng.standard_normal((n, Hkv, D), dtype=np.float32), dtype)
            _place(k_pool, k, table[b, :p], PS)
            _place(v_pool, v, table[b, :p], PS)
    return DecodeBatch(q, k_pool, v_pool, table, lens.astype(np.int32), dtype)


def _place(pool: np.ndarray, logical: np.ndarray, pages: np.ndarray, PS: int):
    """Write logical rows [n, Hkv, D] into the pool pages listed in order (in place)."""
    n = logical.shape[0]
    full = n // PS
    if full:
        pool[pages[:full]] = logical[:full * PS].reshape(full, PS, *logical.shape[1:])
    if n - full * PS:
        pool[pages[full], :n - full * PS] = logical[full * PS:]


@dataclass
class SeqBatch:
    """A batch of chunks over one shared page pool (host side): sequence b has hist_lens[b]
    keys of history and q_lens[b] query rows (whose K/V are in the pool too), on the pages
    block_table[b, :ceil((hist + rows)/PS)]; its rows are q[q_row0[b] : q_row0[b] + q_lens[b]].
    Pages of different sequences are disjoint; table padding is -1, unowned slots NaN."""
    q: np.ndarray            # [sum q_lens, Hq, D]
    k_pool: np.ndarray
    v_pool: np.ndarray
    block_table: np.ndarray  # int32 [B, max_pages]
    q_lens: np.ndarray       # int32 [B]
    hist_lens: np.ndarray    # int64 [B]
    dtype: str
    scale: float = 0.0

    @property
    def q_row0(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)[:-1]]).astype(np.int64)


def seq_batch(seed: int, hist_lens, q_lens, Hq: int, Hkv: int, D: int, PS: int, dtype: str,
              pool_factor: float = 1.1, poison: bool = True) -> SeqBatch:
    """Seeded N(0, 1) inputs for a batch of chunks: sequence b keeps hist_lens[b] + q_lens[b]
    keys on its own shuffled pages of one pool."""
    hist = np.asarray(hist_lens, dtype=np.int64)
    rows = np.asarray(q_lens, dtype=np.int32)
    keys = hist + rows
    db = decode_batch(seed, keys, Hq, Hkv, D, PS, dtype, pool_factor, poison)
    rng = np.random.default_rng(seed + 7)
    q = to_bits(rng.standard_normal((int(rows.sum()), Hq, D), dtype=np.float32), dtype)
    return SeqBatch(q, db.k_pool, db.v_pool, db.block_table, rows, hist, dtype)
