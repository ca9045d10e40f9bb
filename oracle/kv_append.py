"""Oracle of the KV-append step: the chunk's new K/V rows written into the page pools through
the page table (BaseRT issue #51, "Results": the chunk's K/V are published to pages before
prefill reads every key through the table).

TEST INFRASTRUCTURE ONLY: the correctness reference for ``pa_kv_append``. Only ``tests/`` and
``bench.py`` may import it; it shares no code with the CUDA package.

Plain numpy on the 16-bit patterns, one row at a time, in the order of the definition: row i of
the chunk is position p = H + i, which lives in page ``page_table[p // PS]`` at slot ``p % PS``.
Pinned by ``tests/test_kv_append.py`` (read-back through the table, untouched slots,
composition of two appends, the contiguous special case).
"""
from __future__ import annotations

import numpy as np


def kv_append(pool: np.ndarray, new: np.ndarray, page_table: np.ndarray, hist_len: int):
    """Returns (the pool after the append, number of rows whose page entry was out of range).

    pool: [num_pages, PS, Hkv, D] uint16 bit patterns; new: [R, Hkv, D] uint16;
    page_table: int32. The input pool is not modified."""
    out = pool.copy()
    num_pages, ps = pool.shape[0], pool.shape[1]
    bad = 0
    for i in range(new.shape[0]):
        p = hist_len + i
        e = int(page_table[p // ps])
        if 0 <= e < num_pages:
            out[e, p % ps] = new[i]
        else:
            bad += 1
    return out, bad
