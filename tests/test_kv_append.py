"""KV append (pa_kv_append): the chunk's new K/V rows written into the page pools through the
page table, the step before prefill.

CPU tests pin the numpy oracle (oracle/kv_append.py) to properties the definition fixes: reading
the pool back through the table returns the new rows at their positions, every other slot keeps
its bits, two appends compose into one, and with an identity table the pool is the contiguous
cache. GPU tests compare the CUDA kernel with the oracle bit for bit, check the bad-page report,
and run append -> prefill end to end against the attention oracle.
"""
import math

import numpy as np
import pytest

from oracle.kv_append import kv_append as oracle_append
from tests.conftest import cuda_available

SHAPES = [
    # Hkv, D, PS, H, R
    (2, 256, 16, 0, 1024),
    (2, 256, 16, 30720, 2048),
    (4, 256, 64, 32768 + 37, 512),   # history ends inside a page
    (1, 64, 16, 5, 3),
    (8, 128, 128, 1000, 300),
    (3, 64, 32, 95, 1),
]


def make(Hkv, D, PS, H, R, seed, pool_factor=1.25):
    rng = np.random.default_rng(seed)
    pages = math.ceil((H + R) / PS)
    num_pages = max(pages, math.ceil(pages * pool_factor))
    pool = rng.integers(0, 1 << 16, size=(num_pages, PS, Hkv, D), dtype=np.uint16)
    new = rng.integers(0, 1 << 16, size=(R, Hkv, D), dtype=np.uint16)
    table = rng.permutation(num_pages)[:pages].astype(np.int32)
    return pool, new, table


def gather(pool, table, positions):
    Hkv, D = pool.shape[2], pool.shape[3]
    ps = pool.shape[1]
    flat = pool.reshape(-1, Hkv, D)
    return flat[table[positions // ps].astype(np.int64) * ps + positions % ps]


@pytest.mark.parametrize("idx", range(len(SHAPES)))
def test_oracle_read_back_and_untouched_slots(idx):
    Hkv, D, PS, H, R = SHAPES[idx]
    pool, new, table = make(Hkv, D, PS, H, R, seed=100 + idx)
    out, bad = oracle_append(pool, new, table, H)
    assert bad == 0
    pos = np.arange(H, H + R)
    assert np.array_equal(gather(out, table, pos), new)
    written = np.zeros(pool.shape[:2], dtype=bool)
    written[table[pos // PS], pos % PS] = True
    assert np.array_equal(out[~written], pool[~written])
    assert np.array_equal(pool, make(Hkv, D, PS, H, R, seed=100 + idx)[0]), "input modified"


def test_oracle_two_appends_compose():
    Hkv, D, PS, H, R = 2, 64, 16, 70, 200
    pool, new, table = make(Hkv, D, PS, H, R, seed=7)
    once, _ = oracle_append(pool, new, table, H)
    a = 77
    first, _ = oracle_append(pool, new[:a], table, H)
    twice, _ = oracle_append(first, new[a:], table, H + a)
    assert np.array_equal(once, twice)


def test_oracle_identity_table_is_the_contiguous_cache():
    Hkv, D, PS, H, R = 2, 64, 16, 37, 100
    pool, new, _ = make(Hkv, D, PS, H, R, seed=8, pool_factor=1.0)
    table = np.arange(pool.shape[0], dtype=np.int32)
    out, _ = oracle_append(pool, new, table, H)
    flat = out.reshape(-1, Hkv, D)
    assert np.array_equal(flat[H:H + R], new)
    assert np.array_equal(flat[:H], pool.reshape(-1, Hkv, D)[:H])


def test_oracle_bad_entries_are_skipped():
    Hkv, D, PS, H, R = 1, 64, 16, 0, 64
    pool, new, table = make(Hkv, D, PS, H, R, seed=9)
    table[1] = pool.shape[0] + 3
    out, bad = oracle_append(pool, new, table, H)
    assert bad == 16
    pos = np.arange(0, 16)
    assert np.array_equal(gather(out, table, pos), new[:16])


# ---------------------------------------------------------------------------------- GPU


def _dev(bits, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def _host(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("idx", range(len(SHAPES)))
def test_gpu_append_is_bit_exact(idx):
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.build import build
    build()
    binding.device_error(reset=True)
    Hkv, D, PS, H, R = SHAPES[idx]
    dtype = "bf16" if idx % 2 else "f16"
    kp, kn, table = make(Hkv, D, PS, H, R, seed=200 + idx)
    vp, vn, _ = make(Hkv, D, PS, H, R, seed=300 + idx)
    want_k, _ = oracle_append(kp, kn, table, H)
    want_v, _ = oracle_append(vp, vn, table, H)
    dkp, dvp = _dev(kp, dtype), _dev(vp, dtype)
    binding.kv_append(_dev(kn, dtype), _dev(vn, dtype), dkp, dvp,
                      torch.from_numpy(table).cuda(), H)
    torch.cuda.synchronize()
    assert np.array_equal(_host(dkp), want_k)
    assert np.array_equal(_host(dvp), want_v)
    assert binding.device_error(reset=True)[0] == 0


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_bad_page_entry_is_reported_and_skipped():
    import torch
    from paged_kv_long_b200 import binding
    binding.device_error(reset=True)
    Hkv, D, PS, H, R = 2, 64, 16, 0, 64
    kp, kn, table = make(Hkv, D, PS, H, R, seed=11)
    table[2] = -1
    want, bad = oracle_append(kp, kn, table, H)
    assert bad == 16
    dkp, dvp = _dev(kp, "f16"), _dev(kp.copy(), "f16")
    binding.kv_append(_dev(kn, "f16"), _dev(kn, "f16"), dkp, dvp,
                      torch.from_numpy(table).cuda(), H)
    st, flags = binding.device_error(reset=True)
    assert binding.STATUS[st] == "PA_ERR_PAGE_INDEX" and flags & 1
    assert np.array_equal(_host(dkp), want)


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_append_then_prefill_matches_attention_oracle():
    """The pool holds only the history; the chunk's K/V arrive by pa_kv_append, then pa_prefill
    reads all keys through the table."""
    import torch
    from paged_kv_long_b200 import binding
    from tests import parity_util as U
    wl = U.custom_workload("append+prefill", 16, 2, 256, 16, "f16", [(600, 300)], seed=4242)
    inp = U.gen(wl)
    h, r = wl.pieces[0]
    PS = wl.page_size
    pos = np.arange(h, h + r)
    k_pool = inp.k_pool.copy()
    v_pool = inp.v_pool.copy()
    nan = np.uint16(0x7E00)
    k_pool[inp.page_table[pos // PS], pos % PS] = nan   # the chunk's slots start as NaN
    v_pool[inp.page_table[pos // PS], pos % PS] = nan
    dk, dv = _dev(k_pool, "f16"), _dev(v_pool, "f16")
    tab = torch.from_numpy(inp.page_table).cuda()
    binding.kv_append(_dev(inp.k_logical[h:h + r], "f16"), _dev(inp.v_logical[h:h + r], "f16"),
                      dk, dv, tab, h)
    p = binding.plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, PS, r, h, "f16")
    out = binding.prefill_combine(p, _dev(inp.piece_q(0), "f16"), dk, dv, tab)
    torch.cuda.synchronize()
    from oracle import oracle
    ref, _ = oracle.attend(U.oracle_problem(inp, 0))
    U.assert_close(out.cpu().numpy().reshape(ref.shape), ref, "append -> prefill")
