"""Batched paged decode (pa_decode_plan, pa_decode): one new query token per sequence, every
key of its own sequence visible, K/V read through that sequence's row of the block table.

Decode attention of sequence b is the prefill definition with one chunk row: the query at
position len_b - 1 sees keys 0 .. len_b - 1. The oracle is therefore oracle.attend on the
one-row problem of each sequence; the CPU tests pin that use of it (the table row, the length)
to a brute-force softmax and to closed forms, and check the planner and the argument checks of
the C ABI. GPU tests compare pa_decode (+ pa_combine) with the oracle element by element.
"""
import ctypes
import math
import zlib

import numpy as np
import pytest

from oracle import oracle
from paged_kv_long_b200.inputs import decode_batch
from tests.conftest import cuda_available
from tests import parity_util as U


def seq_problem(db, b: int) -> oracle.Problem:
    """The one-row prefill problem equal to decode of sequence b (len >= 1)."""
    n = int(db.seq_lens[b])
    PS = db.k_pool.shape[1]
    pages = db.block_table[b, :math.ceil(n / PS)]
    return oracle.Problem(q=db.q[b:b + 1], k=db.k_pool, v=db.v_pool, hist_len=n - 1,
                          dtype=db.dtype, page_table=pages, scale=db.scale)


def oracle_decode(db) -> np.ndarray:
    """fp64 [B, Hq, D]; a sequence with no key is zero."""
    B, Hq, D = db.q.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        if db.seq_lens[b] > 0:
            o, _ = oracle.attend(seq_problem(db, b))
            out[b] = o.reshape(Hq, D)
    return out


def brute_decode(db, b: int) -> np.ndarray:
    """Plain numpy softmax of sequence b through its table row (tiny cases only)."""
    n = int(db.seq_lens[b])
    _, Hq, D = db.q.shape
    PS, Hkv = db.k_pool.shape[1], db.k_pool.shape[2]
    G = Hq // Hkv
    pos = np.arange(n)
    phys = db.block_table[b, pos // PS].astype(np.int64)
    k = oracle.decode(db.dtype, db.k_pool[phys, pos % PS])  # [n, Hkv, D]
    v = oracle.decode(db.dtype, db.v_pool[phys, pos % PS])
    q = oracle.decode(db.dtype, db.q[b])                   # [Hq, D]
    scale = db.scale or 1.0 / math.sqrt(D)
    out = np.zeros((Hq, D))
    for h in range(Hq):
        s = k[:, h // G, :] @ q[h] * scale
        w = np.exp(s - s.max())
        out[h] = (w / w.sum()) @ v[:, h // G, :]
    return out


# ------------------------------------------------------------------------------ oracle pins


def test_oracle_decode_matches_brute_force_through_the_table():
    db = decode_batch(11, [1, 15, 16, 17, 40, 3], Hq=4, Hkv=2, D=64, PS=16, dtype="f16")
    got = oracle_decode(db)
    for b in range(len(db.seq_lens)):
        np.testing.assert_allclose(got[b], brute_decode(db, b), rtol=1e-12, atol=1e-12)


def test_oracle_decode_one_key_returns_that_value_row():
    db = decode_batch(12, [1, 1], Hq=6, Hkv=3, D=64, PS=32, dtype="bf16")
    got = oracle_decode(db)
    for b in range(2):
        page = db.block_table[b, 0]
        v = oracle.decode("bf16", db.v_pool[page, 0])  # [Hkv, D]
        np.testing.assert_array_equal(got[b], np.repeat(v, 2, axis=0))


def test_oracle_decode_equal_keys_average_the_values():
    """All keys equal: the weights are uniform, the output is the mean of V."""
    db = decode_batch(13, [37], Hq=2, Hkv=1, D=64, PS=16, dtype="f16")
    n, PS = 37, 16
    pos = np.arange(n)
    phys = db.block_table[0, pos // PS]
    db.k_pool[phys, pos % PS] = db.k_pool[phys[0], 0]
    v = oracle.decode("f16", db.v_pool[phys, pos % PS])
    got = oracle_decode(db)
    np.testing.assert_allclose(got[0], np.repeat(v.mean(axis=0), 2, axis=0), atol=1e-12)


def test_generator_pages_are_disjoint_and_padding_is_minus_one():
    db = decode_batch(14, [0, 5, 16, 33, 100], Hq=2, Hkv=1, D=64, PS=16, dtype="f16")
    used = []
    for b, n in enumerate(db.seq_lens):
        p = math.ceil(int(n) / 16)
        used += list(db.block_table[b, :p])
        assert (db.block_table[b, p:] == -1).all()
    assert len(used) == len(set(used))


# ------------------------------------------------------------------------------ planner / ABI


def _binding():
    from paged_kv_long_b200 import binding
    return binding


def test_decode_plan_fields_and_workspace():
    bd = _binding()
    p = bd.decode_plan(16, 2, 256, 16, batch=8, max_seq_len=32768, dtype="f16", num_sms=148)
    assert p.batch == 8 and p.chunk_rows == 8 and p.q_tiles == 1 and p.ctas_per_unit == 1
    S = p.splits
    # G = 8 at head dim 256: the swapped-operand kernel, two CTA slots per SM, two units each
    assert S == min(32, math.ceil(2 * 2 * 148 / (8 * 2)))
    assert p.units == 8 * 2 * S
    assert p.ws_bytes == S * 8 * 16 * (256 + 1) * 4
    assert abs(p.scale - 1 / 16) < 1e-7


def test_decode_plan_splits_bounded_by_tiles_and_override():
    bd = _binding()
    p = bd.decode_plan(8, 1, 128, 16, batch=1, max_seq_len=300, dtype="bf16", num_sms=148)
    assert p.splits == 3                     # three 128-key tiles
    # the batch alone gives two units per CTA slot (2 x 148 slots of the swapped kernel)
    p = bd.decode_plan(8, 1, 128, 16, batch=600, max_seq_len=1 << 20, dtype="bf16", num_sms=148)
    assert p.splits == 1 and p.ws_bytes == 0
    p = bd.decode_plan(8, 1, 128, 16, batch=512, max_seq_len=1 << 20, dtype="bf16", num_sms=148)
    assert p.splits == 2
    p = bd.decode_plan(16, 1, 128, 16, batch=512, max_seq_len=1 << 20, dtype="bf16", num_sms=148)
    assert p.splits == 1                      # G = 16: one CTA slot per SM
    p = bd.decode_plan(8, 1, 128, 16, batch=2, max_seq_len=4096, dtype="bf16", splits=5,
                       num_sms=148)
    assert p.splits == 5 and p.units == 2 * 1 * 5


@pytest.mark.parametrize("args", [
    dict(n_q_heads=16, n_kv_heads=2, head_dim=256, page_size=16, batch=0, max_seq_len=10),
    dict(n_q_heads=16, n_kv_heads=2, head_dim=256, page_size=16, batch=4, max_seq_len=0),
    dict(n_q_heads=16, n_kv_heads=3, head_dim=256, page_size=16, batch=4, max_seq_len=10),
    dict(n_q_heads=16, n_kv_heads=2, head_dim=96, page_size=16, batch=4, max_seq_len=10),
    dict(n_q_heads=16, n_kv_heads=2, head_dim=256, page_size=24, batch=4, max_seq_len=10),
    dict(n_q_heads=256, n_kv_heads=1, head_dim=64, page_size=16, batch=4, max_seq_len=10),
])
def test_decode_plan_rejects(args):
    bd = _binding()
    with pytest.raises(bd.PaError):
        bd.decode_plan(dtype="f16", num_sms=148, **args)


def test_prefill_and_decode_refuse_each_others_plans():
    """Checked before any device work, so this runs without a GPU."""
    bd = _binding()
    lib = bd.load_library()
    dp = bd.decode_plan(16, 2, 256, 16, batch=4, max_seq_len=1000, dtype="f16", num_sms=148)
    fake = ctypes.c_void_p(1 << 20)
    st = lib.pa_prefill(ctypes.byref(dp), fake, fake, fake, fake, 100, dp.hist_len, 4, fake,
                        fake, 1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    pp = bd.plan(16, 2, 256, 16, 512, 4096, "f16", num_sms=148)
    st = lib.pa_decode(ctypes.byref(pp), fake, fake, fake, fake, 8, fake, 100, fake, fake,
                       1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"


# ------------------------------------------------------------------------------ GPU parity

CASES = [
    # name, seq_lens, Hq, Hkv, D, PS, dtype, splits (0: planner)
    ("d256_ragged", [1, 16, 17, 127, 128, 129, 1000, 4097], 16, 2, 256, 16, "f16", 0),
    ("d256_bf16_s1", [300, 2, 5000, 64], 24, 4, 256, 64, "bf16", 1),
    ("d256_many_splits", [9000, 1, 130], 16, 2, 256, 16, "f16", 32),
    ("d128_empty_and_one", [0, 1, 255, 256, 257, 0], 32, 8, 128, 32, "bf16", 0),
    ("d128_empty_s1", [0, 3, 1], 8, 8, 128, 16, "f16", 1),
    ("d64_g16", [700, 64, 1500], 32, 2, 64, 128, "f16", 0),
    ("d64_g1", [33, 800], 4, 4, 64, 16, "bf16", 4),
    ("d64_24_splits", [3000, 5, 130], 8, 1, 64, 16, "f16", 24),
    # G > 8 at head dim 256: the single-CTA kernel with a whole Q tile (not the swapped one)
    ("d256_g16_unswapped", [2000, 129, 5], 32, 2, 256, 16, "bf16", 0),
    # the swapped kernel with V boxes of 32 keys (D 256) and 64 keys (D 128)
    ("d256_ps128", [5000, 128, 1, 257], 8, 1, 256, 128, "f16", 0),
    ("d128_ps128_g8", [4000, 700, 0, 129], 16, 2, 128, 128, "bf16", 0),
]


def _dev(bits, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def run_decode(db, splits=0):
    import torch
    bd = _binding()
    B, Hq, D = db.q.shape
    Hkv, PS = db.k_pool.shape[2], db.k_pool.shape[1]
    p = bd.decode_plan(Hq, Hkv, D, PS, B, max(1, int(db.seq_lens.max())), db.dtype,
                       scale=db.scale, splits=splits)
    out = torch.full((B, Hq, D), float("nan"), device="cuda")  # every entry must be written
    ws = bd.workspace(p)
    if ws is not None:
        ws.fill_(float("nan"))
    out = bd.decode(p, _dev(db.q, db.dtype), _dev(db.k_pool, db.dtype),
                    _dev(db.v_pool, db.dtype), torch.from_numpy(db.block_table).cuda(),
                    torch.from_numpy(db.seq_lens).cuda(), out, ws)
    torch.cuda.synchronize()
    return p, out.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_decode_matches_oracle(case):
    from paged_kv_long_b200.build import build
    build()
    bd = _binding()
    bd.device_error(reset=True)
    name, lens, Hq, Hkv, D, PS, dtype, splits = case
    db = decode_batch(zlib.crc32(name.encode()) & 0xFFFF, lens, Hq, Hkv, D, PS, dtype)
    p, got = run_decode(db, splits)
    assert bd.device_error(reset=True)[0] == 0
    ref = oracle_decode(db)
    empty = db.seq_lens == 0
    assert (got[empty] == 0).all(), f"{name}: empty sequences must give zeros"
    U.assert_close(got[~empty], ref[~empty], f"{name} (S={p.splits})")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_decode_long_batch_sampled():
    """Serving-sized batch (32 sequences of 1K..32K keys, D256, 16/2 heads): every output
    against the oracle."""
    rng = np.random.default_rng(77)
    lens = rng.integers(1024, 32768, size=32)
    db = decode_batch(78, lens, 16, 2, 256, 16, "bf16")
    p, got = run_decode(db)
    assert _binding().device_error(reset=True)[0] == 0
    U.assert_close(got, oracle_decode(db), f"batch32 (S={p.splits})")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("B,max_len,Hkv,D", [(255, 400, 2, 64), (256, 400, 2, 64),
                                              (257, 400, 2, 64), (700, 400, 2, 64),
                                              (600, 6000, 1, 64), (256, 1500, 2, 256),
                                              (300, 1500, 1, 128)])
def test_gpu_decode_longest_first_dispatch_edges(B, max_len, Hkv, D):
    """Blocks go to sequences longest first (ties by index) up to 256 sequences, and by length
    class (floor(log2(KV tiles)), sequence order within a class) beyond: both sides of that
    edge, with runs of equal lengths and empty sequences, every output against the oracle
    (head dim 64 on the single-CTA kernel, 128 and 256 on the swapped one)."""
    rng = np.random.default_rng(800 + B)
    lens = rng.integers(0, max_len, size=B)
    lens[::7] = 129          # a run of ties across the batch
    lens[3::11] = 0
    db = decode_batch(801 + B, lens, 4 * Hkv, Hkv, D, 16, "f16")
    p, got = run_decode(db, splits=3)
    assert _binding().device_error(reset=True)[0] == 0
    empty = db.seq_lens == 0
    assert (got[empty] == 0).all()
    U.assert_close(got[~empty], oracle_decode(db)[~empty], f"B={B} (S={p.splits})")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_decode_graph_replay_follows_device_lengths():
    """pa_decode (+ pa_combine) captured once in a CUDA graph, then replayed while the lengths
    and the query tokens change in place on the device: a step that appends one token to every
    sequence, then lengths redrawn so that the longest-first order changes. Each replay equals
    the oracle at that step's lengths."""
    import dataclasses
    import torch
    from paged_kv_long_b200.inputs import to_bits
    bd = _binding()
    B, Hq, Hkv, D, PS, dt = 12, 16, 2, 128, 16, "bf16"
    rng = np.random.default_rng(91)
    lens0 = rng.integers(100, 3000, size=B)
    cap = lens0 + 600                                   # pages for the longest lengths below
    db = decode_batch(92, cap, Hq, Hkv, D, PS, dt)
    p = bd.decode_plan(Hq, Hkv, D, PS, B, int(cap.max()), dt)
    assert p.splits > 1                                 # the combine is in the graph too
    q = _dev(db.q, dt).clone()
    kp, vp = _dev(db.k_pool, dt), _dev(db.v_pool, dt)
    tab = torch.from_numpy(db.block_table).cuda()
    sl = torch.from_numpy(lens0.astype(np.int32)).cuda()
    out = torch.zeros((B, Hq, D), device="cuda")
    ws = bd.workspace(p)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bd.decode(p, q, kp, vp, tab, sl, out, ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        bd.decode(p, q, kp, vp, tab, sl, out, ws, stream=s)
    bd.device_error(reset=True)
    steps = [lens0, lens0 + 1, cap - rng.integers(0, 600, size=B)]
    for i, lens in enumerate(steps):
        q_bits = to_bits(rng.standard_normal((B, Hq, D), dtype=np.float32), dt)
        q.copy_(_dev(q_bits, dt))
        sl.copy_(torch.from_numpy(lens.astype(np.int32)))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert bd.device_error(reset=True)[0] == 0
        ref = oracle_decode(dataclasses.replace(db, q=q_bits, seq_lens=lens.astype(np.int32)))
        U.assert_close(out.cpu().numpy(), ref, f"graph replay {i} (S={p.splits})")
    del g


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("D", [64, 256])
def test_gpu_decode_length_past_table_is_reported(D):
    import torch
    bd = _binding()
    bd.device_error(reset=True)
    db = decode_batch(79, [40, 20], 4, 2, D, 16, "f16")
    lens = db.seq_lens.copy()
    lens[1] = db.block_table.shape[1] * 16 + 1  # more keys than the table row maps
    p = bd.decode_plan(4, 2, D, 16, 2, 64, "f16")
    bd.decode(p, _dev(db.q, "f16"), _dev(db.k_pool, "f16"), _dev(db.v_pool, "f16"),
              torch.from_numpy(db.block_table).cuda(), torch.from_numpy(lens).cuda())
    st, flags = bd.device_error(reset=True)
    assert bd.STATUS[st] == "PA_ERR_PAGE_INDEX" and flags & 1
