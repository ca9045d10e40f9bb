"""Batched prefill (pa_batch_plan, pa_batch_prefill, pa_batch_combine): several sequences, each a
chunk of q_lens[b] rows at its own history hist_lens[b], in one launch over one page pool.

Each sequence's attention is the single-piece definition on that sequence's keys, so the oracle
is oracle.attend per sequence. CPU tests pin that use to a brute-force softmax, check that the
planner's items cover every row block's KV tiles exactly once with consistent workspace slots,
and that the C ABI refuses mixed-up plans and arrays. GPU tests compare the kernels with the
oracle element by element, and a batch of one sequence with the single-piece launch bit for bit.
"""
import ctypes
import math
import zlib

import numpy as np
import pytest

from oracle import oracle
from paged_kv_long_b200.inputs import seq_batch
from tests.conftest import cuda_available
from tests import parity_util as U

TILE = 128


def seq_problem(sb, b: int) -> oracle.Problem:
    h, r = int(sb.hist_lens[b]), int(sb.q_lens[b])
    PS = sb.k_pool.shape[1]
    r0 = int(sb.q_row0[b])
    return oracle.Problem(q=sb.q[r0:r0 + r], k=sb.k_pool, v=sb.v_pool, hist_len=h,
                          dtype=sb.dtype, page_table=sb.block_table[b, :math.ceil((h + r) / PS)],
                          scale=sb.scale)


def oracle_batch(sb) -> np.ndarray:
    rows, Hq, D = sb.q.shape
    out = np.zeros((rows, Hq, D))
    for b in range(len(sb.q_lens)):
        r = int(sb.q_lens[b])
        if r:
            r0 = int(sb.q_row0[b])
            o, _ = oracle.attend(seq_problem(sb, b))
            out[r0:r0 + r] = o.reshape(r, Hq, D)
    return out


def brute_batch(sb) -> np.ndarray:
    """numpy fp64 softmax per (sequence, row, head) through the table (tiny cases only)."""
    rows, Hq, D = sb.q.shape
    PS, Hkv = sb.k_pool.shape[1], sb.k_pool.shape[2]
    G = Hq // Hkv
    scale = sb.scale or 1.0 / math.sqrt(D)
    out = np.zeros((rows, Hq, D))
    for b in range(len(sb.q_lens)):
        h, r, r0 = int(sb.hist_lens[b]), int(sb.q_lens[b]), int(sb.q_row0[b])
        pos = np.arange(h + r)
        phys = sb.block_table[b, pos // PS].astype(np.int64)
        k = oracle.decode(sb.dtype, sb.k_pool[phys, pos % PS])
        v = oracle.decode(sb.dtype, sb.v_pool[phys, pos % PS])
        for i in range(r):
            q = oracle.decode(sb.dtype, sb.q[r0 + i])
            for hq in range(Hq):
                s = k[:h + i + 1, hq // G] @ q[hq] * scale
                w = np.exp(s - s.max())
                out[r0 + i, hq] = (w / w.sum()) @ v[:h + i + 1, hq // G]
    return out


# ------------------------------------------------------------------------------ oracle pins


def test_oracle_batch_matches_brute_force():
    sb = seq_batch(21, [0, 37, 5, 16], [9, 1, 20, 3], Hq=4, Hkv=2, D=64, PS=16, dtype="f16")
    np.testing.assert_allclose(oracle_batch(sb), brute_batch(sb), rtol=1e-12, atol=1e-12)


def test_oracle_first_row_of_empty_history_is_its_value():
    """A chunk at history 0: its first row sees only its own key, so the output is that V."""
    sb = seq_batch(22, [0, 0], [4, 2], Hq=2, Hkv=1, D=64, PS=16, dtype="bf16")
    got = oracle_batch(sb)
    for b in range(2):
        v0 = oracle.decode("bf16", sb.v_pool[sb.block_table[b, 0], 0])  # [Hkv, D]
        np.testing.assert_array_equal(got[int(sb.q_row0[b])], np.repeat(v0, 2, axis=0))


# ------------------------------------------------------------------------------ planner / ABI


def _bd():
    from paged_kv_long_b200 import binding
    return binding


def row_block_tiles(q_lens, hist_lens, Hkv, G, per):
    """Expected KV-tile count of every global row block (independent restatement: the last
    token of a unit's last Q tile sees hist + token + 1 keys)."""
    out = []
    for r, h in zip(q_lens, hist_lens):
        q_tiles = math.ceil(r * G / TILE)
        q_units = math.ceil(q_tiles / per)
        for local in range(q_units * Hkv):
            qu = q_units - 1 - local // Hkv
            last_tile = min(qu * per + per - 1, q_tiles - 1)
            t_last = min((last_tile * TILE + TILE - 1) // G, r - 1)
            out.append(math.ceil((h + t_last + 1) / TILE))
    return out


def check_items(items, tiles, rows_per_block):
    covered = [np.zeros(n, dtype=np.int32) for n in tiles]
    parts = {}
    for rb, k0, k1, slot in items:
        assert 0 <= k0 < k1 <= tiles[rb]
        covered[rb][k0:k1] += 1
        parts.setdefault(rb, []).append(slot)
    for rb, c in enumerate(covered):
        assert (c == 1).all(), f"row block {rb} not covered exactly once"
    slots = []
    for rb, s in parts.items():
        if len(s) == 1:
            assert s[0] == -1
        else:
            assert -1 not in s
            slots += s
    assert sorted(slots) == list(range(len(slots)))


@pytest.mark.parametrize("seed", range(40))
def test_batch_schedule_covers_every_tile_once(seed):
    bd = _bd()
    rng = np.random.default_rng(seed)
    D = [64, 128, 256][seed % 3]
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    B = int(rng.integers(1, 24))
    q_lens = rng.integers(0, [700, 200, 40][seed % 3], size=B)
    q_lens[rng.integers(0, B)] = max(1, q_lens[0])
    if seed % 4 == 0:
        q_lens[:] = 1  # decode-like
    hist = rng.integers(0, 40000, size=B)
    num_sms = int(rng.choice([148, 132, 16, 7]))
    # CTA pairs at head dim 256 unless every sequence fits one Q tile
    per = 2 if D == 256 and max(math.ceil(r * G / TILE) for r in q_lens) > 1 else 1
    tiles = row_block_tiles(q_lens, hist, Hkv, G, per)
    try:
        bp = bd.batch_plan(G * Hkv, Hkv, D, 16, q_lens, hist, "bf16", num_sms=num_sms)
    except bd.PaError as e:
        # the item table holds 512 row blocks (whole, when cuts no longer fit)
        assert bd.STATUS[e.status] == "PA_ERR_UNSUPPORTED" and len(tiles) > 512
        return
    assert bp.plan.ctas_per_unit == per
    items = bd.batch_schedule_items(bp)
    assert len(items) == bp.plan.units
    check_items(items, tiles, per * TILE)
    assert bp.plan.chunk_rows == q_lens.sum() and bp.plan.batch == B
    n_slots = sum(1 for it in items if it[3] >= 0)
    assert bp.plan.ws_bytes == n_slots * per * TILE * (D + 1) * 4


def test_batch_pairs_only_when_a_sequence_has_two_q_tiles():
    bd = _bd()
    one = bd.batch_plan(16, 2, 256, 16, [1, 16, 3], [900, 20, 5000], "f16", num_sms=148)
    assert one.plan.ctas_per_unit == 1            # 16 rows x 8 heads = one 128-row tile
    two = bd.batch_plan(16, 2, 256, 16, [1, 17, 3], [900, 20, 5000], "f16", num_sms=148)
    assert two.plan.ctas_per_unit == 2
    small_d = bd.batch_plan(16, 2, 128, 16, [500, 17], [900, 20], "f16", num_sms=148)
    assert small_d.plan.ctas_per_unit == 1


def test_batch_of_many_row_blocks_keeps_them_whole():
    """256 one-row sequences x 2 KV heads = 512 row blocks: too many to add cuts, so every row
    block is one item, longest first."""
    bd = _bd()
    rng = np.random.default_rng(9)
    hist = rng.integers(0, 20000, size=256)
    bp = bd.batch_plan(16, 2, 128, 16, np.ones(256, dtype=np.int32), hist, "f16", num_sms=148)
    items = bd.batch_schedule_items(bp)
    assert len(items) == 512 and (items[:, 3] == -1).all() and bp.plan.ws_bytes == 0
    tiles = row_block_tiles(np.ones(256, dtype=int), hist, 2, 8, 1)
    check_items(items, tiles, TILE)
    lens = items[:, 2] - items[:, 1]
    assert (np.diff(lens) <= 0).all()
    with pytest.raises(bd.PaError):   # 257 sequences: more than the sequence table holds
        bd.batch_plan(16, 2, 128, 16, np.ones(257, dtype=np.int32), np.zeros(257), "f16",
                      num_sms=148)


def test_batch_schedule_balances_the_sms():
    """Many sequences of mixed length: no SM (pair) gets much more than the even share."""
    bd = _bd()
    rng = np.random.default_rng(5)
    q_lens = rng.integers(1, 200, size=24)
    hist = rng.integers(0, 30000, size=24)
    bp = bd.batch_plan(16, 2, 256, 16, q_lens, hist, "f16", num_sms=148)
    items = bd.batch_schedule_items(bp)
    tiles = row_block_tiles(q_lens, hist, 2, 8, 2)
    share = sum(tiles) / 74
    # simulate the first-free dispatch in launch order with the same per-item cost
    loads = np.zeros(74)
    for rb, k0, k1, _ in items:
        i = int(np.argmin(loads))
        loads[i] += (k1 - k0) + 5
    assert loads.max() <= 1.15 * share + 40


def test_batch_abi_refuses_mixed_up_plans_and_arrays():
    """All checked before any device work: runs without a GPU."""
    bd = _bd()
    lib = bd.load_library()
    fake = ctypes.c_void_p(1 << 20)
    bp = bd.batch_plan(16, 2, 256, 16, [100, 3], [500, 9000], "f16", num_sms=148)
    ql, hl = bp._arrays()
    st = lib.pa_prefill(ctypes.byref(bp.plan), fake, fake, fake, fake, 10, bp.plan.hist_len,
                        bp.plan.chunk_rows, fake, fake, 1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    st = lib.pa_combine(ctypes.byref(bp.plan), fake, 1 << 30, fake, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    other = np.array([100, 4], dtype=np.int32)   # not the arrays the plan was made from
    st = lib.pa_batch_prefill(ctypes.byref(bp.plan), other.ctypes.data, hl, fake, fake, fake,
                              fake, 64, 100, fake, fake, 1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    single = bd.plan(16, 2, 256, 16, 512, 4096, "f16", policy="balanced", num_sms=148)
    st = lib.pa_batch_prefill(ctypes.byref(single), ql, hl, fake, fake, fake, fake, 64, 100,
                              fake, fake, 1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    st = lib.pa_batch_prefill(ctypes.byref(bp.plan), ql, hl, fake, fake, fake, fake, 1, 100,
                              fake, fake, 1 << 30, None)   # table rows too short
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"
    one = bd.batch_plan(16, 2, 256, 16, [1], [50], "f16", num_sms=148)  # looks like decode
    st = lib.pa_decode(ctypes.byref(one.plan), fake, fake, fake, fake, 8, fake, 100, fake, fake,
                       1 << 30, None)
    assert bd.STATUS[st] == "PA_ERR_INVALID_ARG"


@pytest.mark.parametrize("q_lens,hist,err", [
    ([1] * 257, [0] * 257, "PA_ERR_UNSUPPORTED"),    # more sequences than the table holds
    ([0, 0], [5, 5], "PA_ERR_INVALID_ARG"),           # no rows at all
    ([3, -1], [5, 5], "PA_ERR_INVALID_ARG"),
    ([3, 1], [5, -2], "PA_ERR_INVALID_ARG"),
])
def test_batch_plan_rejects(q_lens, hist, err):
    bd = _bd()
    with pytest.raises(bd.PaError) as e:
        bd.batch_plan(8, 2, 128, 16, q_lens, hist, "f16", num_sms=148)
    assert bd.STATUS[e.value.status] == err


# ------------------------------------------------------------------------------ GPU parity

CASES = [
    # name, hist_lens, q_lens, Hq, Hkv, D, PS, dtype, num_sms (None: the device's)
    ("d256_mixed", [0, 3000, 17, 9000], [700, 129, 1, 300], 16, 2, 256, 16, "f16", None),
    ("d256_decode_like", [5, 4096, 130, 0, 20000], [1, 1, 1, 1, 1], 24, 4, 256, 64, "bf16", None),
    ("d256_cut_heavy", [12000, 8000], [256, 512], 16, 2, 256, 16, "bf16", 8),
    ("d256_g6", [1000, 70], [50, 200], 24, 4, 256, 64, "bf16", 6),
    ("d128_empty_seq", [100, 5, 2000], [64, 0, 333], 32, 8, 128, 32, "bf16", None),
    ("d128_cuts", [3000, 50, 7000], [128, 300, 40], 8, 1, 128, 16, "f16", 5),
    ("d64_g16", [0, 900], [300, 77], 32, 2, 64, 128, "f16", 4),
    # one-row batches on the swapped-operand decode kernel (G <= 8 at head dim 128 / 256): empty
    # sequences, one key, page and tile edges, and few SMs so that items are cut and merged
    ("d128_one_row_swapped", [0, 15, 16, 127, 128, 4000, 9000, 0], [1, 1, 1, 1, 1, 1, 1, 0],
     16, 4, 128, 16, "bf16", 12),
    ("d256_one_row_g1_swapped", [3000, 1, 511], [1, 1, 1], 2, 2, 256, 32, "f16", 4),
    ("d256_one_row_ps128_swapped", [10000, 300, 64], [1, 1, 1], 16, 2, 256, 128, "bf16", 8),
]


def _dev(bits, dtype):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def run_batch(sb, num_sms=None):
    import torch
    bd = _bd()
    rows, Hq, D = sb.q.shape
    Hkv, PS = sb.k_pool.shape[2], sb.k_pool.shape[1]
    bp = bd.batch_plan(Hq, Hkv, D, PS, sb.q_lens, sb.hist_lens, sb.dtype, sb.scale,
                       num_sms=num_sms)
    out = torch.full((rows, Hq, D), float("nan"), device="cuda")  # every entry must be written
    ws = bd.workspace(bp.plan)
    if ws is not None:
        ws.fill_(float("nan"))
    out = bd.batch_prefill(bp, _dev(sb.q, sb.dtype), _dev(sb.k_pool, sb.dtype),
                           _dev(sb.v_pool, sb.dtype), torch.from_numpy(sb.block_table).cuda(),
                           out, ws)
    torch.cuda.synchronize()
    return bp, out.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_batch_matches_oracle(case):
    from paged_kv_long_b200.build import build
    build()
    bd = _bd()
    bd.device_error(reset=True)
    name, hist, q_lens, Hq, Hkv, D, PS, dtype, num_sms = case
    sb = seq_batch(zlib.crc32(name.encode()) & 0xFFFF, hist, q_lens, Hq, Hkv, D, PS, dtype)
    bp, got = run_batch(sb, num_sms)
    assert bd.device_error(reset=True)[0] == 0
    U.assert_close(got, oracle_batch(sb), f"{name} (items={bp.plan.units}, "
                                          f"max parts={bp.plan.splits})")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_batch_of_256_sequences_matches_oracle():
    """The largest batch: 256 sequences (one-row chunks and short chunks), 512 row blocks."""
    bd = _bd()
    rng = np.random.default_rng(51)
    hist = rng.integers(0, 3000, size=256)
    q_lens = np.where(np.arange(256) % 5 == 0, rng.integers(2, 16, size=256), 1)
    sb = seq_batch(52, hist, q_lens, 16, 2, 128, 16, "bf16")
    bp, got = run_batch(sb)
    assert bp.plan.batch == 256 and bd.device_error(reset=True)[0] == 0
    U.assert_close(got, oracle_batch(sb), f"256 sequences (items={bp.plan.units})")


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("D,num_sms", [(256, 148), (256, 10), (128, 9)])
def test_gpu_batch_of_one_equals_single_piece(D, num_sms):
    """One sequence: the same schedule as the balanced single-piece plan, the same bits."""
    import torch
    bd = _bd()
    h, r, Hq, Hkv, PS = 2500, 600, 16, 2, 16
    sb = seq_batch(31, [h], [r], Hq, Hkv, D, PS, "bf16")
    bp, got = run_batch(sb, num_sms)
    p = bd.plan(Hq, Hkv, D, PS, r, h, "bf16", policy="balanced", num_sms=num_sms)
    assert p.units == bp.plan.units and p.ws_bytes == bp.plan.ws_bytes
    tab = torch.from_numpy(np.ascontiguousarray(sb.block_table[0])).cuda()
    single = bd.prefill_combine(p, _dev(sb.q, "bf16"), _dev(sb.k_pool, "bf16"),
                                _dev(sb.v_pool, "bf16"), tab)
    torch.cuda.synchronize()
    assert np.array_equal(single.cpu().numpy(), got)


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_batched_decode_matches_uniform_decode_and_oracle():
    """Decode as a batch of one-row chunks (host lengths, balanced) against pa_decode (device
    lengths, uniform splits) and the oracle."""
    import torch
    bd = _bd()
    rng = np.random.default_rng(41)
    lens = rng.integers(1, 20000, size=24)
    sb = seq_batch(42, lens - 1, np.ones(24, dtype=np.int32), 16, 2, 256, 16, "f16")
    bp, got = run_batch(sb)
    ref = oracle_batch(sb)
    U.assert_close(got, ref, "batched decode")
    p = bd.decode_plan(16, 2, 256, 16, 24, int(lens.max()), "f16")
    dec = bd.decode(p, _dev(sb.q, "f16"), _dev(sb.k_pool, "f16"), _dev(sb.v_pool, "f16"),
                    torch.from_numpy(sb.block_table).cuda(),
                    torch.from_numpy(lens.astype(np.int32)).cuda())
    torch.cuda.synchronize()
    U.assert_close(dec.cpu().numpy(), ref, "uniform decode")
    assert bd.device_error(reset=True)[0] == 0


def test_one_row_batches_plan_two_cta_slots_per_sm():
    """One-row batches with G <= 8 at head dim 128 / 256 run the swapped-operand decode kernel,
    two CTAs per SM: their items are cut for 2 x num_sms workers (each worker's share ends at a
    cut, so there are at least that many items); other batches keep one worker per SM."""
    bd = _bd()
    B, hist = 32, np.full(32, 20000)
    ones = np.ones(B, dtype=np.int32)
    for D in (128, 256):
        bp = bd.batch_plan(16, 2, D, 16, ones, hist, "bf16", num_sms=148)
        assert bp.plan.ctas_per_unit == 1 and bp.plan.units >= 2 * 148
    for Hq, D, q_lens in ((32, 256, ones), (16, 64, ones), (16, 256, 2 * ones)):
        bp = bd.batch_plan(Hq, 2, D, 16, q_lens, hist, "bf16", num_sms=148)
        assert bp.plan.units < 2 * 148
