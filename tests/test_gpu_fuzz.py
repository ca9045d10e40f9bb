"""Seeded GPU fuzz: random shapes through every launch path, each checked against the oracle on
sampled (row, head) pairs (first and last rows, Q-tile edges, random rest) with NaN-filled pools
beyond the keys, workspaces and outputs, so a wrong key, a missed write or a stale partial fails.

Single pieces: head dim, GQA group, page size, dtype, history (0 .. 40K, often off a page or
tile edge), chunk rows (1 .. 1,500), policy (planner, balanced, forced splits 1 .. 32), paged
or contiguous K/V.
Batches: 1 .. 12 sequences of random histories and rows, one-row (decode) batches included.
Decode (pa_decode, device-side lengths): 1 .. 40 sequences of 0 .. 20,000 keys, split counts
from the planner or forced (1 .. 32).
"""
import math

import numpy as np
import pytest

from oracle import oracle
from tests.conftest import cuda_available
from tests import parity_util as U

N_PIECE = 48
N_BATCH = 20
N_DECODE = 12


def piece_case(seed):
    rng = np.random.default_rng(1000 + seed)
    D = int(rng.choice([64, 128, 256, 256]))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 3, 4, 6, 8, 16]))
    PS = int(rng.choice([16, 32, 64, 128]))
    dtype = str(rng.choice(["f16", "bf16"]))
    H = int(rng.choice([0, int(rng.integers(1, 600)), int(rng.integers(600, 40000))]))
    R = int(rng.choice([1, int(rng.integers(2, 130)), int(rng.integers(130, 1500))]))
    mode = str(rng.choice(["planner", "balanced", "forced"]))
    S = int(rng.choice([1, 2, 3, 5, 8, 17, 32])) if mode == "forced" else None
    num_sms = int(rng.choice([148, 148, 37, 9]))
    paged = bool(seed % 5 != 4)  # every fifth piece reads contiguous K/V
    return D, Hkv, G, PS, dtype, H, R, mode, S, num_sms, paged


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("seed", range(N_PIECE))
def test_gpu_fuzz_piece(seed):
    from paged_kv_long_b200 import binding
    D, Hkv, G, PS, dtype, H, R, mode, S, num_sms, paged = piece_case(seed)
    name = (f"fuzz{seed}: D{D} Hkv{Hkv} G{G} PS{PS} {dtype} H{H} R{R} {mode} S={S} "
            f"sms{num_sms} {'paged' if paged else 'contiguous'}")
    wl = U.custom_workload(name, Hkv * G, Hkv, D, PS, dtype, [(H, R)], seed=20000 + 10 * seed,
                           splits=S or 0)
    inp = U.gen(wl, poison=True)
    binding.device_error(reset=True)
    policy = "balanced" if mode == "balanced" else "makespan"
    dw, outs = U.run_gpu(inp, paged=paged, splits=S if S else 0, policy=policy,
                         num_sms=num_sms)
    assert binding.device_error(reset=True)[0] == 0, name
    U.check_sampled(inp, outs, n=40, paged=paged, what=name)


def batch_case(seed):
    rng = np.random.default_rng(5000 + seed)
    D = int(rng.choice([64, 128, 256]))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 4, 6, 8]))
    PS = int(rng.choice([16, 64]))
    dtype = str(rng.choice(["f16", "bf16"]))
    B = int(rng.integers(1, 13))
    hist = rng.integers(0, 20000, size=B)
    if seed % 3 == 0:
        rows = np.ones(B, dtype=np.int64)          # a decode step
    else:
        rows = rng.integers(0, 700, size=B)
        rows[0] = max(rows[0], 1)
    num_sms = int(rng.choice([148, 23]))
    return D, Hkv, G, PS, dtype, hist, rows, num_sms


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("seed", range(N_BATCH))
def test_gpu_fuzz_batch(seed):
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.inputs import seq_batch
    D, Hkv, G, PS, dtype, hist, rows, num_sms = batch_case(seed)
    Hq = Hkv * G
    name = f"batch fuzz{seed}: D{D} Hkv{Hkv} G{G} PS{PS} {dtype} B{len(rows)} sms{num_sms}"
    sb = seq_batch(30000 + seed, hist, rows, Hq, Hkv, D, PS, dtype)
    try:
        bp = binding.batch_plan(Hq, Hkv, D, PS, sb.q_lens, sb.hist_lens, dtype, num_sms=num_sms)
    except binding.PaError as e:
        assert binding.STATUS[e.status] == "PA_ERR_UNSUPPORTED", name
        pytest.skip(f"{name}: more row blocks than the item table holds")
    binding.device_error(reset=True)

    def dev(bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
        return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)

    out = torch.full((int(sb.q_lens.sum()), Hq, D), float("nan"), device="cuda")
    ws = binding.workspace(bp.plan)
    if ws is not None:
        ws.fill_(float("nan"))
    binding.batch_prefill(bp, dev(sb.q), dev(sb.k_pool), dev(sb.v_pool),
                          torch.from_numpy(sb.block_table).cuda(), out, ws)
    torch.cuda.synchronize()
    assert binding.device_error(reset=True)[0] == 0, name
    got = out.cpu().numpy()
    r0s = sb.q_row0
    for b in range(len(rows)):
        r = int(sb.q_lens[b])
        if r == 0:
            continue
        h = int(sb.hist_lens[b])
        pb = oracle.Problem(q=sb.q[r0s[b]:r0s[b] + r], k=sb.k_pool, v=sb.v_pool, hist_len=h,
                            dtype=dtype, page_table=sb.block_table[b, :math.ceil((h + r) / PS)])
        sel_r, sel_h = U.sample_pairs(r, Hq, 12, 40000 + seed * 64 + b, G)
        ref, _ = oracle.attend(pb, sel_r, sel_h)
        U.assert_close(got[r0s[b] + sel_r, sel_h], ref, f"{name} sequence {b} (H={h}, R={r})")


def decode_case(seed):
    rng = np.random.default_rng(9000 + seed)
    D = int(rng.choice([64, 128, 256]))
    Hkv = int(rng.choice([1, 2, 8]))
    G = int(rng.choice([1, 4, 8, 16]))
    PS = int(rng.choice([16, 32, 128]))
    dtype = str(rng.choice(["f16", "bf16"]))
    B = int(rng.integers(1, 41))
    lens = rng.integers(0, 20000, size=B)
    lens[rng.integers(0, B)] = int(rng.choice([0, 1, 128, 129]))
    S = int(rng.choice([0, 0, 1, 7, 19, 32]))
    return D, Hkv, G, PS, dtype, lens, S


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("seed", range(N_DECODE))
def test_gpu_fuzz_decode(seed):
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.inputs import decode_batch
    D, Hkv, G, PS, dtype, lens, S = decode_case(seed)
    Hq = Hkv * G
    name = f"decode fuzz{seed}: D{D} Hkv{Hkv} G{G} PS{PS} {dtype} B{len(lens)} S={S}"
    db = decode_batch(50000 + seed, lens, Hq, Hkv, D, PS, dtype)
    p = binding.decode_plan(Hq, Hkv, D, PS, len(lens), max(1, int(lens.max())), dtype, splits=S)
    binding.device_error(reset=True)

    def dev(bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
        return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)

    out = torch.full((len(lens), Hq, D), float("nan"), device="cuda")
    ws = binding.workspace(p)
    if ws is not None:
        ws.fill_(float("nan"))
    binding.decode(p, dev(db.q), dev(db.k_pool), dev(db.v_pool),
                   torch.from_numpy(db.block_table).cuda(), torch.from_numpy(db.seq_lens).cuda(),
                   out, ws)
    torch.cuda.synchronize()
    assert binding.device_error(reset=True)[0] == 0, name
    got = out.cpu().numpy()
    heads = np.random.default_rng(seed).integers(0, Hq, size=len(lens)).astype(np.int32)
    for b, n in enumerate(lens):
        n = int(n)
        if n == 0:
            assert (got[b] == 0).all(), f"{name}: sequence {b} has no key, output must be 0"
            continue
        pb = oracle.Problem(q=db.q[b:b + 1], k=db.k_pool, v=db.v_pool, hist_len=n - 1,
                            dtype=dtype, page_table=db.block_table[b, :math.ceil(n / PS)])
        hs = np.array([0, Hq - 1, heads[b]], dtype=np.int32)
        ref, _ = oracle.attend(pb, np.zeros(3, dtype=np.int64), hs)
        U.assert_close(got[b, hs], ref, f"{name} sequence {b} ({n} keys)")


N_APPEND = 8


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("seed", range(N_APPEND))
def test_gpu_fuzz_kv_append(seed):
    """pa_kv_append on random shapes and positions, bit for bit against the append oracle."""
    import torch
    from oracle.kv_append import kv_append as oracle_append
    from paged_kv_long_b200 import binding
    rng = np.random.default_rng(60000 + seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    D = int(rng.choice([64, 128, 256]))
    PS = int(rng.choice([16, 32, 64, 128]))
    H = int(rng.choice([0, int(rng.integers(1, 5000))]))
    R = int(rng.choice([1, int(rng.integers(2, 3000))]))
    pages = math.ceil((H + R) / PS)
    num_pages = pages + int(rng.integers(0, 9))
    pool = rng.integers(0, 1 << 16, size=(num_pages, PS, Hkv, D), dtype=np.uint16)
    new = rng.integers(0, 1 << 16, size=(R, Hkv, D), dtype=np.uint16)
    table = rng.permutation(num_pages)[:pages].astype(np.int32)
    want, bad = oracle_append(pool, new, table, H)
    assert bad == 0

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(
            torch.bfloat16)

    kp, vp = dev(pool), dev(pool.copy())
    binding.device_error(reset=True)
    binding.kv_append(dev(new), dev(new), kp, vp, torch.from_numpy(table).cuda(), H)
    torch.cuda.synchronize()
    assert binding.device_error(reset=True)[0] == 0
    for t in (kp, vp):
        assert np.array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16), want)
