"""Seeded GPU fuzz: random shapes through every launch path, each checked against the oracle on
sampled (row, head) pairs (first and last rows, Q-tile edges, random rest) with NaN-filled pools
beyond the keys, workspaces and outputs, so a wrong key, a missed write or a stale partial fails.

Single pieces: head dim, GQA group, page size, dtype, history (0 .. 40K, often off a page or
tile edge), chunk rows (1 .. 1,500), policy (planner, balanced, forced splits 1 .. 32).
Batches: 1 .. 12 sequences of random histories and rows, one-row (decode) batches included.
"""
import math

import numpy as np
import pytest

from oracle import oracle
from tests.conftest import cuda_available
from tests import parity_util as U

N_PIECE = 24
N_BATCH = 10


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
    return D, Hkv, G, PS, dtype, H, R, mode, S, num_sms


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("seed", range(N_PIECE))
def test_gpu_fuzz_piece(seed):
    from paged_kv_long_b200 import binding
    D, Hkv, G, PS, dtype, H, R, mode, S, num_sms = piece_case(seed)
    name = f"fuzz{seed}: D{D} Hkv{Hkv} G{G} PS{PS} {dtype} H{H} R{R} {mode} S={S} sms{num_sms}"
    wl = U.custom_workload(name, Hkv * G, Hkv, D, PS, dtype, [(H, R)], seed=20000 + 10 * seed,
                           splits=S or 0)
    inp = U.gen(wl, poison=True)
    binding.device_error(reset=True)
    policy = "balanced" if mode == "balanced" else "makespan"
    dw, outs = U.run_gpu(inp, splits=S if S else 0, policy=policy, num_sms=num_sms)
    assert binding.device_error(reset=True)[0] == 0, name
    U.check_sampled(inp, outs, n=40, what=name)


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
