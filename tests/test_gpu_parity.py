"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element (several Q tiles, ragged tails, every split
count family); the five workloads at full size are compared on seeded samples of outputs
the oracle computes one by one. Tolerance: max-abs <= 1e-2 and relative RMS <= 2e-3.
"""
import numpy as np
import pytest

from paged_kv_long_b200 import binding
from tests import parity_util as U
from tests.conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def built():
    from oracle import oracle
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.build import build
    oracle.build()
    build()
    binding.load_library()
    binding.device_error(reset=True)
    yield
    st, flags = binding.device_error(reset=True)
    assert st == 0, f"device error flags {flags} left set"


# ------------------------------------------------------------------ small, element by element
def test_c1_tiny_full():
    inp = U.gen("c1")
    _, outs = U.run_gpu(inp)
    U.check_full(inp, outs, what="c1 paged")
    _, outc = U.run_gpu(inp, paged=False)
    U.check_full(inp, outc, paged=False, what="c1 contiguous")
    assert np.array_equal(outs[0], outc[0])


def test_c2_short_full_paged_and_contiguous():
    inp = U.gen("c2")
    _, outs = U.run_gpu(inp)
    U.check_full(inp, outs, what="c2 paged")
    _, outc = U.run_gpu(inp, paged=False)
    assert np.array_equal(outs[0], outc[0]), "paged and contiguous must agree bit for bit"


RAGGED = [
    # Hq, Hkv, D, PS, dtype, pieces, splits
    (24, 4, 256, 64, "bf16", [(333, 200)], 1),
    (24, 4, 256, 64, "bf16", [(333, 200)], 3),
    (24, 4, 256, 64, "bf16", [(1000, 77), (1077, 50)], 7),
    (16, 2, 256, 16, "f16", [(0, 300), (300, 213)], 0),
    (6, 2, 128, 32, "f16", [(517, 131)], 2),
    (8, 8, 128, 128, "bf16", [(45, 260)], 1),
    (4, 1, 64, 16, "bf16", [(1500, 99)], 5),
    (12, 3, 64, 64, "f16", [(0, 1)], 1),
    (24, 4, 256, 64, "bf16", [(4000, 1)], 32),
    (16, 2, 256, 16, "f16", [(10, 16)], 8),      # more splits than KV tiles: empty splits
    # head dim 64 merges more than 16 splits: lanes 16-31 own no columns but hold weights
    (8, 1, 64, 128, "bf16", [(0, 1)], 32),
    (8, 2, 64, 16, "bf16", [(0, 369)], 17),
]


@pytest.mark.parametrize("idx", range(len(RAGGED)), ids=[f"r{i}" for i in range(len(RAGGED))])
def test_ragged_full(idx):
    case = RAGGED[idx]
    Hq, Hkv, D, PS, dt, pieces, S = case
    wl = U.custom_workload("ragged", Hq, Hkv, D, PS, dt, pieces, seed=600 + 10 * idx, splits=S)
    inp = U.gen(wl)
    _, outs = U.run_gpu(inp)
    U.check_full(inp, outs, what=str(case))
    _, outc = U.run_gpu(inp, paged=False)
    for a, b in zip(outs, outc):
        assert np.array_equal(a, b)


MULTI_TILE = [
    # a single unit spanning 2-3 KV tiles, and many units with 1-2 KV tiles (head dim 256)
    (8, 1, 256, 16, "f16", [(200, 16)], 1),
    (8, 1, 256, 16, "f16", [(300, 16)], 1),
    (8, 1, 256, 64, "bf16", [(0, 256)], 1),
    (8, 1, 256, 128, "f16", [(0, 256)], 1),
]


@pytest.mark.parametrize("idx", range(len(MULTI_TILE)), ids=[f"m{i}" for i in range(len(MULTI_TILE))])
def test_units_spanning_several_kv_tiles(idx):
    """Every PV group must be complete before O is rescaled or read (the softmax tracks the
    PV completions one by one); a unit with several KV tiles exercises that ordering."""
    Hq, Hkv, D, PS, dt, pieces, S = MULTI_TILE[idx]
    wl = U.custom_workload("multi", Hq, Hkv, D, PS, dt, pieces, seed=900 + idx, splits=S)
    inp = U.gen(wl)
    for paged in (True, False):
        _, outs = U.run_gpu(inp, paged=paged)
        U.check_full(inp, outs, paged=paged, what=f"{MULTI_TILE[idx]} paged={paged}")


BALANCED = [
    # Hq, Hkv, D, PS, dtype, pieces, num_sms: few SMs, so that row blocks are cut into parts
    (24, 4, 256, 64, "bf16", [(3000, 100), (3100, 77)], 16),
    (16, 2, 256, 16, "f16", [(5000, 40)], 6),
    (16, 2, 256, 16, "f16", [(20000, 16)], 8),
    (6, 2, 128, 32, "f16", [(1500, 131)], 6),
    (4, 1, 64, 16, "bf16", [(2500, 99)], 3),
    (4, 1, 64, 16, "f16", [(9000, 30)], 4),
    # one long row block over 148 SMs at head dim 64: more than 16 parts to merge
    (4, 1, 64, 16, "f16", [(30000, 20)], 148),
]


@pytest.mark.parametrize("idx", range(len(BALANCED)), ids=[f"b{i}" for i in range(len(BALANCED))])
def test_balanced_schedule_full(idx):
    """Work items that cut row blocks at arbitrary KV tiles (the balanced policy), merged by
    the combine of cut row blocks; uncut row blocks write the output directly."""
    Hq, Hkv, D, PS, dt, pieces, sms = BALANCED[idx]
    wl = U.custom_workload("balanced", Hq, Hkv, D, PS, dt, pieces, seed=1300 + 10 * idx)
    inp = U.gen(wl)
    dw, outs = U.run_gpu(inp, policy="balanced", num_sms=sms)
    assert all(p.policy == binding.PA_POLICY_BALANCED for p in dw.plans)
    assert any((binding.schedule_items(p)[:, 3] >= 0).any() for p in dw.plans)
    U.check_full(inp, outs, what=f"{BALANCED[idx]}")
    _, outc = U.run_gpu(inp, paged=False, policy="balanced", num_sms=sms)
    for a, b in zip(outs, outc):
        assert np.array_equal(a, b)


def test_online_rescale_with_growing_scores():
    wl = U.custom_workload("ramp", 16, 4, 256, 16, "bf16", [(1200, 160)], seed=77, splits=2)
    inp = U.gen(wl, distribution="ramp")
    _, outs = U.run_gpu(inp)
    U.check_full(inp, outs, what="ramp")


def test_explicit_scale():
    wl = U.custom_workload("scale", 8, 2, 128, 32, "f16", [(300, 64)], seed=5, scale=0.03)
    inp = U.gen(wl)
    _, outs = U.run_gpu(inp)
    U.check_full(inp, outs, what="scale 0.03")


# ------------------------------------------------------------------ invariants on the GPU
def test_split_invariance_matches_pages_agreement():
    """S=1 vs S=8 on one layer: the pages report max |d| 2^-10 (one bf16 step) for their
    bf16-output kernel (splash PR #33, "Testing"). Our output is fp32, so the two runs differ
    by the bf16 rounding of P under different running maxima (relative ~1e-3), well inside
    that max bound; mean and cosine are reported, not compared (theirs round the output)."""
    wl = U.custom_workload("split", 24, 4, 256, 64, "bf16", [(8192, 256)], seed=9)
    inp = U.gen(wl)
    _, o1 = U.run_gpu(inp, splits=1)
    _, o8 = U.run_gpu(inp, splits=8)
    d = np.abs(o1[0].astype(np.float64) - o8[0])
    a, b = o1[0].ravel().astype(np.float64), o8[0].ravel().astype(np.float64)
    cos = a @ b / np.linalg.norm(a) / np.linalg.norm(b)
    print(f"S=1 vs S=8: max|d|={d.max():.3e} mean|d|={d.mean():.3e} cosine={cos:.9f}")
    assert d.max() <= 2.0 ** -10 and cos >= 0.99999
    U.check_sampled(inp, o8, n=64, what="split 8")


def test_page_shuffle_and_determinism():
    wl = U.custom_workload("shuffle", 16, 2, 256, 16, "f16", [(700, 300)], seed=11, splits=3)
    inp = U.gen(wl)
    _, a = U.run_gpu(inp)
    _, a2 = U.run_gpu(inp)
    assert np.array_equal(a[0], a2[0]), "same inputs must give the same bits"
    rng = np.random.default_rng(3)
    perm = rng.permutation(inp.k_pool.shape[0])
    k2, v2 = np.empty_like(inp.k_pool), np.empty_like(inp.v_pool)
    k2[perm], v2[perm] = inp.k_pool, inp.v_pool
    inp.k_pool, inp.v_pool = k2, v2
    inp.page_table = perm[inp.page_table].astype(np.int32)
    _, b = U.run_gpu(inp)
    assert np.array_equal(a[0], b[0]), "shuffling physical pages must not change a bit"


def test_bad_page_entry_is_reported_not_faulted():
    from paged_kv_long_b200 import binding
    wl = U.custom_workload("badpage", 8, 2, 128, 16, "f16", [(100, 40)], seed=13)
    inp = U.gen(wl)
    inp.page_table[2] = inp.k_pool.shape[0] + 5      # past the pool: reads zeros
    inp.page_table[3] = -7
    U.run_gpu(inp)
    st, flags = binding.device_error(reset=True)
    assert binding.STATUS[st] == "PA_ERR_PAGE_INDEX" and flags & 1


def test_wait_timeout_returns_status():
    from paged_kv_long_b200 import binding
    binding.selftest_timeout(2_000_000)  # 2 ms
    st, flags = binding.device_error(reset=True)
    assert binding.STATUS[st] == "PA_ERR_TIMEOUT" and flags & 2


def test_argument_errors():
    import torch
    from paged_kv_long_b200 import binding
    p = binding.plan(8, 2, 128, 16, 64, 100, "f16", splits=2)
    q = torch.zeros((64, 8, 128), dtype=torch.float16, device="cuda")
    pool = torch.zeros((20, 16, 2, 128), dtype=torch.float16, device="cuda")
    tab = torch.arange(11, dtype=torch.int32, device="cuda")
    out = torch.empty((64, 8, 128), dtype=torch.float32, device="cuda")
    small_ws = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.PaError) as e:
        binding.prefill(p, q, pool, pool, tab, out, small_ws)
    assert binding.STATUS[e.value.status] == "PA_ERR_WORKSPACE"
    lib = binding.load_library()
    import ctypes
    st = lib.pa_prefill(ctypes.byref(p), q.data_ptr() + 2, pool.data_ptr(), pool.data_ptr(),
                        tab.data_ptr(), 20, 100, 64, out.data_ptr(), None, 0, None)
    assert binding.STATUS[st] == "PA_ERR_INVALID_ARG"   # misaligned q
    st = lib.pa_prefill(ctypes.byref(p), q.data_ptr(), pool.data_ptr(), pool.data_ptr(),
                        tab.data_ptr(), 20, 101, 64, out.data_ptr(), None, 0, None)
    assert binding.STATUS[st] == "PA_ERR_INVALID_ARG"   # hist_len differs from the plan


# ------------------------------------------------------------------ the five workloads, full size
# Dense at full size: c4's 3,072 outputs all, under 16 splits (the workload's), 1 split and the
# planner's items; the last piece of c3 and the last chunk of c5 on every 8th row, all heads;
# the other pieces of c3 on seeded samples and the other chunks of c5 on every 64th row, all
# heads. Relative RMS is taken over each compared set.
def test_c3_full_size_dense_last_piece():
    inp = U.gen("c3")
    _, outs = U.run_gpu(inp)                 # 4 splits per piece, as the workload states
    _, outp = U.run_gpu(inp, splits=0)      # the planner's split count (balanced items)
    last = len(inp.wl.pieces) - 1
    ref, pairs = U.oracle_rows(inp, last, np.arange(0, inp.wl.pieces[last][1], 8))
    U.check_rows(outs[last], ref, pairs, "c3 S=4 last piece, every 8th row")
    U.check_rows(outp[last], ref, pairs, "c3 planned last piece, every 8th row")
    for i in range(last):
        rows, heads = U.sample_pairs(inp.wl.pieces[i][1], inp.wl.n_q_heads, 48, 7919 + i, 6)
        ref_i, _ = U.oracle.attend(U.oracle_problem(inp, i), rows, heads)
        U.assert_close(outs[i][rows, heads], ref_i, f"c3 S=4 piece {i} sampled")
        U.assert_close(outp[i][rows, heads], ref_i, f"c3 planned piece {i} sampled")
    _, outc = U.run_gpu(inp, paged=False)
    for a, b in zip(outs, outc):
        assert np.array_equal(a, b)


def test_c4_full_size_every_output():
    inp = U.gen("c4")
    ref, pairs = U.oracle_rows(inp, 0, np.arange(inp.wl.pieces[0][1]))   # 128 rows x 24 heads
    _, o16 = U.run_gpu(inp)                  # 16 splits + combine
    U.check_rows(o16[0], ref, pairs, "c4 S=16, every output")
    _, o1 = U.run_gpu(inp, splits=1)
    U.check_rows(o1[0], ref, pairs, "c4 S=1, every output")
    dw, op = U.run_gpu(inp, splits=0)        # the planner's choice (uniform or balanced)
    U.check_rows(op[0], ref, pairs, f"c4 planned (policy {dw.plans[0].policy}, "
                                    f"{dw.plans[0].units} units), every output")
    assert np.abs(o1[0].astype(np.float64) - o16[0]).max() <= 2.0 ** -10
    _, oc = U.run_gpu(inp, paged=False)
    assert np.array_equal(o16[0], oc[0])


def test_c5_full_size_dense_paged_equals_contiguous():
    inp = U.gen("c5")
    _, outs = U.run_gpu(inp)                 # planner's split count per chunk
    n = len(inp.wl.pieces)
    for i, (h, r) in enumerate(inp.wl.pieces):
        step = 8 if i == n - 1 else 64
        ref, pairs = U.oracle_rows(inp, i, np.arange(i % step, r, step))
        U.check_rows(outs[i], ref, pairs, f"c5 chunk {i} (H={h}), every {step}th row")
    _, outc = U.run_gpu(inp, paged=False)
    for a, b in zip(outs, outc):
        assert np.array_equal(a, b)


# ------------------------------------------------------------------ beyond the five workloads
@pytest.mark.parametrize("case", [
    # name, Hq, Hkv, D, PS, dtype, (H, R): histories of 2^20 and 2^22 keys plus a ragged tail,
    # 8,000-33,000 KV tiles per row block and 5.2 M pool rows (the largest coordinates here)
    ("million_d256", 8, 1, 256, 128, "bf16", (1_048_576 + 77, 200)),
    ("four_million_d64", 4, 1, 64, 64, "f16", (4_194_304 + 1_000, 130)),
], ids=lambda c: c[0])
def test_longest_histories_sampled(case):
    name, Hq, Hkv, D, PS, dt, piece = case
    wl = U.custom_workload(name, Hq, Hkv, D, PS, dt, [piece], seed=4242)
    inp = U.gen(wl)
    _, o_plan = U.run_gpu(inp)                          # the planner (balanced items)
    U.check_sampled(inp, o_plan, n=24, what=f"{name} planned")
    _, o_32 = U.run_gpu(inp, splits=32)                 # the most uniform splits
    U.check_sampled(inp, o_32, n=12, what=f"{name} S=32")
    assert np.abs(o_plan[0].astype(np.float64) - o_32[0]).max() <= 2.0 ** -10


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
def test_gpu_streamed_step_equals_the_plain_step():
    """DeviceWorkload.run_streamed (copies overlapped with compute on three streams, pinned host
    buffers in and out) gives the plain run's outputs bit for bit, two steps back to back."""
    import numpy as np
    import torch
    wl = U.custom_workload("streamed", 16, 2, 256, 16, "f16", [(0, 700), (700, 900), (1600, 513)],
                           seed=8800)
    inp = U.gen(wl, poison=True)
    dw, want = U.run_gpu(inp)

    def pinned(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dt is not None:
            t = t.view(torch.int16).view(dt)
        return t.pin_memory()

    hq = pinned(inp.q.view(np.int16), torch.float16)
    hk = pinned(inp.k_pool.view(np.int16), torch.float16)
    hv = pinned(inp.v_pool.view(np.int16), torch.float16)
    ht = pinned(inp.page_table)
    for o in dw.outs:
        o.fill_(float("nan"))
    houts = [torch.full(tuple(o.shape), float("nan")).pin_memory() for o in dw.outs]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    dw.run_streamed(hq, hk, hv, ht, houts, s_in, s_c, s_out)
    done = dw.run_streamed(hq, hk, hv, ht, houts, s_in, s_c, s_out)
    done.synchronize()
    torch.cuda.synchronize()
    for i, (h, w) in enumerate(zip(houts, want)):
        assert np.array_equal(h.numpy(), w), f"piece {i}"


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("policy", ["makespan", "balanced"])
def test_gpu_graph_replay_equals_eager(policy):
    """A step captured as a CUDA graph (DeviceWorkload.capture) and replayed twice gives the
    eager step's outputs bit for bit: the launches carry their plans by value."""
    import numpy as np
    import torch
    wl = U.custom_workload("graph", 24, 4, 256, 64, "bf16", [(3000, 512), (3512, 300)],
                           seed=9100)
    inp = U.gen(wl, poison=True)
    dw, want = U.run_gpu(inp, policy=policy)
    graph = dw.capture()
    for _ in range(2):
        for o in dw.outs:
            o.fill_(float("nan"))
        dw.ws.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        for i, (o, w) in enumerate(zip(dw.outs, want)):
            assert np.array_equal(o.cpu().numpy(), w), f"piece {i}"
    assert binding.device_error(reset=True)[0] == 0
