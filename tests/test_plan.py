"""Host logic of the C ABI (pa_plan and the split policies). CPU only: no CUDA calls."""
import math
import os

import pytest

from paged_kv_long_b200 import binding
from paged_kv_long_b200.inputs import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cores_policy_splits.txt")


def golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.fixture(scope="module")
def lib():
    from paged_kv_long_b200.build import build
    build()
    return binding.load_library()


@pytest.mark.parametrize("cores", [32, 38])
def test_cores_policy_matches_pages_table(lib, cores):
    for rows, tiles, before, now in golden_rows():
        assert lib.pa_cores_policy_splits(cores, 4, tiles) == now
        assert lib.pa_legacy_policy_splits(4, tiles) == before


def test_cores_policy_16_cores_is_half(lib):
    for rows, tiles, before, now in golden_rows():
        assert lib.pa_cores_policy_splits(16, 4, tiles) == max(1, now // 2)


@pytest.mark.parametrize("cores,kv", [(76, 4), (38, 2), (76, 2)])
def test_cores_policy_cap_holds(lib, cores, kv):
    for rows, tiles, before, now in golden_rows():
        assert lib.pa_cores_policy_splits(cores, kv, tiles) == now


def test_cores_policy_workspace_never_grows(lib):
    # splits * tiles <= 256 slots (the 2048-row chunk's) whenever tiles <= 256
    for cores in (8, 16, 32, 38, 76, 148, 1000):
        for kv in (1, 2, 4, 8):
            for tiles in range(1, 257):
                s = lib.pa_cores_policy_splits(cores, kv, tiles)
                assert 1 <= s <= 32 and s * tiles <= max(256, tiles)


def P(**kw):
    args = dict(n_q_heads=24, n_kv_heads=4, head_dim=256, page_size=64, chunk_rows=512,
                hist_len=32768, dtype="bf16", num_sms=148)
    args.update(kw)
    return binding.plan(**args)


def test_plan_fields(lib):
    p = P(splits=4)
    # head dim 256 runs on CTA pairs: a unit is two consecutive Q tiles
    assert p.group == 6 and p.q_tiles == 24 and p.splits == 4 and p.ctas_per_unit == 2
    assert p.units == 12 * 4 * 4
    assert p.ws_bytes == 4 * 512 * 24 * 257 * 4
    assert abs(p.scale - 1 / 16) < 1e-7 and p.paged == 1 and p.policy == -1


def test_plan_single_split_has_no_workspace(lib):
    p = P(splits=1)
    assert p.ws_bytes == 0 and p.units == 48
    q = P(splits=1, head_dim=128)
    assert q.ctas_per_unit == 1 and q.units == 4 * q.q_tiles


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_plan_workloads(lib, name):
    wl = WORKLOADS[name]
    for h, r in wl.pieces:
        p = binding.plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.page_size, r, h, wl.dtype,
                         wl.scale, 0, "makespan", True, 148)
        G = wl.n_q_heads // wl.n_kv_heads
        assert p.q_tiles == math.ceil(r * G / 128)
        assert 1 <= p.splits <= 32
        last_token = min(r - 1, (p.q_tiles * 128 - 1) // G)
        assert p.splits <= max(1, math.ceil((h + last_token + 1) / 128))
        if p.policy == binding.PA_POLICY_BALANCED:  # cut row blocks: see test_schedule.py
            assert p.ws_bytes % (p.ctas_per_unit * 128 * (wl.head_dim + 1) * 4) == 0
        else:
            assert p.ws_bytes == (0 if p.splits == 1 else
                                  p.splits * r * wl.n_q_heads * (wl.head_dim + 1) * 4)


def test_makespan_policy_fills_the_gpu_at_long_history(lib):
    # 128 rows at 131072 history: 24 (tile, head) units alone would leave 124 SMs idle
    p = P(chunk_rows=128, hist_len=131072)
    assert p.units * p.ctas_per_unit >= 120
    # an empty-history full chunk already fills the GPU: no split
    q = P(chunk_rows=2048, hist_len=0, n_q_heads=16, n_kv_heads=2, page_size=16, dtype="f16")
    assert q.splits == 1


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), "PA_ERR_UNSUPPORTED"),
    (dict(page_size=48), "PA_ERR_UNSUPPORTED"),
    (dict(page_size=256), "PA_ERR_UNSUPPORTED"),
    (dict(n_q_heads=10, n_kv_heads=4), "PA_ERR_UNSUPPORTED"),
    (dict(splits=33), "PA_ERR_UNSUPPORTED"),
    (dict(chunk_rows=0), "PA_ERR_INVALID_ARG"),
    (dict(hist_len=-1), "PA_ERR_INVALID_ARG"),
    (dict(num_sms=0), "PA_ERR_INVALID_ARG"),
    (dict(hist_len=2**31), "PA_ERR_UNSUPPORTED"),
])
def test_plan_rejects(lib, kw, status):
    with pytest.raises(binding.PaError) as e:
        P(**kw)
    assert binding.STATUS[e.value.status] == status


def test_contiguous_plan_ignores_page_size(lib):
    p = P(page_size=48, paged=False)
    assert p.paged == 0 and p.page_size == 0


def test_policies_selectable(lib):
    p = P(chunk_rows=128, hist_len=131072, policy="cores")
    assert p.policy == 1 and p.splits == binding.load_library().pa_cores_policy_splits(148, 4, 6)
    p = P(chunk_rows=128, hist_len=131072, policy="legacy")
    assert p.policy == 2 and p.splits == 1


def test_status_strings(lib):
    for code in binding.STATUS:
        assert lib.pa_status_string(code)


# ------------------------------------------------------------------ the pages' piece rule
def test_pieces_reproduce_the_pages_sizes(lib):
    # splash PR #33, "What changed": 512 rows from 32K history, 256 from 64K, 128 past ~128K
    assert binding.pieces(2048, 32768)[0] == 512
    assert binding.pieces(2048, 65536)[0] == 256
    assert binding.pieces(2048, 131072)[0] == 128
    # the 32K-history workload: four 512-row pieces
    assert binding.pieces(2048, 32768) == [512, 512, 512, 512]


@pytest.mark.parametrize("rows,hist", [(2048, 0), (2048, 30000), (1000, 100000), (7, 5),
                                       (2048, 300000), (1, 0), (0, 10)])
def test_pieces_cover_the_chunk_and_are_maximal(lib, rows, hist):
    ps = binding.pieces(rows, hist)
    assert sum(ps) == rows
    h, left = hist, rows
    for r in ps:
        assert r >= 1 and (r & (r - 1)) == 0
        assert r == 1 or r * (h + r) <= 1 << 25
        # doubling would break the budget or run past the chunk
        assert 2 * r > left or 2 * r * (h + 2 * r) > 1 << 25
        h += r
        left -= r
