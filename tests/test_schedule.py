"""Host checks of the balanced schedule (pa_schedule_items): on many seeded shapes, the work
items of a plan cover every KV tile of every row block exactly once, the workspace slots of the
cut row blocks are consecutive and distinct and match the plan's workspace size, and the items
spread the tiles evenly over the SMs. The visible-tile count of a row block is restated here from
the definition (a unit sees the keys up to the last token of its last Q tile), not taken from the
library."""
import math
import time

import numpy as np
import pytest

from paged_kv_long_b200 import binding


@pytest.fixture(scope="module")
def lib():
    from paged_kv_long_b200.build import build
    build()
    return binding.load_library()


def visible_tiles(unit, per, q_tiles, R, G, H):
    last_qt = min(unit * per + per - 1, q_tiles - 1)
    t_last = min(R - 1, ((last_qt + 1) * 128 - 1) // G)
    return math.ceil((H + t_last + 1) / 128)


def check_schedule(p, items):
    per = p.ctas_per_unit
    q_units = math.ceil(p.q_tiles / per)
    Hkv, G, R, H, D = p.n_kv_heads, p.group, p.chunk_rows, p.hist_len, p.head_dim
    assert len(items) == p.units <= 512
    by_rb = {}
    for rb, kt0, kt1, slot in items:
        assert 0 <= rb < q_units * Hkv and 0 <= kt0 < kt1
        by_rb.setdefault(int(rb), []).append((int(kt0), int(kt1), int(slot)))
    assert sorted(by_rb) == list(range(q_units * Hkv)), "every row block has work"
    slots = []
    for rb, parts in by_rb.items():
        unit = q_units - 1 - rb // Hkv
        n = visible_tiles(unit, per, p.q_tiles, R, G, H)
        parts.sort()
        assert parts[0][0] == 0 and parts[-1][1] == n, (rb, parts, n)
        for a, b in zip(parts, parts[1:]):
            assert a[1] == b[0], f"gap or overlap in row block {rb}: {parts}"
        if len(parts) == 1:
            assert parts[0][2] == -1, "an uncut row block writes the output directly"
        else:
            s = [x[2] for x in parts]
            assert s == list(range(s[0], s[0] + len(s))), "parts take consecutive slots"
            slots += s
        assert len(parts) <= min(32, p.splits)
    assert len(slots) == len(set(slots))
    n_slots = len(slots)
    assert sorted(slots) == list(range(n_slots))
    assert p.ws_bytes == n_slots * per * 128 * (D + 1) * 4
    assert p.splits == max(len(v) for v in by_rb.values())


def greedy_makespan(items, workers, fixed):
    import heapq
    heap = [0.0] * workers
    for _, kt0, kt1, _ in items:
        heapq.heappush(heap, heapq.heappop(heap) + (kt1 - kt0) + fixed)
    return max(heap)


def test_balanced_items_cover_every_tile_once(lib):
    rng = np.random.default_rng(1234)
    t0 = time.time()
    seen_cut = 0
    for _ in range(300):
        Hkv = int(rng.choice([1, 2, 4, 8]))
        G = int(rng.integers(1, 9))
        D = int(rng.choice([64, 128, 256]))
        R = int(rng.choice([1, 7, 128, 300, 1000, 2048, int(rng.integers(1, 4097))]))
        H = int(rng.choice([0, 10, 2048, 30720, int(rng.integers(0, 200_000))]))
        sms = int(rng.choice([2, 4, 8, 16, 40, 148]))
        policy = str(rng.choice(["balanced", "makespan"]))
        p = binding.plan(G * Hkv, Hkv, D, 16, R, H, "bf16", 0.0, 0, policy, True, sms)
        if p.policy != binding.PA_POLICY_BALANCED:
            assert policy == "makespan" or p.units > 0
            continue
        items = binding.schedule_items(p)
        check_schedule(p, items)
        seen_cut += int((items[:, 3] >= 0).any())
    assert seen_cut >= 30, "the shapes should exercise cut row blocks"
    assert time.time() - t0 < 60


@pytest.mark.parametrize("H,R,sms", [(30720, 2048, 148), (18432, 2048, 148), (131072, 128, 148),
                                     (2000, 300, 8)])
def test_balanced_items_spread_the_tiles_evenly(lib, H, R, sms):
    p = binding.plan(16, 2, 256, 16, R, H, "f16", 0.0, 0, "balanced", True, sms)
    assert p.policy == binding.PA_POLICY_BALANCED
    items = binding.schedule_items(p)
    check_schedule(p, items)
    workers = sms // p.ctas_per_unit
    fixed = 2.4  # a unit's fixed cost in KV tiles, about what the planner assumes
    total = sum(int(b - a) + fixed for _, a, b, _ in items)
    longest = max(int(b - a) for _, a, b, _ in items)
    # dispatching the items in order to the first free worker stays close to an even split
    assert greedy_makespan(items, workers, fixed) <= total / workers * 1.06 + longest / 8 + fixed


def test_schedule_items_of_a_uniform_plan_is_empty(lib):
    p = binding.plan(16, 2, 256, 16, 2048, 30720, "f16", 0.0, 4, "makespan", True, 148)
    assert p.policy == -1 and len(binding.schedule_items(p)) == 0
