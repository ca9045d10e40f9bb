"""Shared helpers of the GPU parity tests: run a workload on the GPU, ask the oracle for the
same outputs, compare with the tolerance stated for this path (max-abs <= 1e-2 and relative
RMS <= 2e-3 on N(0,1) inputs)."""
from __future__ import annotations

import numpy as np

from oracle import oracle
from paged_kv_long_b200.inputs import Inputs, Workload, generate

MAX_ABS = 1e-2
REL_RMS = 2e-3


def oracle_problem(inp: Inputs, piece: int, paged: bool = True) -> oracle.Problem:
    wl = inp.wl
    h, r = wl.pieces[piece]
    q = inp.piece_q(piece)
    if paged:
        return oracle.Problem(q=q, k=inp.k_pool, v=inp.v_pool, hist_len=h, dtype=wl.dtype,
                              page_table=inp.page_table, scale=wl.scale)
    return oracle.Problem(q=q, k=inp.k_logical[:h + r], v=inp.v_logical[:h + r], hist_len=h,
                          dtype=wl.dtype, scale=wl.scale)


def sample_pairs(R: int, Hq: int, n: int, seed: int, G: int):
    """Seeded (row, head) samples: first/last rows, rows at Q-tile boundaries, random rest."""
    rng = np.random.default_rng(seed)
    rows = [0, R - 1, min(R - 1, 128 // G), min(R - 1, (128 // G) + 1), R // 2]
    rows += list(rng.integers(0, R, size=max(0, n - len(rows))))
    heads = list(rng.integers(0, Hq, size=len(rows)))
    heads[0], heads[1] = 0, Hq - 1
    return np.array(rows, dtype=np.int64), np.array(heads, dtype=np.int32)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    rel_rms = float(np.sqrt(np.sum(diff ** 2) / max(np.sum(ref ** 2), 1e-300)))
    return max_abs, rel_rms


def assert_close(got, ref, what: str):
    assert np.isfinite(got).all(), f"{what}: non-finite GPU output"
    max_abs, rel_rms = errors(got, ref)
    assert max_abs <= MAX_ABS and rel_rms <= REL_RMS, \
        f"{what}: max_abs={max_abs:.3e} rel_rms={rel_rms:.3e}"
    return max_abs, rel_rms


def custom_workload(name, Hq, Hkv, D, PS, dtype, pieces, seed, splits=0, pool_factor=1.25,
                    scale=0.0) -> Workload:
    return Workload(name, Hq, Hkv, D, PS, dtype, tuple(pieces), pool_factor=pool_factor,
                    splits=splits, scale=scale, seed_base=seed)


def run_gpu(inp: Inputs, paged=True, splits=None, policy="makespan", num_sms=None):
    from paged_kv_long_b200.runner import DeviceWorkload
    import torch
    dw = DeviceWorkload(inp, "cuda", paged=paged, splits=splits, policy=policy, num_sms=num_sms)
    # NaN in the workspace and outputs: an entry read before it is written shows up as a
    # non-finite output (assert_close checks finiteness)
    dw.ws.fill_(float("nan"))
    for o in dw.outs:
        o.fill_(float("nan"))
    dw.run()
    torch.cuda.synchronize()
    return dw, dw.outputs_host()


def check_full(inp: Inputs, outs, paged=True, what=""):
    """Every output of every piece against the oracle."""
    stats = []
    for i, (h, r) in enumerate(inp.wl.pieces):
        ref, _ = oracle.attend(oracle_problem(inp, i, paged))
        got = outs[i].reshape(ref.shape)
        stats.append(assert_close(got, ref, f"{what} piece {i} (H={h}, R={r})"))
    return stats


def check_sampled(inp: Inputs, outs, n=48, paged=True, what=""):
    wl = inp.wl
    G = wl.n_q_heads // wl.n_kv_heads
    stats = []
    for i, (h, r) in enumerate(wl.pieces):
        rows, heads = sample_pairs(r, wl.n_q_heads, n, 7919 + i, G)
        ref, _ = oracle.attend(oracle_problem(inp, i, paged), rows, heads)
        got = outs[i][rows, heads]
        stats.append(assert_close(got, ref, f"{what} piece {i} (H={h}, R={r}) sampled"))
    return stats


def all_heads(rows, Hq: int):
    """(row, head) pairs covering every head of each given row."""
    rows = np.asarray(rows, dtype=np.int64)
    return np.repeat(rows, Hq), np.tile(np.arange(Hq, dtype=np.int32), len(rows))


def oracle_rows(inp: Inputs, piece: int, rows, paged: bool = True):
    """The oracle's outputs for every head of the given rows of one piece: (ref [n, D], pairs)."""
    rr, hh = all_heads(rows, inp.wl.n_q_heads)
    ref, _ = oracle.attend(oracle_problem(inp, piece, paged), rr, hh)
    return ref, (rr, hh)


def check_rows(got_piece: np.ndarray, ref: np.ndarray, pairs, what: str):
    """GPU outputs of one piece at the given (row, head) pairs against the oracle's."""
    rr, hh = pairs
    return assert_close(got_piece[rr, hh], ref, what)


def gen(wl, poison=True, distribution="normal"):
    return generate(wl, poison=poison, distribution=distribution)
