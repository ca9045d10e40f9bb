"""Pins of the fp64 CPU oracle against things other than itself.

The pages print no worked example of the attention values, so the oracle is pinned by:
  * the exact decoding of every 16-bit pattern against numpy / torch conversions;
  * brute force on tiny inputs through an independent route (numpy gather of the logical
    K/V, full masked score matrix, scipy's softmax and logsumexp);
  * torch's fp64 scaled-dot-product attention (a library routine) with an explicit causal
    mask and GQA head sharing;
  * closed forms (one visible key, zero queries, two keys, identical keys);
  * invariants the method must keep: page-shuffle invariance (BaseRT issue #51: paged must
    equal contiguous), split-and-merge invariance (splash PR #33, "Testing": splitting the
    history only changes rounding), softmax rows summing to 1, MHA-by-duplication.
A final test plants deliberate mistakes in the oracle (compile-time mutants) and checks that
these pins catch every one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import oracle
from paged_kv_long_b200.inputs import small_problem, to_bits


def np_decode(bits, dtype):
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "f16":
        return bits.view(np.float16).astype(np.float64)
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def brute_force(q, k_log, v_log, H, dtype, scale):
    """Independent route: full masked score matrix over logical K/V + scipy softmax."""
    Q, K, V = np_decode(q, dtype), np_decode(k_log, dtype), np_decode(v_log, dtype)
    R, Hq, D = Q.shape
    G = Hq // K.shape[1]
    Kx, Vx = np.repeat(K, G, axis=1), np.repeat(V, G, axis=1)
    sc = np.einsum("rhd,thd->hrt", Q, Kx) * scale
    T = K.shape[0]
    mask = np.arange(T)[None, :] > (H + np.arange(R))[:, None]
    sc = np.where(mask[None], -np.inf, sc)
    w = scipy.special.softmax(sc, axis=-1)
    out = np.einsum("hrt,thd->rhd", w, Vx)
    lse = scipy.special.logsumexp(sc, axis=-1).T  # [R, Hq]
    return out, lse, w


def sdpa_reference(q, k_log, v_log, H, dtype, scale):
    Q = torch.from_numpy(np_decode(q, dtype)).permute(1, 0, 2)[None]
    K = torch.from_numpy(np_decode(k_log, dtype)).permute(1, 0, 2)[None]
    V = torch.from_numpy(np_decode(v_log, dtype)).permute(1, 0, 2)[None]
    R, T = Q.shape[2], K.shape[2]
    allowed = torch.arange(T)[None, :] <= (H + torch.arange(R))[:, None]
    out = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, attn_mask=allowed, scale=scale, enable_gqa=True)
    return out[0].permute(1, 0, 2).numpy()


def paged_problem(seed, R, H, Hq, Hkv, D, PS, dtype, lib_path=None, scale=0.0):
    q, kp, vp, tab, k, v = small_problem(seed, R, H, Hq, Hkv, D, PS, dtype)
    pb = oracle.Problem(q=q, k=kp, v=vp, hist_len=H, dtype=dtype, page_table=tab, scale=scale,
                        lib_path=lib_path)
    return pb, k, v


TINY_CASES = [
    # seed, R, H, Hq, Hkv, D, PS, dtype
    (1, 5, 0, 2, 1, 8, 4, "f16"),
    (2, 8, 40, 6, 2, 16, 4, "bf16"),
    (3, 7, 13, 3, 3, 12, 4, "f16"),
    (4, 1, 37, 4, 1, 16, 4, "bf16"),
    (5, 8, 3, 8, 2, 4, 4, "f16"),
]


# ----------------------------------------------------------------------------- decoding
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_decode_every_pattern(oracle_lib, dtype):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(dtype, bits)
    ref = np_decode(bits, dtype)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ----------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("case", TINY_CASES)
def test_brute_force_tiny(oracle_lib, case):
    seed, R, H, Hq, Hkv, D, PS, dtype = case
    pb, k, v = paged_problem(seed, R, H, Hq, Hkv, D, PS, dtype)
    scale = 1.0 / math.sqrt(D)
    out, lse = oracle.attend(pb)
    ref, ref_lse, _ = brute_force(pb.q, k, v, H, dtype, scale)
    np.testing.assert_allclose(out.reshape(R, Hq, D), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(R, Hq), ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", TINY_CASES)
def test_torch_sdpa_fp64(oracle_lib, case):
    seed, R, H, Hq, Hkv, D, PS, dtype = case
    pb, k, v = paged_problem(seed, R, H, Hq, Hkv, D, PS, dtype)
    out, _ = oracle.attend(pb)
    ref = sdpa_reference(pb.q, k, v, H, dtype, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out.reshape(ref.shape), ref, rtol=0, atol=1e-12)


def test_explicit_scale(oracle_lib):
    pb, k, v = paged_problem(11, 6, 9, 4, 2, 8, 4, "f16", scale=0.3)
    out, _ = oracle.attend(pb)
    ref, _, _ = brute_force(pb.q, k, v, 9, "f16", 0.3)
    np.testing.assert_allclose(out.reshape(ref.shape), ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- closed forms
def test_first_row_empty_history_is_v0(oracle_lib):
    pb, k, v = paged_problem(21, 4, 0, 4, 2, 16, 4, "bf16")
    out, lse = oracle.attend(pb, rows=[0, 0, 0, 0], heads=[0, 1, 2, 3])
    V = np_decode(v, "bf16")
    for h in range(4):
        assert np.array_equal(out[h], V[0, h // 2])  # one visible key: weight exactly 1
    Q, K = np_decode(pb.q, "bf16"), np_decode(k, "bf16")
    s = np.array([Q[0, h] @ K[0, h // 2] / 4.0 for h in range(4)])
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-13)  # lse of one key = its score


def test_zero_query_gives_mean_of_visible_v(oracle_lib):
    pb, k, v = paged_problem(22, 6, 10, 2, 1, 8, 4, "f16")
    pb.q[:] = 0
    out, lse = oracle.attend(pb)
    V = np_decode(v, "f16")
    for i in range(6):
        mean = V[:10 + i + 1, 0].mean(axis=0)
        for h in range(2):
            np.testing.assert_allclose(out[i * 2 + h], mean, rtol=0, atol=1e-14)
            assert abs(lse[i * 2 + h] - math.log(10 + i + 1)) < 1e-13


def test_two_keys_sigmoid(oracle_lib):
    pb, k, v = paged_problem(23, 1, 1, 1, 1, 16, 4, "f16")
    out, _ = oracle.attend(pb)
    Q, K, V = np_decode(pb.q, "f16"), np_decode(k, "f16"), np_decode(v, "f16")
    s0, s1 = Q[0, 0] @ K[0, 0] / 4.0, Q[0, 0] @ K[1, 0] / 4.0
    w1 = 1.0 / (1.0 + math.exp(-(s1 - s0)))
    np.testing.assert_allclose(out[0], (1 - w1) * V[0, 0] + w1 * V[1, 0], rtol=0, atol=1e-14)


def test_identical_keys_give_that_value(oracle_lib):
    pb, k, v = paged_problem(24, 3, 20, 2, 1, 8, 4, "bf16")
    tab = pb.page_table
    # every used pool slot holds the same K row and the same V row
    krow, vrow = pb.k[tab[0], 0, 0].copy(), pb.v[tab[0], 0, 0].copy()
    pb.k[tab] = krow
    pb.v[tab] = vrow
    out, _ = oracle.attend(pb)
    Vr = np_decode(vrow, "bf16")
    for n in range(out.shape[0]):
        np.testing.assert_allclose(out[n], Vr, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- invariants
def test_page_shuffle_bit_identical(oracle_lib):
    pb, k, v = paged_problem(31, 8, 29, 6, 2, 16, 4, "bf16")
    out, lse = oracle.attend(pb)
    rng = np.random.default_rng(99)
    P = pb.k.shape[0]
    perm = rng.permutation(P)          # new physical position of old page p is perm[p]
    k2 = np.empty_like(pb.k)
    v2 = np.empty_like(pb.v)
    k2[perm] = pb.k
    v2[perm] = pb.v
    tab2 = perm[pb.page_table].astype(np.int32)
    pb2 = oracle.Problem(q=pb.q, k=k2, v=v2, hist_len=pb.hist_len, dtype="bf16", page_table=tab2)
    out2, lse2 = oracle.attend(pb2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_paged_equals_contiguous(oracle_lib):
    pb, k, v = paged_problem(32, 7, 18, 4, 2, 16, 4, "f16")
    out, lse = oracle.attend(pb)
    pc = oracle.Problem(q=pb.q, k=k, v=v, hist_len=pb.hist_len, dtype="f16")
    outc, lsec = oracle.attend(pc)
    assert np.array_equal(out, outc) and np.array_equal(lse, lsec)


@pytest.mark.parametrize("S", [1, 2, 3, 7])
def test_split_and_merge_equals_whole(oracle_lib, S):
    pb, k, v = paged_problem(33, 6, 45, 4, 2, 16, 4, "bf16")
    R, Hq, D = pb.q.shape
    T = pb.hist_len + R
    out, lse = oracle.attend(pb)
    bounds = [T * s // S for s in range(S + 1)]
    parts = [oracle.attend(pb, key_lo=bounds[s], key_hi=bounds[s + 1]) for s in range(S)]
    for n in range(R * Hq):
        o_s = np.stack([p[0][n] for p in parts])
        l_s = np.array([p[1][n] for p in parts])
        m, ml = oracle.merge(l_s, o_s)
        np.testing.assert_allclose(m, out[n], rtol=0, atol=1e-12)
        assert abs(ml - lse[n]) < 1e-12


def test_weights_sum_to_one_and_respect_causality(oracle_lib):
    pb, k, v = paged_problem(34, 5, 12, 4, 1, 8, 4, "f16")
    _, _, wref = brute_force(pb.q, k, v, 12, "f16", 1.0 / math.sqrt(8))
    for i in range(5):
        for h in range(4):
            w = oracle.weights(pb, i, h)
            assert abs(w.sum() - 1.0) < 1e-12
            assert np.all(w[12 + i + 1:] == 0.0)
            assert np.all(w[:12 + i + 1] > 0.0)
            np.testing.assert_allclose(w, wref[h, i], rtol=0, atol=1e-13)


def test_mha_by_duplicated_kv_heads(oracle_lib):
    pb, k, v = paged_problem(35, 6, 10, 6, 2, 8, 4, "bf16")
    out, _ = oracle.attend(pb)
    G = 3
    pm = oracle.Problem(q=pb.q, k=np.repeat(pb.k, G, axis=2), v=np.repeat(pb.v, G, axis=2),
                        hist_len=10, dtype="bf16", page_table=pb.page_table)
    outm, _ = oracle.attend(pm)
    assert np.array_equal(out, outm)


def test_poisoned_slots_never_reach_output(oracle_lib):
    pb, k, v = paged_problem(36, 7, 6, 2, 1, 8, 4, "f16")  # 13 keys: last page partly unused
    assert np.isnan(np_decode(pb.v[pb.page_table[-1], 3], "f16")).all()
    out, lse = oracle.attend(pb)
    assert np.isfinite(out).all() and np.isfinite(lse).all()


def test_bad_page_entry_is_an_error(oracle_lib):
    pb, k, v = paged_problem(37, 4, 4, 2, 1, 8, 4, "f16")
    pb.page_table[0] = pb.k.shape[0]
    with pytest.raises(RuntimeError):
        oracle.attend(pb)


def test_empty_key_range_gives_neg_inf(oracle_lib):
    pb, k, v = paged_problem(38, 4, 8, 2, 1, 8, 4, "bf16")
    out, lse = oracle.attend(pb, rows=[0], heads=[0], key_lo=9, key_hi=12)  # row 0 sees 0..8
    assert lse[0] == -np.inf and np.all(out == 0)


# ----------------------------------------------------------------------------- mutants
def run_pin_battery(lib_path) -> list[str]:
    """Run the value pins against an oracle build; return the names of pins that fail."""
    failed = []
    for case in TINY_CASES:
        seed, R, H, Hq, Hkv, D, PS, dtype = case
        pb, k, v = paged_problem(seed, R, H, Hq, Hkv, D, PS, dtype, lib_path=lib_path)
        try:
            out, lse = oracle.attend(pb)
        except RuntimeError:
            failed.append(f"attend-error{case}")
            continue
        ref, ref_lse, _ = brute_force(pb.q, k, v, H, dtype, 1.0 / math.sqrt(D))
        if not np.allclose(out.reshape(ref.shape), ref, rtol=0, atol=1e-12):
            failed.append(f"brute-out{case}")
        if not np.allclose(lse.reshape(R, Hq), ref_lse, rtol=0, atol=1e-12):
            failed.append(f"brute-lse{case}")
    return failed


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5])
def test_planted_mistakes_are_caught(oracle_lib, mutant, tmp_path):
    path = oracle.build(mutant=mutant, out_path=str(tmp_path / f"mutant{mutant}.so"))
    failed = run_pin_battery(path)
    assert failed, f"mutant {mutant} passed every pin"


def test_real_oracle_passes_battery(oracle_lib):
    assert run_pin_battery(oracle.LIB) == []
