"""The entry point that allocates nothing (pa_prefill_noalloc).

Some callers cannot allocate device memory: a plugin inside a serving engine that has
reserved the device's memory for its KV-cache pool and hands out no allocator, or a caller
that cannot afford the implicit device synchronisation an allocation may cause. For them the
library keeps its split scratch in a device array of its own. These checks call that entry
point through the C ABI (directly, and through the Python binding's argument checks) several
times in a row, with different inputs, so that each call starts from the previous call's
leftover scratch. Each output must equal, bit for bit, what the workspace entry points
(pa_prefill + pa_combine with a caller-allocated workspace) give on the same plan, since both
run the same kernels on the same schedule; and it must agree with the fp64 oracle within the
tolerance of the other GPU tests. This file is collected last so that a stop at its first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

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


def _workload(seed, pieces, splits=0, Hq=24, Hkv=4, PS=64, dtype="bf16"):
    from paged_kv_long_b200.inputs import Workload, generate
    wl = Workload(f"noalloc {Hq}q/{Hkv}kv D256 PS{PS} {dtype}", Hq, Hkv, 256, PS, dtype,
                  tuple(pieces), splits=splits, seed_base=seed)
    return generate(wl)


def _with_workspace(dw):
    """The workspace entry points' output of piece 0 (NaN-filled workspace and output first)."""
    dw.ws.fill_(float("nan"))
    dw.outs[0].fill_(float("nan"))
    dw.run()
    return dw.outs[0].cpu().numpy()


def _noalloc_c(dw, out):
    """pa_prefill_noalloc called through the C symbol."""
    import torch
    from paged_kv_long_b200 import binding
    p = dw.plans[0]
    q, k, v, tab = dw.piece_inputs(0)
    st = binding.load_library().pa_prefill_noalloc(
        ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
        tab.data_ptr() if tab is not None else None, k.shape[0] if tab is not None else 0,
        p.hist_len, p.chunk_rows, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, binding.STATUS.get(st, st)


def _noalloc_py(dw, out):
    """pa_prefill_noalloc called through the binding (its argument checks included)."""
    from paged_kv_long_b200 import binding
    q, k, v, tab = dw.piece_inputs(0)
    binding.prefill_noalloc(dw.plans[0], q, k, v, tab, out)


def _run_noalloc(dw, call):
    import torch
    out = torch.full_like(dw.outs[0], float("nan"))
    call(dw, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.isfinite(got).all(), "output not fully written"
    return got


def _against_oracle(inp, got, full, what):
    from tests import parity_util as U
    if full:
        ref, pairs = U.oracle_rows(inp, 0, np.arange(inp.wl.pieces[0][1]))
    else:
        G = inp.wl.n_q_heads // inp.wl.n_kv_heads
        rows, heads = U.sample_pairs(inp.wl.pieces[0][1], inp.wl.n_q_heads, 48, 31, G)
        ref, pairs = U.oracle.attend(U.oracle_problem(inp, 0, inp.extra.get("paged", True)),
                                     rows, heads)[0], (rows, heads)
    U.check_rows(got, ref, pairs, what)


def test_noalloc_uniform_splits_twice_equals_workspace_bits():
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.runner import DeviceWorkload
    for call, (seed, H, R, fn) in enumerate([(7100, 5000, 200, _noalloc_c),
                                             (7200, 3000, 150, _noalloc_py)]):
        inp = _workload(seed, [(H, R)], splits=8)
        dw = DeviceWorkload(inp, "cuda", paged=True)
        p = dw.plans[0]
        assert p.splits == 8 and p.policy != binding.PA_POLICY_BALANCED
        assert 0 < p.ws_bytes <= 64 << 20
        want = _with_workspace(dw)
        got = _run_noalloc(dw, fn)
        assert np.array_equal(got, want), f"call {call}: differs from the workspace entry points"
        _against_oracle(inp, got, False, f"noalloc uniform call {call}")


def test_noalloc_balanced_cut_row_blocks_against_oracle():
    """A balanced plan whose row blocks are cut into parts: the partials of the cut blocks go
    to the library's scratch and the merge of cut row blocks reads them back from there."""
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.runner import DeviceWorkload
    for call, (seed, pieces, sms, fn) in enumerate([
            (7300, [(3000, 100)], 16, _noalloc_py),
            (7400, [(5000, 40)], 6, _noalloc_c)]):
        inp = _workload(seed, pieces, Hq=24 if call == 0 else 16, Hkv=4 if call == 0 else 2,
                        PS=64 if call == 0 else 16, dtype="bf16" if call == 0 else "f16")
        dw = DeviceWorkload(inp, "cuda", paged=True, policy="balanced", num_sms=sms)
        p = dw.plans[0]
        assert p.policy == binding.PA_POLICY_BALANCED
        assert (binding.schedule_items(p)[:, 3] >= 0).any(), "no row block is cut"
        assert 0 < p.ws_bytes <= 64 << 20
        want = _with_workspace(dw)
        got = _run_noalloc(dw, fn)
        assert np.array_equal(got, want), f"call {call}: differs from the workspace entry points"
        _against_oracle(inp, got, True, f"noalloc balanced call {call}")


def test_noalloc_contiguous_and_single_split():
    """K/V in contiguous buffers (no page table), and a plan of one split (no scratch at all:
    the kernel writes the output directly)."""
    from paged_kv_long_b200.runner import DeviceWorkload
    inp = _workload(7500, [(2500, 120)], splits=4)
    dw = DeviceWorkload(inp, "cuda", paged=False)
    assert dw.plans[0].ws_bytes > 0 and dw.table is None
    want = _with_workspace(dw)
    got = _run_noalloc(dw, _noalloc_py)
    assert np.array_equal(got, want)
    inp.extra["paged"] = False
    _against_oracle(inp, got, False, "noalloc contiguous")
    inp1 = _workload(7600, [(700, 64)], splits=1)
    dw1 = DeviceWorkload(inp1, "cuda", paged=True)
    assert dw1.plans[0].splits == 1 and dw1.plans[0].ws_bytes == 0
    want1 = _with_workspace(dw1)
    got1 = _run_noalloc(dw1, _noalloc_c)
    assert np.array_equal(got1, want1)
    _against_oracle(inp1, got1, False, "noalloc one split")


def test_noalloc_call_changes_no_free_device_memory():
    """After a first call (which loads the kernels and looks the scratch up), a second call
    leaves the device's free memory exactly as it was."""
    import torch
    from paged_kv_long_b200.runner import DeviceWorkload
    inp = _workload(7700, [(4000, 100)], splits=6)
    dw = DeviceWorkload(inp, "cuda", paged=True)
    out = torch.empty_like(dw.outs[0])
    _noalloc_c(dw, out)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    _noalloc_c(dw, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"free device memory moved by {free0 - free1} bytes"


def test_noalloc_rejects_a_workspace_beyond_its_limit():
    import torch
    from paged_kv_long_b200 import binding
    lib = binding.load_library()
    # 32 splits of 2048 rows x 16 heads x 257 floats need 269 MB, past the 64 MiB scratch
    p = binding.plan(16, 2, 256, 16, 2048, 30720, "f16", splits=32)
    assert p.ws_bytes > 64 << 20
    dummy = torch.zeros(16, dtype=torch.float16, device="cuda")
    st = lib.pa_prefill_noalloc(ctypes.byref(p), dummy.data_ptr(), dummy.data_ptr(),
                                dummy.data_ptr(), dummy.data_ptr(), 1, p.hist_len, p.chunk_rows,
                                dummy.data_ptr(), None)
    assert binding.STATUS[st] == "PA_ERR_WORKSPACE"
