"""The entry point that allocates nothing (pa_prefill_noalloc).

Some callers cannot allocate device memory: a plugin inside a serving engine that has
reserved the device's memory for its KV-cache pool and hands out no allocator, or a caller
that cannot afford the implicit device synchronisation an allocation may cause. For them the
library keeps its split scratch in a device array of its own. These checks call that entry
point through the C ABI twice in a row (different inputs, so the second call starts from the
first call's leftover scratch) and compare each output with the workspace entry points
(pa_prefill + pa_combine with a caller-allocated workspace), within the tolerance of the other
GPU tests. This file is collected last so that a stop at its first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest

from tests.conftest import cuda_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

MAX_ABS, REL_RMS = 1e-2, 2e-3


def _inputs(seed, H, R):
    from paged_kv_long_b200.inputs import Workload, generate
    from paged_kv_long_b200.runner import DeviceWorkload
    wl = Workload("noalloc 24q/4kv D256 PS64 bf16", 24, 4, 256, 64, "bf16", ((H, R),), splits=8,
                  seed_base=seed)
    return DeviceWorkload(generate(wl), "cuda", paged=True)


def _close(a, b):
    a, b = a.astype(np.float64), b.astype(np.float64)
    d = a - b
    return np.abs(d).max() <= MAX_ABS and np.sqrt((d ** 2).sum() / (b ** 2).sum()) <= REL_RMS


def test_noalloc_matches_workspace_entry_points_twice():
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.build import build
    build()
    lib = binding.load_library()
    for call, (seed, H, R) in enumerate([(7100, 5000, 200), (7200, 3000, 150)]):
        dw = _inputs(seed, H, R)
        p = dw.plans[0]
        assert p.splits == 8 and 0 < p.ws_bytes <= 64 << 20
        q, k, v, tab = dw.piece_inputs(0)
        dw.run()                                      # workspace entry points
        want = dw.outs[0].cpu().numpy()
        out = torch.full_like(dw.outs[0], float("nan"))
        st = lib.pa_prefill_noalloc(ctypes.byref(p), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    tab.data_ptr(), k.shape[0], p.hist_len, p.chunk_rows,
                                    out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, binding.STATUS.get(st, st)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all(), f"call {call}: output not fully written"
        assert _close(got, want), f"call {call}: differs from the workspace entry points"
    st, flags = binding.device_error(reset=True)
    assert st == 0, flags


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
