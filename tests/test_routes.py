"""The two bulk-prefill routes of a cold prompt: paged (append each chunk's K/V to pages, then
prefill through the table) and contiguous staging + page publish (prefill on the staging
buffer, then publish the chunk's rows to pages). BaseRT issue #51, "Expected vs actual",
proposes the second as an alternative to a faster paged kernel.

Both must give the same attention outputs bit for bit (the kernel's paged and contiguous reads
run the same schedule on the same keys) and leave the same page pools, equal to the KV-append
oracle applied chunk by chunk; the outputs match the attention oracle.
"""
import numpy as np
import pytest

from oracle.kv_append import kv_append as oracle_append
from tests.conftest import cuda_available
from tests import parity_util as U

CASES = [
    # name, Hq, Hkv, D, PS, dtype, pieces (cold prompt in chunks)
    ("d256_three_chunks", 16, 2, 256, 16, "f16", [(0, 300), (300, 500), (800, 333)]),
    ("d128_bf16", 8, 2, 128, 64, "bf16", [(0, 1024), (1024, 1024)]),
    ("d64_ragged", 4, 1, 64, 16, "f16", [(0, 1), (1, 130), (131, 17)]),
]


def _host(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_staged_route_equals_paged_route(case):
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.runner import PrefillRoutes
    name, Hq, Hkv, D, PS, dtype, pieces = case
    wl = U.custom_workload(name, Hq, Hkv, D, PS, dtype, pieces, seed=7100 + len(name))
    inp = U.gen(wl, poison=False)
    binding.device_error(reset=True)
    rt = PrefillRoutes(inp, "cuda")
    rt.run_paged()
    rt.run_staged()
    torch.cuda.synchronize()
    assert binding.device_error(reset=True)[0] == 0
    # the pools: both routes, and the oracle's appends chunk by chunk onto an empty pool
    want_k = np.zeros(inp.k_pool.shape, dtype=np.uint16)
    want_v = np.zeros(inp.v_pool.shape, dtype=np.uint16)
    for h, r in pieces:
        want_k, _ = oracle_append(want_k, inp.k_logical[h:h + r], inp.page_table, h)
        want_v, _ = oracle_append(want_v, inp.v_logical[h:h + r], inp.page_table, h)
    for route in ("paged", "staged"):
        kp, vp = rt.pools[route]
        assert np.array_equal(_host(kp), want_k), f"{route}: K pool"
        assert np.array_equal(_host(vp), want_v), f"{route}: V pool"
    for i in range(len(pieces)):
        a = rt.outs["paged"][i].cpu().numpy()
        b = rt.outs["staged"][i].cpu().numpy()
        assert np.array_equal(a, b), f"chunk {i}: routes differ"
    outs = [o.cpu().numpy() for o in rt.outs["paged"]]
    U.check_full(inp, outs, paged=True, what=name)
