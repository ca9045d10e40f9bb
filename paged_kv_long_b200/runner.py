"""Run a whole workload (a sequence of pieces over one KV cache) through libpa on one GPU.

One step is what a prefill engine does for the chunk's attention: for every piece, plan it
(host), then pa_prefill and, when the piece is split, pa_combine on the same stream. Plans,
outputs and the workspace are made once; ``run()`` only enqueues kernels.
"""
from __future__ import annotations

import numpy as np

from . import binding
from .inputs import Inputs


def _dev_tensor(bits: np.ndarray, dtype: str, device):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    t = t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)
    return t.to(device)


class DeviceWorkload:
    def __init__(self, inp: Inputs, device="cuda", paged: bool = True, splits: int | None = None,
                 policy: str = "makespan", num_sms: int | None = None):
        import torch
        wl = inp.wl
        self.wl, self.paged, self.device = wl, paged, torch.device(device)
        self.q = _dev_tensor(inp.q, wl.dtype, self.device)
        if paged:
            self.k = _dev_tensor(inp.k_pool, wl.dtype, self.device)
            self.v = _dev_tensor(inp.v_pool, wl.dtype, self.device)
            self.table = torch.from_numpy(inp.page_table).to(self.device)
        else:
            self.k = _dev_tensor(inp.k_logical, wl.dtype, self.device)
            self.v = _dev_tensor(inp.v_logical, wl.dtype, self.device)
            self.table = None
        if splits is None:
            splits = wl.splits
        self.plans = []
        for h, r in wl.pieces:
            self.plans.append(binding.plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.page_size,
                                           r, h, wl.dtype, wl.scale, splits, policy, paged,
                                           num_sms))
        self.outs = [torch.empty((r, wl.n_q_heads, wl.head_dim), dtype=torch.float32,
                                 device=self.device) for _, r in wl.pieces]
        ws_elems = max(p.ws_bytes for p in self.plans) // 4
        self.ws = torch.empty(max(ws_elems, 4), dtype=torch.float32, device=self.device)

    def piece_inputs(self, i: int):
        h, r = self.wl.pieces[i]
        off = h - self.wl.first_pos
        q = self.q[off:off + r]
        if self.paged:
            return q, self.k, self.v, self.table
        # contiguous K/V of exactly H+R rows for this piece
        return q, self.k[:h + r], self.v[:h + r], None

    def run_piece(self, i: int, stream=None):
        q, k, v, tab = self.piece_inputs(i)
        p = self.plans[i]
        binding.prefill(p, q, k, v, tab, self.outs[i], self.ws, stream)
        binding.combine(p, self.ws, self.outs[i], stream)

    def run(self, stream=None):
        for i in range(len(self.wl.pieces)):
            self.run_piece(i, stream)

    def capture(self, stream=None):
        """The whole step (every chunk's prefill and combine) captured as one CUDA graph: the
        plans, tensor maps and work-item tables are taken at capture (kernel parameters hold
        them by value), so a replay launches the same work with no host-side planning."""
        import torch
        stream = stream or torch.cuda.Stream(self.device)
        stream.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(stream):
            self.run(stream)  # once outside the capture: lazy library and kernel set-up
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            self.run(torch.cuda.current_stream(self.device))
        return graph

    def outputs_host(self) -> list[np.ndarray]:
        return [o.cpu().numpy() for o in self.outs]

    def run_streamed(self, host_q, host_k, host_v, host_table, host_outs, copy_in, compute,
                     copy_out):
        """One step from pinned host memory to pinned host memory with the copies overlapped:
        the K/V pools and the page table go first (every chunk reads pages all over the pool);
        then chunk i's query rows are copied on `copy_in` while earlier chunks compute on
        `compute`, and chunk i's output goes back on `copy_out` while later chunks compute.
        host_q [rows, Hq, D], host_k / host_v like the device pools, host_table int32,
        host_outs: one pinned fp32 tensor per chunk. Enqueues only; returns the event that
        completes with the last output copy."""
        import torch
        wl = self.wl
        compute.wait_stream(copy_out)  # the previous step's outputs have left
        with torch.cuda.stream(copy_in):
            self.k.copy_(host_k, non_blocking=True)
            self.v.copy_(host_v, non_blocking=True)
            if self.table is not None:
                self.table.copy_(host_table, non_blocking=True)
        done = None
        for i, (h, r) in enumerate(wl.pieces):
            off = h - wl.first_pos
            with torch.cuda.stream(copy_in):
                self.q[off:off + r].copy_(host_q[off:off + r], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(copy_in)
            compute.wait_event(ready)
            self.run_piece(i, compute)
            out_ready = torch.cuda.Event()
            out_ready.record(compute)
            copy_out.wait_event(out_ready)
            with torch.cuda.stream(copy_out):
                host_outs[i].copy_(self.outs[i], non_blocking=True)
                done = torch.cuda.Event(enable_timing=True)
                done.record(copy_out)
        # the next step's copies into q / the pools must not overtake this step's reads
        compute_done = torch.cuda.Event()
        compute_done.record(compute)
        copy_in.wait_event(compute_done)
        return done


class PrefillRoutes:
    """The two bulk-prefill routes of a cold prompt (history 0, chunks in order), with the same
    plans' schedules and the same outputs:

    * paged (the hot path): each chunk's K/V, as the projection leaves them in a contiguous
      [R, Hkv, D] buffer, are appended to their pages (pa_kv_append), then prefill reads every
      key through the page table;
    * staged: the projection writes each chunk's K/V straight into a contiguous staging buffer
      [T, Hkv, D] at the chunk's positions, prefill reads the staged keys contiguously, and the
      chunk's rows are then published to their pages (pa_kv_publish).

    Both leave the same page pools behind. ``k_new``/``v_new`` stand for the projection's output
    (the staged route's staging buffer holds the same rows)."""

    def __init__(self, inp: Inputs, device="cuda", policy: str = "makespan",
                 num_sms: int | None = None):
        import torch
        wl = inp.wl
        assert wl.first_pos == 0, "the routes start from an empty cache"
        self.wl, self.device = wl, torch.device(device)
        self.q = _dev_tensor(inp.q, wl.dtype, self.device)
        self.kv_new = (_dev_tensor(inp.k_logical, wl.dtype, self.device),
                       _dev_tensor(inp.v_logical, wl.dtype, self.device))
        self.staged = (self.kv_new[0].clone(), self.kv_new[1].clone())
        shape = inp.k_pool.shape
        dt = self.q.dtype
        self.pools = {r: (torch.zeros(shape, dtype=dt, device=self.device),
                          torch.zeros(shape, dtype=dt, device=self.device))
                      for r in ("paged", "staged")}
        self.table = torch.from_numpy(inp.page_table).to(self.device)
        self.plans = {}
        for route, paged in (("paged", True), ("staged", False)):
            self.plans[route] = [binding.plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                                              wl.page_size, r, h, wl.dtype, wl.scale, 0, policy,
                                              paged, num_sms) for h, r in wl.pieces]
        self.outs = {r: [torch.empty((n, wl.n_q_heads, wl.head_dim), dtype=torch.float32,
                                     device=self.device) for _, n in wl.pieces]
                     for r in ("paged", "staged")}
        ws = max(p.ws_bytes for ps in self.plans.values() for p in ps) // 4
        self.ws = torch.empty(max(ws, 4), dtype=torch.float32, device=self.device)

    def run_paged(self, stream=None):
        kp, vp = self.pools["paged"]
        for i, (h, r) in enumerate(self.wl.pieces):
            binding.kv_append(self.kv_new[0][h:h + r], self.kv_new[1][h:h + r], kp, vp,
                              self.table, h, stream)
            p = self.plans["paged"][i]
            binding.prefill(p, self.q[h:h + r], kp, vp, self.table, self.outs["paged"][i],
                            self.ws, stream)
            binding.combine(p, self.ws, self.outs["paged"][i], stream)

    def run_staged(self, stream=None):
        kp, vp = self.pools["staged"]
        ks, vs = self.staged
        for i, (h, r) in enumerate(self.wl.pieces):
            p = self.plans["staged"][i]
            binding.prefill(p, self.q[h:h + r], ks[:h + r], vs[:h + r], None,
                            self.outs["staged"][i], self.ws, stream)
            binding.combine(p, self.ws, self.outs["staged"][i], stream)
            binding.kv_publish(ks, vs, kp, vp, self.table, h, r, stream)
