"""The whole forward path captured once into a CUDA graph.

For fixed shapes the chain of launches (optional Hilbert table and permutes,
pooling, select, attention, optional inverse permute) is the same on every
call, so it is recorded once and replayed: one graph launch instead of up to
eleven kernel launches and their host-side argument checks.  This matters for
small problems, whose kernels run for microseconds each.

The graph owns static buffers: the caller writes Q, K, V into ``g.q``, ``g.k``,
``g.v`` (or passes tensors to ``run``, which copies them in), calls ``run`` and
reads ``g.o``.  Every kernel in the graph is the library's own; the graph is
only a recording of the calls the binding makes.
"""
from __future__ import annotations

import torch

from . import (SPARGE_BF16, SPARGE_F16, SPARGE_F32, predict_outputs, sparge_attn_fwd,
               sparge_hilbert_index, sparge_hilbert_permute, sparge_hilbert_workspace_bytes,
               sparge_inverse_permute, sparge_predict_pool, sparge_predict_select, workspace)

_TD = {SPARGE_F16: torch.float16, SPARGE_BF16: torch.bfloat16, SPARGE_F32: torch.float32}


class SpargeGraph:
    """Captured predictor + attention (+ Hilbert permutation) for one shape.

    params: SpargeParams of the problem.  grid: optional (prefix_len, T, Hg, Wg)
    of a token grid; with it the graph builds the Hilbert table, permutes Q, K,
    V, and puts O back in token order, all inside the graph."""

    def __init__(self, params, grid=None, device="cuda"):
        dev = torch.device(device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.params, self.grid, self.device = params, grid, dev
        p = params
        io, od = _TD[p.io_dtype], _TD[p.o_dtype]
        self.q = torch.zeros((p.B, p.Hq, p.N, p.d), dtype=io, device=dev)
        self.k = torch.zeros((p.B, p.Hkv, p.N, p.d), dtype=io, device=dev)
        self.v = torch.zeros((p.B, p.Hkv, p.N, p.d), dtype=io, device=dev)
        self.o = torch.zeros((p.B, p.Hq, p.N, p.d), dtype=od, device=dev)
        self.ws = workspace(p, dev)
        self.mask, self.kv_idx, self.kv_cnt, _, _ = predict_outputs(p, dev)
        if grid is not None:
            _, T, Hg, Wg = grid
            self.perm = torch.empty(p.N, dtype=torch.int32, device=dev)
            self.hws = torch.zeros(sparge_hilbert_workspace_bytes(T, Hg, Wg),
                                   dtype=torch.uint8, device=dev)
            self.qp, self.kp, self.vp = (torch.empty_like(x) for x in (self.q, self.k, self.v))
            self.op = torch.empty_like(self.o)
        self.graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._forward()                   # once outside the capture (lazy setup)
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(self.graph, stream=side, capture_error_mode="relaxed"):
            self._forward()
        torch.cuda.synchronize(dev)

    def _forward(self):
        p = self.params
        q, k, v, o = self.q, self.k, self.v, self.o
        if self.grid is not None:
            prefix, T, Hg, Wg = self.grid
            sparge_hilbert_index(p.N, prefix, T, Hg, Wg, self.perm, self.hws)
            sparge_hilbert_permute(q, self.qp, self.perm)
            sparge_hilbert_permute(k, self.kp, self.perm)
            sparge_hilbert_permute(v, self.vp, self.perm)
            q, k, v, o = self.qp, self.kp, self.vp, self.op
        sparge_predict_pool(p, q, k, self.ws)
        sparge_predict_select(p, self.mask, self.kv_idx, self.kv_cnt, None, None, self.ws)
        sparge_attn_fwd(p, q, k, v, self.kv_idx, self.kv_cnt, o, self.ws)
        if self.grid is not None:
            sparge_inverse_permute(self.op, self.o, self.perm)

    def run(self, q=None, k=None, v=None) -> torch.Tensor:
        """Replays the graph on the current stream; tensors given are copied
        into the static inputs first.  Returns the static output ``o``."""
        for src, dst in ((q, self.q), (k, self.k), (v, self.v)):
            if src is not None:
                dst.copy_(src)
        self.graph.replay()
        return self.o
