"""A decode step over a stack of CSA layers, run as one CUDA graph.

Per layer, in order on one stream (DeepSeek-V4-Flash architecture post,
section (B)): the lightning indexer scores every compressed entry, the top-k
rows are selected, and sparse MQA attention reads those rows plus the
sliding window.  Each layer has its own caches and queries.

The step owns its device buffers and prebuilt C-ABI argument structs, so an
enqueue is nothing but the library calls; `capture()` records them into a
CUDA graph that `replay()` launches with one call.
"""
from __future__ import annotations

import ctypes as C
from typing import List, Optional, Sequence

import torch

from . import (AttnArgs, DeviceKV, ScoreArgs, TopkArgs, BF16, LAUNCH_PDL, OP_ATTN, OP_TOPK, STATS_SPAN, LidxError,
               attn_args, lib, topk_args, workspace, workspace_size)


class LayerCache:
    """Device caches of one CSA layer: index keys (dim 128), compressed KV rows
    and sliding-window rows (dim 512), for B sequences."""

    def __init__(self, keys: DeviceKV, kv: DeviceKV, swa: DeviceKV):
        self.keys, self.kv, self.swa = keys, kv, swa

    def nbytes(self) -> int:
        return self.keys.nbytes() + self.kv.nbytes() + self.swa.nbytes()


class DecodeStep:
    def __init__(self, caches: Sequence[LayerCache], B: int, H: int, N: int, k: int, swa_len: int, scale: float,
                 q_dtype=torch.bfloat16, device="cuda", pdl: bool = True, stats: bool = True):
        self.caches = list(caches)
        self.L, self.B, self.H, self.N, self.k, self.swa_len, self.scale = len(caches), B, H, N, k, swa_len, scale
        L = self.L
        dev = torch.device(device)
        self.q_idx = torch.zeros((L, B, 1, H, 128), dtype=q_dtype, device=dev)
        self.w = torch.zeros((L, B, 1, H), dtype=torch.float32, device=dev)
        self.q_attn = torch.zeros((L, B, H, 512), dtype=q_dtype, device=dev)
        self.scores = torch.zeros((L, B, 1, N), dtype=torch.float32, device=dev)
        self.ids = torch.zeros((L, B, 1, k), dtype=torch.int32, device=dev)
        self.n_sel = torch.zeros((L, B, 1), dtype=torch.int32, device=dev)
        self.out = torch.zeros((L, B, H, 512), dtype=torch.float32, device=dev)
        self.lse = torch.zeros((L, B, H), dtype=torch.float32, device=dev)
        # score bounds per span of entries (scorer -> top-k): the top-k reads
        # the row's range instead of exchanging it among its CTAs
        n_spans = (N + STATS_SPAN - 1) // STATS_SPAN
        self.tile_stats = torch.zeros((L, B, 1, n_spans, 2), dtype=torch.int32, device=dev) if stats else None
        self._lib = lib()
        self._score, self._topk, self._attn, self._ws_topk, self._ws_attn = [], [], [], [], []
        # Programmatic dependent launch: each kernel may start while the previous
        # one finishes; it prefetches only cache-side data (keys, rows, window,
        # attention queries) before waiting, which nothing in the step writes.
        flags = LAUNCH_PDL if pdl else 0
        for l, c in enumerate(self.caches):
            qd = BF16 if q_dtype == torch.bfloat16 else 0
            ts = self.tile_stats[l] if stats else None
            sa = ScoreArgs(B, 1, H, N, qd, self.q_idx[l].data_ptr(), self.w[l].data_ptr(), c.keys.args(),
                           self.scores[l].data_ptr(), N, flags, 0 if ts is None else ts.data_ptr())
            ta = topk_args(self.scores[l], k, None, self.ids[l], self.n_sel[l], flags=flags, tile_stats=ts)
            aa = attn_args(self.q_attn[l], c.kv, N, self.ids[l][:, 0], self.n_sel[l][:, 0], c.swa, swa_len, scale,
                           self.out[l], self.lse[l], flags=flags)
            self._score.append(sa)
            self._topk.append(ta)
            self._attn.append(aa)
            self._ws_topk.append(workspace(workspace_size(OP_TOPK, ta), dev))
            self._ws_attn.append(workspace(workspace_size(OP_ATTN, aa), dev))
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    # ------------------------------------------------------------------ run
    def enqueue(self, stream=None, events: Optional[List] = None):
        """Issue the step's library calls on `stream`.  With `events` (per layer
        a dict mapping "score", "topk" or "attn" to a (start, end) pair of
        external CUDA events), bracket those calls for timing."""
        st = C.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
        lb = self._lib

        def call(l, name, fn, *a):
            ev = events[l].get(name) if events is not None else None
            if ev is not None:
                ev[0].record()
            rc = fn(*a)
            if ev is not None:
                ev[1].record()
            if rc:
                raise LidxError(rc, fn.__name__)

        for l in range(self.L):
            call(l, "score", lb.lidx_index_score, C.byref(self._score[l]), st)
            wt = self._ws_topk[l]
            call(l, "topk", lb.lidx_topk_select, C.byref(self._topk[l]), C.c_void_p(wt.data_ptr()), wt.numel(), st)
            wa = self._ws_attn[l]
            call(l, "attn", lb.lidx_sparse_attn_decode, C.byref(self._attn[l]), C.c_void_p(wa.data_ptr()), wa.numel(),
                 st)

    def capture(self, events: Optional[List] = None) -> torch.cuda.CUDAGraph:
        """Record one step into a CUDA graph (the library calls only)."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.enqueue(s)  # warm the launch paths outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.enqueue(torch.cuda.current_stream(), events)
        if events is None:
            self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def set_inputs(self, q_idx, w, q_attn, non_blocking=True):
        """Copy one step's queries and head weights (host pinned or device)."""
        self.q_idx.copy_(q_idx, non_blocking=non_blocking)
        self.w.copy_(w, non_blocking=non_blocking)
        self.q_attn.copy_(q_attn, non_blocking=non_blocking)

    def kernel_launches(self) -> int:
        """Kernels one step launches: per layer 1 scorer, 1 top-k, attention + merge."""
        return self.L * 4

    def cache_bytes(self) -> int:
        return sum(c.nbytes() for c in self.caches)
