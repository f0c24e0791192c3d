"""A decode step over a stack of CSA layers, run as one CUDA graph.

Per layer, in order on one stream (DeepSeek-V4-Flash architecture post,
section (B)): the lightning indexer scores every compressed entry, the top-k
rows are selected, and sparse MQA attention reads those rows plus the
sliding window.  Each layer has its own caches and queries.

Two forms of a layer: `fused` (the default where the library covers the
shape) issues one lidx_decode_layer call, which runs the three steps in one
launch and pulls the next layer's index keys and window rows into L2 while
it runs; otherwise the layer is the three calls lidx_index_score ->
lidx_topk_select -> lidx_sparse_attn_decode.

The step owns its device buffers and prebuilt C-ABI argument structs, so an
enqueue is nothing but the library calls; `capture()` records them into a
CUDA graph that `replay()` launches with one call.
"""
from __future__ import annotations

import ctypes as C
from typing import List, Optional, Sequence

import torch

from . import (AttnArgs, DeviceKV, ScoreArgs, TopkArgs, BF16, LAUNCH_PDL, OP_ATTN, OP_DECODE, OP_SCORE, OP_TOPK,
               STATS_SPAN, ERR_UNSUPPORTED, LidxError, attn_args, decode_args, launch_count, lib, topk_args,
               workspace, workspace_size)


class LayerCache:
    """Device caches of one CSA layer: index keys (dim 128), compressed KV rows
    and sliding-window rows (dim 512), for B sequences."""

    def __init__(self, keys: DeviceKV, kv: DeviceKV, swa: DeviceKV):
        self.keys, self.kv, self.swa = keys, kv, swa

    def nbytes(self) -> int:
        return self.keys.nbytes() + self.kv.nbytes() + self.swa.nbytes()


class DecodeStep:
    def __init__(self, caches: Sequence[LayerCache], B: int, H: int, N: int, k: int, swa_len: int, scale: float,
                 q_dtype=torch.bfloat16, device="cuda", pdl: bool = True, stats: bool = True, fused=None):
        """fused: True forces the one-launch layer (raises where the library
        does not cover the shape), False the three calls, None picks the
        one-launch layer when it is supported."""
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
        # the one-launch form: each layer prefetches the next one's index keys
        # and window rows (cache-side inputs, known before its query)
        self._dec, self._ws_dec = [], []
        self.fused = False
        if fused is not False:
            try:
                for l, c in enumerate(self.caches):
                    pf = ()
                    if l + 1 < L:
                        n = self.caches[l + 1]
                        pf = tuple((t.data_ptr(), t.numel() * t.element_size())
                                   for t in (n.keys.data, n.swa.data))
                    da = decode_args(self.q_idx[l][:, 0], self.w[l][:, 0], c.keys, N, k, self.q_attn[l], c.kv, c.swa,
                                     swa_len, scale, self.out[l], self.lse[l], scores=self.scores[l][:, 0],
                                     ids=self.ids[l][:, 0], n_sel=self.n_sel[l][:, 0], prefetch=pf, flags=flags)
                    self._ws_dec.append(workspace(workspace_size(OP_DECODE, da), dev))
                    self._dec.append(da)
                self.fused = True
            except LidxError as e:
                if fused or e.status != ERR_UNSUPPORTED:
                    raise
                self._dec, self._ws_dec = [], []
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    # ------------------------------------------------------------------ run
    def enqueue(self, stream=None, events: Optional[List] = None):
        """Issue the step's library calls on `stream`.  With `events` (per layer
        a dict mapping "score", "topk", "attn" or, in the one-launch form,
        "layer" to a (start, end) pair of external CUDA events), bracket those
        calls for timing."""
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

        if self.fused:
            for l in range(self.L):
                wd = self._ws_dec[l]
                call(l, "layer", lb.lidx_decode_layer, C.byref(self._dec[l]), C.c_void_p(wd.data_ptr()), wd.numel(),
                     st)
            return
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
        """Kernels one step launches, as the library reports them: per layer
        one fused kernel, or the scorer, the top-k and the attention's split
        and merge kernels."""
        if self.fused:
            return self.L
        return sum(launch_count(OP_SCORE, self._score[l]) + launch_count(OP_TOPK, self._topk[l]) +
                   launch_count(OP_ATTN, self._attn[l]) for l in range(self.L))

    def workspaces(self):
        """The workspaces whose status words the step's calls report into."""
        return self._ws_dec if self.fused else self._ws_topk + self._ws_attn

    def cache_bytes(self) -> int:
        return sum(c.nbytes() for c in self.caches)


SWA, CSA, HCA = "swa", "csa", "hca"


def model_schedule(n_layers: int = 43):
    """Attention kind of every model layer (architecture post, section (A)):
    layers 0-1 attend over the sliding window only, even layers 2-42 are CSA
    layers (4:1 compression, indexer top-k) and odd layers 3-41 are HCA
    layers (128:1 compression, every entry read)."""
    return [SWA if l < 2 else CSA if l % 2 == 0 else HCA for l in range(n_layers)]


class ModelStep:
    """Attention of one decode token through every layer of the hybrid
    schedule, in model order on one stream, as one CUDA graph.

    CSA layers run the one-launch layer (scores, top-k, sparse attention)
    and pull the next CSA layer's index keys and the next HCA layer's rows
    into L2; HCA layers attend over all of their compressed rows and the
    window (lidx_sparse_attn_decode without ids); SWA layers attend over the
    window alone.  csa / hca / swa_only: the caches of those layers in model
    order (LayerCache for CSA; (rows, window) DeviceKV pairs for HCA; window
    DeviceKV for SWA)."""

    def __init__(self, csa: Sequence[LayerCache], hca: Sequence, swa_only: Sequence[DeviceKV], B: int, H: int,
                 N_csa: int, N_hca: int, k: int, swa_len: int, scale: float, device="cuda", pdl: bool = True):
        self.kinds = model_schedule(len(csa) + len(hca) + len(swa_only))
        assert self.kinds.count(CSA) == len(csa) and self.kinds.count(HCA) == len(hca)
        # the argument structs hold raw device pointers: keep every cache they
        # point into alive for as long as the step (and its graph) exists
        self.hca_caches, self.swa_caches = list(hca), list(swa_only)
        dev = torch.device(device)
        self.B, self.H = B, H
        self.csa = DecodeStep(csa, B, H, N_csa, k, swa_len, scale, device=device, pdl=pdl, fused=True)
        nl = len(self.kinds)
        self.q_attn = torch.zeros((nl, B, H, 512), dtype=torch.bfloat16, device=dev)
        self.out = torch.zeros((nl, B, H, 512), dtype=torch.float32, device=dev)
        flags = LAUNCH_PDL if pdl else 0
        self._calls = []  # (kind, index into that kind's list, args, workspace)
        ci = hi = si = 0
        self._csa_layer = []
        for l, kind in enumerate(self.kinds):
            if kind == CSA:
                self._csa_layer.append(l)
                self._calls.append((CSA, ci, None, None))
                ci += 1
                continue
            if kind == HCA:
                rows, win = hca[hi]
                a = attn_args(self.q_attn[l], rows, N_hca, None, None, win, swa_len, scale, self.out[l], None,
                              flags=flags, n_dense=N_hca)
                hi += 1
            else:
                win = swa_only[si]
                a = attn_args(self.q_attn[l], win, 1, None, None, win, swa_len, scale, self.out[l], None,
                              flags=flags)
                si += 1
            self._calls.append((kind, l, a, workspace(workspace_size(OP_ATTN, a), dev)))
        # CSA layer i prefetches CSA layer i+1's keys (set by DecodeStep) and
        # the rows of the HCA layer that follows it
        for i, l in enumerate(self._csa_layer):
            if l + 1 < nl and self.kinds[l + 1] == HCA:
                rows = hca[(l + 1 - 3) // 2][0].data
                self.csa._dec[i].prefetch[1] = rows.data_ptr()
                self.csa._dec[i].prefetch_bytes[1] = rows.numel() * rows.element_size()
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    def set_inputs(self, q_idx, w, q_attn, non_blocking=True):
        """q_idx [21][B][1][H][128], w [21][B][1][H] for the CSA layers;
        q_attn [43][B][H][512] for every layer."""
        self.csa.q_idx.copy_(q_idx, non_blocking=non_blocking)
        self.csa.w.copy_(w, non_blocking=non_blocking)
        self.q_attn.copy_(q_attn, non_blocking=non_blocking)
        self.csa.q_attn.copy_(self.q_attn[self._csa_layer], non_blocking=non_blocking)

    def enqueue(self, stream=None):
        st = C.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
        lb = lib()
        for kind, i, a, ws in self._calls:
            if kind == CSA:
                wd = self.csa._ws_dec[i]
                rc = lb.lidx_decode_layer(C.byref(self.csa._dec[i]), C.c_void_p(wd.data_ptr()), wd.numel(), st)
                name = "lidx_decode_layer"
            else:
                rc = lb.lidx_sparse_attn_decode(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), st)
                name = "lidx_sparse_attn_decode"
            if rc:
                raise LidxError(rc, name)

    def capture(self) -> torch.cuda.CUDAGraph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.enqueue(s)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.enqueue(torch.cuda.current_stream())
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def outputs(self) -> torch.Tensor:
        """Attention outputs of every layer [43][B][H][512] (the CSA layers'
        gathered from the CSA step)."""
        o = self.out.clone()
        o[self._csa_layer] = self.csa.out
        return o

    def kernel_launches(self) -> int:
        """The CSA step's kernels plus the attention kernels of every HCA and
        SWA layer (as the library reports them)."""
        return self.csa.kernel_launches() + sum(launch_count(OP_ATTN, a) for _, _, a, _ in self._calls
                                                 if a is not None)

    def workspaces(self):
        return self.csa.workspaces() + [ws for _, _, _, ws in self._calls if ws is not None]
