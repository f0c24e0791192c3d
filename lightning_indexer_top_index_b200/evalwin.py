"""Selection evaluation over one tau-window, as the FlashMemory comparison
computes it (FlashMemory deep-dive write-up, sections 2.2, 3.2 and 4.1;
FlashMemory-vs-native post, Acts 1 and 3), on the library's calls:

  per layer     native index scores of the window's T queries and their
                top-k (the native selection)
  all layers    golden dense-attention probabilities (or, with
                golden="index", the softmax of the native index scores: the
                write-up's step 1 read as a softmax of the indexer logits),
                their top-p sets and the golden top-k
  window        the >= min_votes layer vote per query and its union G
  gate          the gate's logits at its layers (the index scorer with the
                gate query and signed head weights) and the fetched set F
  fetched top-k the native top-k inside F (the tiering of the comparison:
                the native indexer keeps its top-k among the entries the gate
                fetched; FlashMemory-vs-native post, "The setup"; write-up,
                reply #2)
  overlap       |A & B|, |A|, |B| for native vs golden top-k (per layer and
                query), native top-k vs F (per layer and query), G vs F, and
                the top-k inside F vs the golden top-k and vs the unrestricted
                native top-k (per layer and query)

The window owns its buffers and workspaces; `enqueue` only issues the calls.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import torch

from . import (DeviceKV, EVAL_GOLDEN, EVAL_GOLDEN_INDEX, EVAL_LSA, EVAL_OVERLAP, EVAL_TOPP, EVAL_VOTE, OP_EVAL, OP_TOPK, EvalArgs,
               index_score, selection_eval, topk_args, topk_select, workspace, workspace_size, KVArgs, BF16)


class EvalWindow:
    def __init__(self, keys: Sequence[DeviceKV], kv_all: DeviceKV, q_idx: torch.Tensor, w: torch.Tensor,
                 qa: torch.Tensor, gate_q: torch.Tensor, gate_u: torch.Tensor, gate_layers: Sequence[int], N: int,
                 k: int = 512, top_p=(3, 5), min_votes: int = 3, scale: Optional[float] = None,
                 golden: str = "attention"):
        """keys: per layer the index keys (dim 128); kv_all: every layer's
        attention rows, layer l at rows [l*batch_rows, l*batch_rows + N);
        q_idx [L][T][H][128], w [L][T][H], qa [L][T][H][512] (bf16);
        gate_q [G][H][128], gate_u [G][H] for the gate layers.  golden:
        "attention" (dense attention probabilities) or "index" (the softmax
        of the native index scores)."""
        if golden not in ("attention", "index"):
            raise ValueError(golden)
        self.golden = golden
        self.keys, self.kv_all = list(keys), kv_all
        self.L, self.T, self.H = q_idx.shape[0], q_idx.shape[1], q_idx.shape[2]
        self.N, self.k, self.top_p, self.min_votes = N, k, top_p, min_votes
        self.scale = 512 ** -0.5 if scale is None else scale
        self.gate_layers = list(gate_layers)
        dev = q_idx.device
        L, T, H = self.L, self.T, self.H
        W = (N + 31) // 32
        self.W = W
        self.q_idx, self.w, self.qa = q_idx, w, qa
        self.gate_q = gate_q.reshape(len(self.gate_layers), 1, 1, H, 128)
        self.gate_u = gate_u.reshape(len(self.gate_layers), 1, 1, H)
        self.scores = torch.empty((L, 1, T, N), dtype=torch.float32, device=dev)
        self.nat_ids = torch.empty((L, 1, T, k), dtype=torch.int32, device=dev)
        self.nat_n = torch.empty((L, 1, T), dtype=torch.int32, device=dev)
        self.nat_bits = torch.zeros((L, 1, T, W), dtype=torch.int32, device=dev)
        self.probs = torch.empty((L, T, N), dtype=torch.float32, device=dev)
        self.gold_ids = torch.empty((L * T, 1, k), dtype=torch.int32, device=dev)
        self.gold_n = torch.empty((L * T, 1), dtype=torch.int32, device=dev)
        self.gold_bits = torch.zeros((L * T, 1, W), dtype=torch.int32, device=dev)
        self.topp_bits = torch.zeros((L, T, W), dtype=torch.int32, device=dev)
        self.vote_bits = torch.zeros((T, W), dtype=torch.int32, device=dev)
        self.window_bits = torch.zeros((W,), dtype=torch.int32, device=dev)
        self.gate_logits = torch.empty((len(self.gate_layers), 1, 1, N), dtype=torch.float32, device=dev)
        self.fetched_bits = torch.zeros((W,), dtype=torch.int32, device=dev)
        self.counts_nat_gold = torch.zeros((L * T, 3), dtype=torch.int64, device=dev)
        self.counts_nat_f = torch.zeros((L * T, 3), dtype=torch.int64, device=dev)
        self.counts_g_f = torch.zeros((1, 3), dtype=torch.int64, device=dev)
        self.natf_ids = torch.empty((L, 1, T, k), dtype=torch.int32, device=dev)
        self.natf_n = torch.empty((L, 1, T), dtype=torch.int32, device=dev)
        self.natf_bits = torch.zeros((L, 1, T, W), dtype=torch.int32, device=dev)
        self.counts_natf_gold = torch.zeros((L * T, 3), dtype=torch.int64, device=dev)
        self.counts_natf_nat = torch.zeros((L * T, 3), dtype=torch.int64, device=dev)
        # workspaces sized once
        ta = topk_args(self.scores[0], k, None, self.nat_ids[0], self.nat_n[0], None, self.nat_bits[0])
        self.ws_topk_nat = workspace(workspace_size(OP_TOPK, ta), dev)
        tg = topk_args(self.probs.view(L * T, 1, N), k, None, self.gold_ids, self.gold_n, None, self.gold_bits)
        self.ws_topk_gold = workspace(workspace_size(OP_TOPK, tg), dev)
        ea = EvalArgs(EVAL_GOLDEN | EVAL_TOPP, L, T, H, N, BF16, qa.data_ptr(), kv_all.args(), float(self.scale),
                      self.probs.data_ptr(), top_p[0], top_p[1], self.topp_bits.data_ptr())
        self.ws_golden = workspace(workspace_size(OP_EVAL, ea), dev)
        self.ws_small = workspace(1 << 20, dev)

    # ------------------------------------------------------------------ run
    def enqueue(self, stream=None, events: Optional[Dict] = None):
        """Issue the window's calls on `stream` (default: current).  With
        `events` (name -> (start, end) CUDA events) the stages "score",
        "topk", "golden", "topp", "gold_topk", "vote", "gate", "fetched_topk"
        and "overlap" are bracketed for timing."""
        L, T, H, N, k = self.L, self.T, self.H, self.N, self.k
        st = stream or torch.cuda.current_stream()

        def mark(name, i):
            if events is not None and name in events:
                events[name][i].record(st)

        mark("score", 0)
        for l in range(L):
            index_score(self.q_idx[l].unsqueeze(0), self.w[l].unsqueeze(0), self.keys[l], N,
                        scores=self.scores[l], stream=st)
        mark("score", 1)
        mark("topk", 0)
        for l in range(L):
            topk_select(self.scores[l], k, want_bits=True, ids=self.nat_ids[l], n_sel=self.nat_n[l],
                        bits=self.nat_bits[l], ws=self.ws_topk_nat, stream=st)
        mark("topk", 1)
        mark("golden", 0)
        if self.golden == "index":
            selection_eval(EVAL_GOLDEN_INDEX, L=L, T=T, N=N, index_scores=self.scores.view(L * T, N),
                           probs=self.probs, ws=self.ws_small, stream=st)
        else:
            selection_eval(EVAL_GOLDEN, L=L, T=T, H=H, N=N, qa=self.qa, kv=self.kv_all, scale=self.scale,
                           probs=self.probs, ws=self.ws_golden, stream=st)
        mark("golden", 1)
        mark("topp", 0)
        selection_eval(EVAL_TOPP, L=L, T=T, N=N, probs=self.probs, top_p=self.top_p, topp_bits=self.topp_bits,
                       ws=self.ws_small, stream=st)
        mark("topp", 1)
        mark("gold_topk", 0)
        topk_select(self.probs.view(L * T, 1, N), k, want_bits=True, ids=self.gold_ids, n_sel=self.gold_n,
                    bits=self.gold_bits, ws=self.ws_topk_gold, stream=st)
        mark("gold_topk", 1)
        mark("vote", 0)
        selection_eval(EVAL_VOTE, L=L, T=T, N=N, topp_bits=self.topp_bits, min_votes=self.min_votes,
                       vote_bits=self.vote_bits, window_bits=self.window_bits, ws=self.ws_small, stream=st)
        mark("vote", 1)
        mark("gate", 0)
        for i, gl in enumerate(self.gate_layers):
            index_score(self.gate_q[i], self.gate_u[i], self.keys[gl], N, scores=self.gate_logits[i], stream=st)
        selection_eval(EVAL_LSA, N=N, gate_logits=self.gate_logits.view(-1, N), fetched_bits=self.fetched_bits,
                       ws=self.ws_small, stream=st)
        mark("gate", 1)
        mark("fetched_topk", 0)
        fb = self.fetched_bits.view(1, self.W)
        for l in range(L):
            topk_select(self.scores[l], k, want_bits=True, ids=self.natf_ids[l], n_sel=self.natf_n[l],
                        bits=self.natf_bits[l], ws=self.ws_topk_nat, stream=st, allowed_bits=fb)
        mark("fetched_topk", 1)
        mark("overlap", 0)
        W = self.W
        selection_eval(EVAL_OVERLAP, N=N, set_a=self.nat_bits.view(L * T, W), set_b=self.gold_bits.view(L * T, W),
                       n_pairs=L * T, counts=self.counts_nat_gold, ws=self.ws_small, stream=st)
        selection_eval(EVAL_OVERLAP, N=N, set_a=self.nat_bits.view(L * T, W), set_b=self.fetched_bits, ld_b=0,
                       n_pairs=L * T, counts=self.counts_nat_f, ws=self.ws_small, stream=st)
        selection_eval(EVAL_OVERLAP, N=N, set_a=self.window_bits, set_b=self.fetched_bits, ld_a=0, ld_b=0,
                       n_pairs=1, counts=self.counts_g_f, ws=self.ws_small, stream=st)
        selection_eval(EVAL_OVERLAP, N=N, set_a=self.natf_bits.view(L * T, W), set_b=self.gold_bits.view(L * T, W),
                       n_pairs=L * T, counts=self.counts_natf_gold, ws=self.ws_small, stream=st)
        selection_eval(EVAL_OVERLAP, N=N, set_a=self.natf_bits.view(L * T, W), set_b=self.nat_bits.view(L * T, W),
                       n_pairs=L * T, counts=self.counts_natf_nat, ws=self.ws_small, stream=st)
        mark("overlap", 1)

    def kernel_launches(self) -> int:
        """Kernels one window launches: per layer a scorer, a top-k and a
        top-k inside the fetched set, the golden probabilities (two
        tensor-core passes around the lse merge on the tcgen05 path, else the
        lse and probability kernels), top-p, the golden top-k, the vote and
        its union, a scorer per gate layer and the gate OR, and five overlap
        counts."""
        golden = 3 if self.H == 64 and self.qa.dtype == torch.bfloat16 and self.kv_all.dtype == BF16 else 2
        return 3 * self.L + golden + 1 + 1 + 2 + len(self.gate_layers) + 1 + 5

    def golden_flops(self) -> float:
        """Tensor FLOPs of the golden passes: two GEMMs of (T*H) x N x 512 per layer."""
        return 2.0 * self.L * 2.0 * self.T * self.H * self.N * 512

    def score_flops(self) -> float:
        return self.L * 2.0 * self.T * self.H * self.N * 128
