"""Shared helpers of the GPU parity tests: move synthetic inputs to the device
and apply the parity rules.

Tolerances (fp32 accumulation of exact bf16 / E4M3 products):
  scores     |g - o| <= 1e-5 |o| + 1e-6 * sum_h |w_h| |q_h . k_j|
             (1e-5 relative; the absolute term only keeps the bar finite
             where the head terms cancel to near zero)
  attention  max_d |g - o| / max_d |o| <= 2e-3 per (b, h)
  sets       bit-exact on identical inputs; end to end, differences only for
             entries tied with the k-th score within 1e-6 relative
"""
import numpy as np
import torch

import lightning_indexer_top_index_b200 as L

SCORE_RTOL = 1e-5
SCORE_CTOL = 1e-6
ATTN_TOL = 2e-3


def dev_kv(kv, batch_rows=0):
    """synth.KV -> DeviceKV on cuda:0."""
    return L.DeviceKV.from_arrays(kv.dtype, kv.dim, kv.data, kv.scale, kv.rope, batch_rows=batch_rows)


def dev_q(q, dtype):
    """float32 array or bf16 bits -> torch tensor on cuda:0."""
    t = torch.from_numpy(np.ascontiguousarray(q))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda().contiguous()


def score_rel_err(got, ref):
    """Largest |g - o| / |o| over the entries with |o| > 1e-3 max |o| (the
    relative error away from the near-zero scores)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    big = np.abs(ref) > 1e-3 * np.abs(ref).max()
    if not big.any():
        return 0.0
    return float((np.abs(got - ref)[big] / np.abs(ref)[big]).max())


def assert_scores_close(got, ref, cond):
    """Element-wise score check; returns (and prints) score_rel_err."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    bound = SCORE_RTOL * np.abs(ref) + SCORE_CTOL * cond
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} scores outside tolerance; worst err {err.max():.3e} "
                           f"bound there {bound.ravel()[np.argmax(err)]:.3e}")
    rel = score_rel_err(got, ref)
    print(f"score max rel err {rel:.3e} over {ref.size} entries")
    return rel


def assert_attn_close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    rel = num / den
    assert rel.max() <= ATTN_TOL, f"max relative error {rel.max():.3e}"
    return rel.max()


def topk_sets_equivalent(ids_gpu, ids_ref, scores_ref, bound=None, rtol=1e-6):
    """End-to-end set check: every entry in the symmetric difference must tie
    with the k-th selected oracle score, within rtol relative plus the score
    tolerance `bound` (per entry) of both entries."""
    a = set(int(i) for i in ids_gpu if i >= 0)
    b = set(int(i) for i in ids_ref if i >= 0)
    if a == b:
        return True
    if len(a) != len(b):
        return False
    sel = np.array(sorted(b))
    jk = sel[np.argmin(scores_ref[sel])]
    kth = float(scores_ref[jk])
    for j in a ^ b:
        slack = rtol * abs(kth)
        if bound is not None:
            slack += float(bound[j]) + float(bound[jk])
        if abs(float(scores_ref[j]) - kth) > slack:
            return False
    return True


def score_bound(ref, cond):
    return SCORE_RTOL * np.abs(np.asarray(ref, dtype=np.float64)) + SCORE_CTOL * cond


def graph_kernel_count(enqueue):
    """Kernels one call of `enqueue(stream)` launches: the call is captured
    into a CUDA graph (after one warm call outside capture) and the graph's
    kernel nodes are counted."""
    from cuda.bindings import runtime as rt

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        enqueue(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g):
        enqueue(torch.cuda.current_stream())
    raw = rt.cudaGraph_t(init_value=int(g.raw_cuda_graph()))
    err, _, n = rt.cudaGraphGetNodes(raw, 0)
    assert err == rt.cudaError_t.cudaSuccess, err
    err, nodes, n = rt.cudaGraphGetNodes(raw, n)
    assert err == rt.cudaError_t.cudaSuccess, err
    kinds = [rt.cudaGraphNodeGetType(x)[1] for x in nodes[:n]]
    count = sum(k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel for k in kinds)
    torch.cuda.synchronize()
    del g
    return count
