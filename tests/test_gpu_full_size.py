"""Parity at the benchmark workloads' full sizes, in the configuration the
bench times: the captured decode step (PDL launches, score bounds) built by
the bench's own helpers, and the evaluation window.  The oracle checks
sampled outputs one by one (whole score rows or row ranges, the attention of
sampled layers and sequences, golden rows of sampled queries); the top-k,
top-p, vote, gate and overlap outputs are checked bit for bit against the
oracle run on the GPU's own upstream outputs, and the planted workload's
top-k against its planted rows."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from _helpers import assert_attn_close, assert_scores_close

pytestmark = pytest.mark.gpu


def _bench_step(spec):
    layers = [synth.decode_layer(spec, l) for l in range(spec.layers)]
    step = bench.make_replica_steps(spec, layers, 1, torch.device("cuda", 0))[0]
    q_idx, w, q_attn = bench.host_queries(spec, layers)
    step.set_inputs(q_idx.cuda(), w.cuda(), q_attn.cuda())
    step.capture()
    for _ in range(3):
        step.replay()
    torch.cuda.synchronize()
    return layers, step


def _check_layer(spec, x, scores, ids, n_sel, out, b, ranges=None):
    """Sequence b of one layer: scores (all, or the given entry ranges) within
    tolerance; ids bit-exact against the oracle's top-k of the GPU's scores;
    attention over the GPU's ids against the oracle."""
    N, H = spec.N, spec.H
    keys = x["keys"].slice(b * N, (b + 1) * N)
    for j0, j1 in ranges or [(0, N)]:
        ref, cond = oracle.index_score(x["q_idx"][b].reshape(1, 1, H, 128), x["w"][b], keys.slice(j0, j1), 1, 1, H,
                                       j1 - j0, want_cond=True)
        assert_scores_close(scores[j0:j1], ref[0, 0], cond[0, 0])
    ref_ids, ref_n, _ = oracle.topk(scores, spec.k)
    assert n_sel == ref_n
    assert np.array_equal(ids, ref_ids)
    ro, _ = oracle.attn(x["q_attn"][b], x["kv"].slice(b * N, (b + 1) * N), N, ids[:n_sel],
                        swa=x["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=spec.swa, scale=spec.scale)
    assert_attn_close(out, ro)


def test_decode_64k_full_step(cuda_device):
    """21 layers x 16384 entries, bf16: three layers checked whole."""
    spec = synth.DECODE_64K
    layers, st = _bench_step(spec)
    scores, ids, n_sel, out = (t.cpu().numpy() for t in (st.scores, st.ids, st.n_sel, st.out))
    for l in (0, 10, 20):
        _check_layer(spec, layers[l], scores[l, 0, 0], ids[l, 0, 0], n_sel[l, 0, 0], out[l, 0], 0)


def test_decode_500k_fp8_full_step(cuda_device):
    """B=4 x 125000 entries, E4M3 keys and rows, top-1024: every sequence's
    top-k and attention; scores on the first and the last 2048 entries (the
    ragged tail tile)."""
    spec = synth.DECODE_500K_FP8
    layers, st = _bench_step(spec)
    scores, ids, n_sel, out = (t.cpu().numpy() for t in (st.scores, st.ids, st.n_sel, st.out))
    N = spec.N
    for b in range(spec.B):
        _check_layer(spec, layers[0], scores[0, b, 0], ids[0, b, 0], n_sel[0, b, 0], out[0, b], b,
                     ranges=[(0, 2048), (N - 2048, N)])


def test_decode_128k_b32_planted_full_step(cuda_device):
    """B=32 x 32768 entries: every sequence's top-512 is its planted set;
    two sequences checked whole."""
    spec = synth.DECODE_128K_B32
    layers, st = _bench_step(spec)
    scores, ids, n_sel, out = (t.cpu().numpy() for t in (st.scores, st.ids, st.n_sel, st.out))
    x = layers[0]
    for b in range(spec.B):
        assert n_sel[0, b, 0] == spec.k
        assert np.array_equal(ids[0, b, 0], x["planted"][b]), f"sequence {b}"
    for b in (0, spec.B - 1):
        _check_layer(spec, x, scores[0, b, 0], ids[0, b, 0], n_sel[0, b, 0], out[0, b], b)


def test_eval_window_full_size(cuda_device):
    """64 queries x 21 layers x 32768 entries: golden rows and native scores of
    sampled (layer, query) pairs against the oracle; every top-p set, the
    vote, the union, the gate and every overlap count bit-exact on the GPU's
    upstream outputs; sampled native and golden top-k bit-exact."""
    import lightning_indexer_top_index_b200 as L
    from lightning_indexer_top_index_b200.evalwin import EvalWindow

    spec = synth.EVAL_WINDOW
    layers, gate = bench.eval_inputs(spec)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16).cuda()

    keys = [L.DeviceKV.from_arrays("bf16", 128, x["keys"].data, batch_rows=spec.N) for x in layers]
    kv_all = L.DeviceKV.from_arrays("bf16", 512, np.concatenate([x["kv"].data for x in layers]), batch_rows=spec.N)
    win = EvalWindow(keys, kv_all, torch.stack([bf(x["q_idx"]) for x in layers]),
                     torch.stack([torch.from_numpy(x["w"]) for x in layers]).cuda(),
                     torch.stack([bf(x["qa"]) for x in layers]), bf(gate["g"]), torch.from_numpy(gate["u"]).cuda(),
                     spec.gate_layers, spec.N, spec.k, (spec.top_p_num, spec.top_p_den), spec.min_votes, spec.scale)
    win.enqueue()
    win.enqueue()
    torch.cuda.synchronize()
    outs = {name: getattr(win, name).cpu().numpy() for name in (
        "scores", "probs", "nat_bits", "gold_bits", "topp_bits", "vote_bits", "window_bits", "gate_logits",
        "fetched_bits", "counts_nat_gold", "counts_nat_f", "counts_g_f")}
    _check_window(spec, layers, outs, samples=((0, 0), (9, 31), (20, 63)))


def _check_window(spec, layers, outs, samples):
    N, T, H, Lq, W = spec.N, spec.T, spec.H, spec.L, (spec.N + 31) // 32
    u32 = lambda a: np.ascontiguousarray(a).view(np.uint32)  # noqa: E731
    scores, probs = outs["scores"], outs["probs"]
    nat_bits = u32(outs["nat_bits"]).reshape(Lq, T, W)
    gold_bits = u32(outs["gold_bits"]).reshape(Lq, T, W)
    topp_bits = u32(outs["topp_bits"]).reshape(Lq, T, W)

    def dense_bits(ids, n):
        d = np.zeros(N, bool)
        d[ids[:n]] = True
        return synth.pack_bits(d)[0]

    for l, t in samples:
        x = layers[l]
        ref, cond = oracle.index_score(x["q_idx"][t].reshape(1, 1, H, 128), x["w"][t], x["keys"], 1, 1, H, N,
                                       want_cond=True)
        assert_scores_close(scores[l, 0, t], ref[0, 0], cond[0, 0])
        np.testing.assert_allclose(probs[l, t], oracle.golden(x["qa"][t:t + 1], x["kv"], 1, H, N, spec.scale)[0],
                                   rtol=1e-4, atol=1e-10)
        ids, n, _ = oracle.topk(scores[l, 0, t], spec.k)
        assert np.array_equal(nat_bits[l, t], dense_bits(ids, n))
        ids, n, _ = oracle.topk(probs[l, t], spec.k)
        assert np.array_equal(gold_bits[l, t], dense_bits(ids, n))
    for l in range(Lq):
        for t in range(T):
            assert np.array_equal(topp_bits[l, t], oracle.topp(probs[l, t])[0]), (l, t)
    votes = np.stack([oracle.vote(topp_bits[:, t], N, spec.min_votes) for t in range(T)])
    assert np.array_equal(u32(outs["vote_bits"]).reshape(T, W), votes)
    window_bits = u32(outs["window_bits"]).reshape(W)
    assert np.array_equal(window_bits, oracle.union(votes, N))
    logits = outs["gate_logits"].reshape(len(spec.gate_layers), N)
    fetched = u32(outs["fetched_bits"]).reshape(W)
    assert np.array_equal(fetched, oracle.lsa_gate(logits))
    c_ng, c_nf = outs["counts_nat_gold"], outs["counts_nat_f"]
    for l in range(Lq):
        for t in range(T):
            assert tuple(c_ng[l * T + t]) == oracle.overlap(nat_bits[l, t], gold_bits[l, t], N)
            assert tuple(c_nf[l * T + t]) == oracle.overlap(nat_bits[l, t], fetched, N)
    assert tuple(outs["counts_g_f"][0]) == oracle.overlap(window_bits, fetched, N)
