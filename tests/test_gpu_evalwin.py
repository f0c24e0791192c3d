"""The tau-window evaluation pipeline (EvalWindow) as the eval-window bench
runs it, at a size the oracle finishes in seconds: every stage against the
oracle on the GPU's own upstream outputs (bit-exact for sets and counts,
the score and probability tolerances elsewhere)."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import assert_scores_close, dev_kv, dev_q, graph_kernel_count
from lightning_indexer_top_index_b200.evalwin import EvalWindow

pytestmark = pytest.mark.gpu


def _window(spec, golden="attention"):
    layers = [synth.eval_layer(spec, l) for l in range(spec.L)]
    gate = synth.eval_gate(spec)
    keys = [dev_kv(x["keys"], batch_rows=spec.N) for x in layers]
    kv_all = dev_kv(synth.concat_kv([x["kv"] for x in layers]), batch_rows=spec.N)
    q_idx = torch.stack([dev_q(x["q_idx"], "bf16") for x in layers])
    w = torch.stack([torch.from_numpy(x["w"]).cuda() for x in layers])
    qa = torch.stack([dev_q(x["qa"], "bf16") for x in layers])
    win = EvalWindow(keys, kv_all, q_idx, w, qa, dev_q(gate["g"], "bf16"), torch.from_numpy(gate["u"]).cuda(),
                     spec.gate_layers, spec.N, spec.k, (spec.top_p_num, spec.top_p_den), spec.min_votes, spec.scale,
                     golden=golden)
    return layers, gate, win


def test_eval_window_kernel_count(cuda_device):
    spec = synth.scaled(synth.EVAL_WINDOW, L=4, T=3, N=1100, k=64, gate_layers=(0, 1, 3))
    _, _, win = _window(spec)
    assert graph_kernel_count(win.enqueue) == win.kernel_launches()


def test_eval_window_against_oracle(cuda_device):
    spec = synth.scaled(synth.EVAL_WINDOW, L=4, T=3, N=1100, k=64, gate_layers=(0, 1, 3))
    layers, gate, win = _window(spec)
    win.enqueue()
    win.enqueue()  # a second window on the same buffers
    torch.cuda.synchronize()
    N, T, Lq, W = spec.N, spec.T, spec.L, (spec.N + 31) // 32
    scores = win.scores.cpu().numpy()
    probs = win.probs.cpu().numpy()
    nat_bits = win.nat_bits.cpu().numpy().view(np.uint32).reshape(Lq, T, W)
    gold_bits = win.gold_bits.cpu().numpy().view(np.uint32).reshape(Lq, T, W)
    topp_bits = win.topp_bits.cpu().numpy().view(np.uint32)
    window_bits = win.window_bits.cpu().numpy().view(np.uint32)
    fetched = win.fetched_bits.cpu().numpy().view(np.uint32)
    for l, x in enumerate(layers):
        ref, cond = oracle.index_score(x["q_idx"].reshape(1, T, spec.H, 128), x["w"].reshape(1, T, spec.H),
                                       x["keys"], 1, T, spec.H, N, want_cond=True)
        assert_scores_close(scores[l], ref, cond)
        np.testing.assert_allclose(probs[l], oracle.golden(x["qa"], x["kv"], T, spec.H, N, spec.scale),
                                   rtol=1e-4, atol=1e-10)
        for t in range(T):
            ids, n, _ = oracle.topk(scores[l, 0, t], spec.k)
            dense = np.zeros(N, bool)
            dense[ids[:n]] = True
            assert np.array_equal(nat_bits[l, t], synth.pack_bits(dense)[0])
            ids, n, _ = oracle.topk(probs[l, t], spec.k)
            dense = np.zeros(N, bool)
            dense[ids[:n]] = True
            assert np.array_equal(gold_bits[l, t], synth.pack_bits(dense)[0])
            assert np.array_equal(topp_bits[l, t], oracle.topp(probs[l, t])[0])
    votes = [oracle.vote(topp_bits[:, t], N, spec.min_votes) for t in range(T)]
    assert np.array_equal(window_bits, oracle.union(np.stack(votes), N))
    logits = win.gate_logits.cpu().numpy().reshape(len(spec.gate_layers), N)
    for i, gl in enumerate(spec.gate_layers):
        ref, cond = oracle.index_score(gate["g"][i].reshape(1, 1, spec.H, 128), gate["u"][i].reshape(1, 1, spec.H),
                                       layers[gl]["keys"], 1, 1, spec.H, N, want_cond=True)
        assert_scores_close(logits[i], ref[0, 0], cond[0, 0])
    assert np.array_equal(fetched, oracle.lsa_gate(logits))
    c_ng = win.counts_nat_gold.cpu().numpy()
    c_nf = win.counts_nat_f.cpu().numpy()
    for l in range(Lq):
        for t in range(T):
            assert tuple(c_ng[l * T + t]) == oracle.overlap(nat_bits[l, t], gold_bits[l, t], N)
            assert tuple(c_nf[l * T + t]) == oracle.overlap(nat_bits[l, t], fetched, N)
    assert tuple(win.counts_g_f.cpu().numpy()[0]) == oracle.overlap(window_bits, fetched, N)
    # the native top-k inside the fetched set, and its overlaps
    natf_bits = win.natf_bits.cpu().numpy().view(np.uint32).reshape(Lq, T, W)
    natf_ids = win.natf_ids.cpu().numpy().reshape(Lq, T, spec.k)
    natf_n = win.natf_n.cpu().numpy().reshape(Lq, T)
    allowed = synth.unpack_bits(fetched[None], N)[0].astype(np.uint8)
    assert 0 < allowed.sum() < N  # the gate neither fetched nothing nor everything
    c_fg = win.counts_natf_gold.cpu().numpy()
    c_fn = win.counts_natf_nat.cpu().numpy()
    for l in range(Lq):
        for t in range(T):
            ids, n, _ = oracle.topk(scores[l, 0, t], spec.k, allowed)
            assert natf_n[l, t] == n and np.array_equal(natf_ids[l, t], ids)
            dense = np.zeros(N, bool)
            dense[ids[:n]] = True
            assert np.array_equal(natf_bits[l, t], synth.pack_bits(dense)[0])
            assert tuple(c_fg[l * T + t]) == oracle.overlap(natf_bits[l, t], gold_bits[l, t], N)
            assert tuple(c_fn[l * T + t]) == oracle.overlap(natf_bits[l, t], nat_bits[l, t], N)


def test_eval_window_golden_from_index_logits(cuda_device):
    """golden="index": the golden probabilities are the softmax of the
    window's native index scores (the write-up's step 1 read as a softmax of
    the indexer logits).  Against the oracle on the GPU's own scores, and the
    top-p sets and vote bit-exact on the GPU's own probabilities."""
    spec = synth.scaled(synth.EVAL_WINDOW, L=3, T=2, N=1500, k=64, gate_layers=(0, 1, 2))
    _, _, win = _window(spec, golden="index")
    win.enqueue()
    torch.cuda.synchronize()
    N, T, Lq, W = spec.N, spec.T, spec.L, (spec.N + 31) // 32
    scores = win.scores.cpu().numpy().reshape(Lq, T, N)
    probs = win.probs.cpu().numpy()
    np.testing.assert_allclose(probs, oracle.golden_index(scores), rtol=2e-5, atol=1e-30)
    topp_bits = win.topp_bits.cpu().numpy().view(np.uint32)
    for l in range(Lq):
        for t in range(T):
            bits, _ = oracle.topp(probs[l, t], spec.top_p_num, spec.top_p_den)
            assert np.array_equal(topp_bits[l, t], bits)
    assert np.array_equal(win.window_bits.cpu().numpy().view(np.uint32),
                          oracle.union(np.stack([oracle.vote(topp_bits[:, t], N, spec.min_votes) for t in range(T)]), N))
