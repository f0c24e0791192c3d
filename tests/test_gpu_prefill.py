"""The prefill-time indexer (architecture post, section (B): the indexer and
its top-k run for every token, prefill included).  A chunk of T consecutive
prefill tokens at positions p0 .. p0+T-1 scores one shared compressed cache
in one batched call; query t may only see the compressed entries whose four
tokens all lie at or before its own position: n_visible[t] = (p_t + 1) // 4.
Then each query keeps its own top-k among its visible entries and attends
over them plus the 128 raw tokens ending at its position.

Against the oracle run query by query on exactly the visible prefix: scores
within the score tolerance and -inf beyond the prefix, ids bit-exact on the
GPU's own scores, attention within the attention tolerance."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import assert_attn_close, assert_scores_close, dev_kv, dev_q

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,N,T,p0,k", [("bf16", 1024, 64, 3000, 128), ("bf16", 1024, 64, 200, 128),
                                            ("bf16", 4096, 17, 16000, 512), ("f32", 700, 9, 2500, 64)])
def test_prefill_chunk(cuda_device, dtype, N, T, p0, k):
    H, swa = 64 if dtype == "bf16" else 16, 128
    scale = 512 ** -0.5
    g = np.random.default_rng(90 + T)
    # one sequence's compressed cache, T query tokens, the raw-token window rows
    x = synth.decode_layer(synth.scaled(synth.DECODE_64K if dtype == "bf16" else synth.TINY_1K_F32, N=N, H=H,
                                        k=k, swa=p0 + T), 0)
    q = g.standard_normal((T, H, 128)) / np.sqrt(128)
    qs = synth.bf16_bits(q) if dtype == "bf16" else q.astype(np.float32)
    w = g.random((T, H)).astype(np.float32)
    pos = p0 + np.arange(T)
    n_vis = ((pos + 1) // 4).astype(np.int32)
    assert n_vis.max() <= N
    keys = dev_kv(x["keys"])
    nv = torch.from_numpy(n_vis.reshape(1, T)).cuda()
    scores = L.index_score(dev_q(qs.reshape(1, T, H, 128), dtype), torch.from_numpy(w.reshape(1, T, H)).cuda(), keys,
                           N, n_visible=nv)
    ids, n_sel, _, _ = L.topk_select(scores, k, n_valid=nv)
    s_np, ids_np, n_np = scores.cpu().numpy()[0], ids.cpu().numpy()[0], n_sel.cpu().numpy()[0]
    # attention: B = T queries sharing the compressed cache (batch_rows 0);
    # query t's window is raw rows p_t-127 .. p_t (row t of a view starting at p0-127)
    qa = g.standard_normal((T, H, 512))
    qa_st = synth.bf16_bits(qa) if dtype == "bf16" else qa.astype(np.float32)
    kv = dev_kv(x["kv"])
    kv.batch_rows = 0
    win_all = dev_kv(x["swa"])
    w0 = p0 - swa + 1
    win = L.DeviceKV(win_all.dtype, 512, win_all.data[w0:], batch_rows=1)
    out, lse = L.sparse_attn_decode(dev_q(qa_st, dtype), kv, N, ids[0], n_sel[0], win, swa, scale)
    out = out.cpu().numpy()
    for t in range(T):
        nvt = int(n_vis[t])
        ref, cond = oracle.index_score(qs[t].reshape(1, 1, H, 128), w[t], x["keys"].slice(0, nvt), 1, 1, H, nvt,
                                       want_cond=True)
        assert_scores_close(s_np[t, :nvt], ref[0, 0], cond[0, 0])
        assert np.all(np.isneginf(s_np[t, nvt:])), "entries beyond the causal prefix must score -inf"
        rid, rn, _ = oracle.topk(s_np[t, :nvt], k)
        assert n_np[t] == rn == min(k, nvt) and np.array_equal(ids_np[t], rid), f"query {t}"
        ro, rl = oracle.attn(qa_st[t], x["kv"], N, rid[:rn], swa=x["swa"].slice(pos[t] - swa + 1, pos[t] + 1),
                             swa_len=swa, scale=scale)
        assert_attn_close(out[t], ro)
