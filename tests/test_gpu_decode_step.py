"""The multi-layer decode step as the benchmark runs it (CUDA graph, PDL
launches, rotating buffers): every layer's outputs against the oracle chain.
Scores within the score tolerance, top-k sets equal up to near-ties, attention
within 2e-3 of the oracle run on the GPU's own selection."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import assert_attn_close, assert_scores_close, graph_kernel_count, score_bound, topk_sets_equivalent
from lightning_indexer_top_index_b200.decode import DecodeStep, LayerCache

pytestmark = pytest.mark.gpu


def _step(spec, layers, pdl):
    inp = [synth.decode_layer(spec, l) for l in range(layers)]
    caches = []
    for x in inp:
        caches.append(LayerCache(
            L.DeviceKV.from_arrays(spec.key_dtype, 128, x["keys"].data, x["keys"].scale, x["keys"].rope,
                                   batch_rows=spec.N),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, x["kv"].data, x["kv"].scale, x["kv"].rope, batch_rows=spec.N),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, x["swa"].data, x["swa"].scale, x["swa"].rope,
                                   batch_rows=spec.swa)))
    st = DecodeStep(caches, spec.B, spec.H, spec.N, spec.k, spec.swa, spec.scale, pdl=pdl)

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16)

    st.set_inputs(torch.stack([t(x["q_idx"]) for x in inp]).reshape(layers, spec.B, 1, spec.H, 128).cuda(),
                  torch.stack([torch.from_numpy(x["w"]) for x in inp]).reshape(layers, spec.B, 1, spec.H).cuda(),
                  torch.stack([t(x["q_attn"]) for x in inp]).cuda())
    st.capture()
    for _ in range(3):
        st.replay()
    torch.cuda.synchronize()
    return inp, st


@pytest.mark.parametrize("pdl", [True, False])
def test_decode_step_against_oracle(cuda_device, pdl):
    spec = synth.scaled(synth.DECODE_64K, N=4099, layers=3)
    inp, st = _step(spec, 3, pdl)
    scores, ids, n_sel = st.scores.cpu().numpy(), st.ids.cpu().numpy(), st.n_sel.cpu().numpy()
    out = st.out.cpu().numpy()
    for l, x in enumerate(inp):
        ref, cond = oracle.index_score(x["q_idx"].reshape(1, 1, spec.H, 128), x["w"], x["keys"], 1, 1, spec.H,
                                       spec.N, want_cond=True)
        assert_scores_close(scores[l], ref, cond)
        ref_ids, _, _ = oracle.topk(ref[0, 0], spec.k)
        assert n_sel[l, 0, 0] == spec.k
        assert topk_sets_equivalent(ids[l, 0, 0], ref_ids, ref[0, 0], score_bound(ref[0, 0], cond[0, 0]))
        ro, _ = oracle.attn(x["q_attn"][0], x["kv"], spec.N, ids[l, 0, 0], swa=x["swa"], swa_len=spec.swa,
                            scale=spec.scale)
        assert_attn_close(out[l, 0], ro)


def test_decode_step_fp8_batched(cuda_device):
    spec = synth.scaled(synth.DECODE_500K_FP8, N=5000, B=2, layers=2)
    inp, st = _step(spec, 2, True)
    ids, out = st.ids.cpu().numpy(), st.out.cpu().numpy()
    for l, x in enumerate(inp):
        for b in range(spec.B):
            N = spec.N
            ro, _ = oracle.attn(x["q_attn"][b], x["kv"].slice(b * N, (b + 1) * N), N, ids[l, b, 0],
                                swa=x["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=spec.swa,
                                scale=spec.scale)
            assert_attn_close(out[l, b], ro)


@pytest.mark.parametrize("pdl", [True, False])
def test_decode_step_kernel_count(cuda_device, pdl):
    spec = synth.scaled(synth.DECODE_64K, N=4099, layers=3)
    _, st = _step(spec, 3, pdl)
    assert graph_kernel_count(st.enqueue) == st.kernel_launches()
