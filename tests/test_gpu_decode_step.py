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


def _step(spec, layers, pdl, fused=None):
    inp = [synth.decode_layer(spec, l) for l in range(layers)]
    caches = []
    for x in inp:
        caches.append(LayerCache(
            L.DeviceKV.from_arrays(spec.key_dtype, 128, x["keys"].data, x["keys"].scale, x["keys"].rope,
                                   batch_rows=spec.N),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, x["kv"].data, x["kv"].scale, x["kv"].rope, batch_rows=spec.N),
            L.DeviceKV.from_arrays(spec.kv_dtype, 512, x["swa"].data, x["swa"].scale, x["swa"].rope,
                                   batch_rows=spec.swa)))
    st = DecodeStep(caches, spec.B, spec.H, spec.N, spec.k, spec.swa, spec.scale, pdl=pdl, fused=fused)

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
@pytest.mark.parametrize("fused", [True, False])
def test_decode_step_against_oracle(cuda_device, pdl, fused):
    spec = synth.scaled(synth.DECODE_64K, N=4099, layers=3)
    inp, st = _step(spec, 3, pdl, fused)
    assert st.fused == fused
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
    assert not st.fused  # E4M3 caches take the three calls
    ids, out = st.ids.cpu().numpy(), st.out.cpu().numpy()
    for l, x in enumerate(inp):
        for b in range(spec.B):
            N = spec.N
            ro, _ = oracle.attn(x["q_attn"][b], x["kv"].slice(b * N, (b + 1) * N), N, ids[l, b, 0],
                                swa=x["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=spec.swa,
                                scale=spec.scale)
            assert_attn_close(out[l, b], ro)


@pytest.mark.parametrize("pdl", [True, False])
@pytest.mark.parametrize("fused", [True, False])
def test_decode_step_kernel_count(cuda_device, pdl, fused):
    spec = synth.scaled(synth.DECODE_64K, N=4099, layers=3)
    _, st = _step(spec, 3, pdl, fused)
    assert graph_kernel_count(st.enqueue) == st.kernel_launches()


def _model_step(spec):
    from lightning_indexer_top_index_b200.decode import ModelStep, model_schedule
    kinds = model_schedule()
    xs = [synth.model_layer(spec, l) for l in range(len(kinds))]

    def kv(k, rows):
        return L.DeviceKV.from_arrays(k.dtype, k.dim, k.data, k.scale, k.rope, batch_rows=rows)

    csa = [LayerCache(kv(x["keys"], spec.N), kv(x["kv"], spec.N), kv(x["swa"], spec.swa)) for x in xs
           if x["kind"] == "csa"]
    hca = [(kv(x["kv"], x["N"]), kv(x["swa"], spec.swa)) for x in xs if x["kind"] == "hca"]
    swa = [kv(x["swa"], spec.swa) for x in xs if x["kind"] == "swa"]
    n_hca = next(x["N"] for x in xs if x["kind"] == "hca")
    st = ModelStep(csa, hca, swa, spec.B, spec.H, spec.N, n_hca, spec.k, spec.swa, spec.scale)

    def t(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16)

    cx = [x for x in xs if x["kind"] == "csa"]
    st.set_inputs(torch.stack([t(x["q_idx"]) for x in cx]).reshape(len(cx), spec.B, 1, spec.H, 128).cuda(),
                  torch.stack([torch.from_numpy(x["w"]) for x in cx]).reshape(len(cx), spec.B, 1, spec.H).cuda(),
                  torch.stack([t(x["q_attn"]) for x in xs]).cuda())
    return xs, st


def test_model_step_all_layer_kinds(cuda_device):
    """One decode token through the 43 attention layers of the hybrid
    schedule (2 window-only, 21 CSA, 20 HCA; architecture post, section (A)),
    captured as one graph: every layer's output against the oracle."""
    spec = synth.scaled(synth.DECODE_64K, N=2048, k=256)
    xs, st = _model_step(spec)
    st.capture()
    for _ in range(2):
        st.replay()
    torch.cuda.synchronize()
    out = st.outputs().cpu().numpy()
    ids, n_sel = st.csa.ids.cpu().numpy(), st.csa.n_sel.cpu().numpy()
    scores = st.csa.scores.cpu().numpy()
    ci = 0
    for l, x in enumerate(xs):
        if x["kind"] == "csa":
            ref_ids, ref_n, _ = oracle.topk(scores[ci, 0, 0], spec.k)
            assert np.array_equal(ids[ci, 0, 0], ref_ids)
            ro, _ = oracle.attn(x["q_attn"][0], x["kv"], spec.N, ids[ci, 0, 0][:ref_n], swa=x["swa"],
                                swa_len=spec.swa, scale=spec.scale)
            ci += 1
        elif x["kind"] == "hca":
            ro, _ = oracle.attn(x["q_attn"][0], x["kv"], x["N"], np.arange(x["N"], dtype=np.int32), swa=x["swa"],
                                swa_len=spec.swa, scale=spec.scale)
        else:
            ro, _ = oracle.attn(x["q_attn"][0], x["swa"], 1, np.zeros(0, dtype=np.int32), swa=x["swa"],
                                swa_len=spec.swa, scale=spec.scale)
        assert_attn_close(out[l, 0], ro)
    assert graph_kernel_count(st.enqueue) == st.kernel_launches() == 21 + 2 * 22
    for ws in st.workspaces():
        assert L.read_device_status(ws) == 0
