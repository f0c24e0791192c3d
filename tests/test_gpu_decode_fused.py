"""The fused decode layer (lidx_decode_layer: index scores -> top-k -> sparse
attention in one launch) against the oracle, element by element: scores
within the score tolerance, the ids bit-exact against the oracle's top-k of
the GPU's own scores, and the attention output within the attention
tolerance of the oracle's attention over those ids (architecture post,
section (B)).  Also: the three-call path on the same inputs, repeated calls
on one workspace, a captured graph of stacked layers with programmatic
dependent launch and L2 prefetch, and the bounded-wait give-up path."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import assert_attn_close, assert_scores_close, dev_kv, dev_q, score_bound, topk_sets_equivalent

pytestmark = pytest.mark.gpu


def _inputs(spec, layer=0):
    """Inputs of one layer; the attention always has 64 query heads (the
    generator ties them to the index heads, so other index head counts get
    their own 64-head attention queries)."""
    x = synth.decode_layer(spec, layer)
    B, H, N = spec.B, spec.H, spec.N
    if H != 64:
        x["q_attn"] = synth.decode_layer(synth.scaled(spec, H=64, N=1), 500 + layer)["q_attn"]
    d = dict(q_idx=dev_q(x["q_idx"].reshape(B, H, 128), "bf16"), w=torch.from_numpy(x["w"].reshape(B, H)).cuda(),
             keys=dev_kv(x["keys"], batch_rows=N), q_attn=dev_q(x["q_attn"], "bf16"),
             kv=dev_kv(x["kv"], batch_rows=N), swa=dev_kv(x["swa"], batch_rows=spec.swa))
    return x, d


def _run(spec, d, swa_len, ws=None, flags=0, prefetch=()):
    B, N, k = spec.B, spec.N, spec.k
    scores = torch.full((B, N), float("nan"), device="cuda")
    ids = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out, lse = L.decode_layer(d["q_idx"], d["w"], d["keys"], N, k, d["q_attn"], d["kv"], d["swa"], swa_len,
                              spec.scale, scores=scores, ids=ids, n_sel=n_sel, ws=ws, flags=flags, prefetch=prefetch)
    torch.cuda.synchronize()
    return scores.cpu().numpy(), ids.cpu().numpy(), n_sel.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def _check_against_oracle(spec, x, res, swa_len):
    scores, ids, n_sel, out, lse = res
    B, H, N, k = spec.B, spec.H, spec.N, spec.k
    for b in range(B):
        ref, cond = oracle.index_score(x["q_idx"][b].reshape(1, 1, H, 128), x["w"][b],
                                       x["keys"].slice(b * N, (b + 1) * N), 1, 1, H, N, want_cond=True)
        assert_scores_close(scores[b], ref[0, 0], cond[0, 0])
        # the ids: bit-exact against the oracle's top-k of the same scores
        ref_ids, ref_n, _ = oracle.topk(scores[b], k)
        assert n_sel[b] == ref_n and np.array_equal(ids[b], ref_ids), f"sequence {b}"
        # end to end: the set is the oracle's own top-k up to ties at the k-th score
        oids, _, _ = oracle.topk(ref[0, 0], k)
        assert topk_sets_equivalent(ids[b], oids, ref[0, 0], score_bound(ref[0, 0], cond[0, 0]))
        ro, rl = oracle.attn(x["q_attn"][b], x["kv"].slice(b * N, (b + 1) * N), N, ids[b][:ref_n],
                             swa=x["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=swa_len,
                             scale=spec.scale)
        assert_attn_close(out[b], ro)
        np.testing.assert_allclose(lse[b], rl, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("spec,swa_len", [
    (synth.scaled(synth.DECODE_64K, N=3000, k=256), 128),
    (synth.scaled(synth.DECODE_64K, N=4099, k=512, B=2), 128),
    (synth.scaled(synth.DECODE_64K, N=1000, k=64, B=3, H=32), 77),
    (synth.scaled(synth.DECODE_64K, N=300, k=512), 128),
    (synth.scaled(synth.DECODE_64K, N=777, k=100, H=128), 0),
    (synth.scaled(synth.DECODE_64K, N=16383, k=512), 128),
], ids=lambda x: f"{x.name}-N{x.N}-B{x.B}-H{x.H}-k{x.k}" if hasattr(x, "name") else f"swa{x}")
def test_fused_layer_parity(cuda_device, spec, swa_len):
    x, d = _inputs(spec)
    _check_against_oracle(spec, x, _run(spec, d, swa_len), swa_len)


def test_fused_layer_rejects_rows_beyond_one_selector(cuda_device):
    """One CTA selects a row of at most 16384 entries: a longer row is
    LIDX_ERR_UNSUPPORTED (the three-call layer takes it), before any launch."""
    spec = synth.scaled(synth.DECODE_64K, N=16385, k=512)
    x, d = _inputs(spec)
    with pytest.raises(L.LidxError) as e:
        _run(spec, d, 128)
    assert e.value.status == L.ERR_UNSUPPORTED


def test_fused_layer_full_size_64k(cuda_device):
    """The 64K decode layer as the bench runs it (N = 16384, 64 heads,
    top-512, 128-row window), on two layers of the stack."""
    spec = synth.DECODE_64K
    for layer in (0, 13):
        x, d = _inputs(spec, layer)
        _check_against_oracle(spec, x, _run(spec, d, spec.swa), spec.swa)


def test_fused_matches_three_calls_and_reuses_workspace(cuda_device):
    """Same inputs through lidx_index_score -> lidx_topk_select ->
    lidx_sparse_attn_decode: identical scores and ids, outputs within 1e-5
    (the split layouts match).  Three calls in a row on one workspace give
    the same results each time (the control words are reset)."""
    spec = synth.scaled(synth.DECODE_64K, N=5000, k=512)
    x, d = _inputs(spec)
    N, k = spec.N, spec.k
    s3 = L.index_score(d["q_idx"].reshape(1, 1, spec.H, 128), d["w"].reshape(1, 1, spec.H), d["keys"], N)
    ids3, n3, _, _ = L.topk_select(s3, k)
    o3, l3 = L.sparse_attn_decode(d["q_attn"], d["kv"], N, ids3[:, 0], n3[:, 0], d["swa"], spec.swa, spec.scale)
    a = L.decode_args(d["q_idx"], d["w"], d["keys"], N, k, d["q_attn"], d["kv"], d["swa"], spec.swa, spec.scale,
                      o3)
    ws = L.workspace(L.workspace_size(L.OP_DECODE, a))
    first = None
    for _ in range(3):
        res = _run(spec, d, spec.swa, ws=ws)
        assert L.read_device_status(ws) == 0
        if first is None:
            first = res
        for u, v in zip(res, first):
            np.testing.assert_array_equal(u, v)
    scores, ids, n_sel, out, lse = first
    assert np.array_equal(scores[0], s3.cpu().numpy()[0, 0])
    assert np.array_equal(ids[0], ids3.cpu().numpy()[0, 0])
    np.testing.assert_allclose(out, o3.cpu().numpy(), rtol=1e-5, atol=1e-6)
    # the control words are zero again after the calls
    assert int(ws[256:256 + 64 * 4].view(torch.int32).abs().sum().item()) == 0


def test_fused_ties_and_nan(cuda_device):
    """Keys that repeat give exactly tied scores (ties go to the lower index);
    a NaN head weight makes every score NaN: none is selected, and the
    device status flag is raised."""
    spec = synth.scaled(synth.DECODE_64K, N=4096, k=512)
    x, d = _inputs(spec)
    keys = d["keys"].data.clone()
    keys[1024:2048] = keys[0:1024]  # every score of [1024, 2048) ties one of [0, 1024)
    keys[3000:4096] = keys[5]       # 1096 entries share one score
    d["keys"] = L.DeviceKV(L.BF16, 128, keys, batch_rows=spec.N)
    ws = L.workspace(1 << 24)
    scores, ids, n_sel, out, _ = _run(spec, d, spec.swa, ws=ws)
    ref_ids, ref_n, _ = oracle.topk(scores[0], spec.k)
    assert np.array_equal(ids[0], ref_ids)
    assert L.read_device_status(ws) == 0
    w = d["w"].clone()
    w[0, 3] = float("nan")
    d["w"] = w
    scores, ids, n_sel, _, _ = _run(spec, d, spec.swa, ws=ws)
    assert np.isnan(scores[0]).all() and n_sel[0] == 0 and (ids[0] == -1).all()
    assert L.read_device_status(ws) & L.DEV_NAN


def test_fused_stack_in_graph_with_pdl_and_prefetch(cuda_device):
    """Four layers captured in one CUDA graph with programmatic dependent
    launch, each prefetching the next layer's keys and window into L2: every
    layer's output equals its single-call result."""
    spec = synth.scaled(synth.DECODE_64K, N=16384, k=512, layers=4)
    layers = [_inputs(spec, l) for l in range(4)]
    singles = [_run(spec, d, spec.swa) for _, d in layers]
    outs = [torch.empty((1, 64, 512), device="cuda") for _ in range(4)]
    wss = []
    args = []
    for l, (_, d) in enumerate(layers):
        pf = ()
        if l + 1 < 4:
            nd = layers[l + 1][1]
            pf = ((nd["keys"].data.data_ptr(), nd["keys"].nbytes()), (nd["swa"].data.data_ptr(), nd["swa"].nbytes()))
        a = L.decode_args(d["q_idx"], d["w"], d["keys"], spec.N, spec.k, d["q_attn"], d["kv"], d["swa"], spec.swa,
                          spec.scale, outs[l], prefetch=pf, flags=L.LAUNCH_PDL)
        args.append(a)
        wss.append(L.workspace(L.workspace_size(L.OP_DECODE, a)))
    import ctypes as C

    def enqueue(st):
        for a, ws in zip(args, wss):
            rc = L.lib().lidx_decode_layer(C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(),
                                           C.c_void_p(st.cuda_stream))
            assert rc == L.OK

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        enqueue(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        enqueue(torch.cuda.current_stream())
    for _ in range(3):
        for o in outs:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for l in range(4):
            np.testing.assert_array_equal(outs[l].cpu().numpy(), singles[l][3])
    for ws in wss:
        assert L.read_device_status(ws) == 0


def test_fused_lost_arrival_times_out_and_recovers(cuda_device):
    """Test hook: one score CTA withholds its arrival.  The selector's bounded
    wait gives up (about 2 ms), the call finishes and reports
    LIDX_DEV_TIMEOUT; the next call on the same workspace is correct."""
    spec = synth.scaled(synth.DECODE_64K, N=3000, k=256)
    x, d = _inputs(spec)
    ws = L.workspace(1 << 24)
    _run(spec, d, spec.swa, ws=ws, flags=L.LAUNCH_TEST_LOST_ARRIVAL)
    assert L.read_device_status(ws) & L.DEV_TIMEOUT
    res = _run(spec, d, spec.swa, ws=ws)
    assert L.read_device_status(ws) == 0
    _check_against_oracle(spec, x, res, spec.swa)


def test_fused_rejects_what_it_does_not_cover(cuda_device):
    spec = synth.scaled(synth.DECODE_500K_FP8, N=2000, k=128, B=1)
    x = synth.decode_layer(spec)
    d = dict(q_idx=dev_q(x["q_idx"].reshape(1, 64, 128), "bf16"), w=torch.from_numpy(x["w"].reshape(1, 64)).cuda(),
             keys=dev_kv(x["keys"], batch_rows=spec.N), q_attn=dev_q(x["q_attn"], "bf16"),
             kv=dev_kv(x["kv"], batch_rows=spec.N), swa=dev_kv(x["swa"], batch_rows=spec.swa))
    with pytest.raises(L.LidxError) as e:
        L.decode_layer(d["q_idx"], d["w"], d["keys"], spec.N, spec.k, d["q_attn"], d["kv"], d["swa"], spec.swa)
    assert e.value.status == L.ERR_UNSUPPORTED
