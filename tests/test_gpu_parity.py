"""GPU parity: every call of the C ABI against the CPU oracle on the same
seeded inputs (elementwise), at sizes the oracle finishes in seconds that span
several tiles and a ragged tail, plus edge cases."""
import numpy as np
import pytest
import torch

import lightning_indexer_top_index_b200 as L
import oracle
import synth
from _helpers import (assert_attn_close, assert_scores_close, dev_kv, dev_q, graph_kernel_count, score_bound,
                      topk_sets_equivalent)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_device):
    from lightning_indexer_top_index_b200 import build
    build.build()
    yield


# ------------------------------------------------------------------ scoring
def _score_case(spec, layer=0):
    inp = synth.decode_layer(spec, layer)
    B, H, N = spec.B, spec.H, spec.N
    keys = dev_kv(inp["keys"], batch_rows=N)
    q = dev_q(inp["q_idx"].reshape(B, 1, H, 128), spec.q_dtype)
    w = torch.from_numpy(inp["w"].reshape(B, 1, H)).cuda()
    got = L.index_score(q, w, keys, N).cpu().numpy()
    ref, cond = oracle.index_score(inp["q_idx"].reshape(B, 1, H, 128), inp["w"], inp["keys"], B, 1, H, N,
                                   want_cond=True)
    return inp, got, ref, cond


@pytest.mark.parametrize("spec", [
    synth.TINY_1K_F32,
    synth.scaled(synth.DECODE_64K, N=1000),
    synth.scaled(synth.DECODE_64K, N=16384),
    synth.scaled(synth.DECODE_64K, N=4099, B=3, H=32),
    synth.scaled(synth.DECODE_500K_FP8, N=3001, B=2),
    # E4M3 keys over more tiles per CTA than the ring has stages (7 at 64
    # heads, 6 at 128), so every stage and conversion buffer is reused
    synth.scaled(synth.DECODE_500K_FP8, N=80000, B=2),
    synth.scaled(synth.DECODE_500K_FP8, N=70001, B=2, H=128),
    synth.scaled(synth.DECODE_500K_FP8, N=5000, B=3, H=32),
    synth.scaled(synth.DECODE_128K_B32, N=2500, B=2, k=64),
], ids=lambda s: f"{s.name}-N{s.N}-B{s.B}-H{s.H}")
def test_score_parity(spec):
    _, got, ref, cond = _score_case(spec)
    rel = assert_scores_close(got, ref, cond)
    # away from near-zero scores the bar is 1e-5 relative with no floor at all
    assert rel <= 1e-5, rel


@pytest.mark.parametrize("T,N,H", [(64, 700, 64), (5, 1029, 64), (3, 300, 16)])
def test_score_batched_queries(T, N, H):
    """Prefill-style: many queries of one layer scored against the same keys."""
    spec = synth.scaled(synth.EVAL_WINDOW, T=T, N=N, H=H, L=2)
    B = 2
    qs, ws, ks = [], [], []
    for l in range(B):
        e = synth.eval_layer(spec, l)
        qs.append(e["q_idx"])
        ws.append(e["w"])
        ks.append(e["keys"])
    q = np.stack(qs)  # [B][T][H][128]
    w = np.stack(ws)
    keys = synth.concat_kv(ks)
    got = L.index_score(dev_q(q, "bf16"), torch.from_numpy(w).cuda(), dev_kv(keys, batch_rows=N), N).cpu().numpy()
    ref, cond = oracle.index_score(q, w, keys, B, T, H, N, want_cond=True)
    assert_scores_close(got, ref, cond)


def test_score_signed_weights_and_ld():
    """Signed head weights (gate use) and a padded score row stride."""
    spec = synth.scaled(synth.DECODE_64K, N=777)
    inp = synth.decode_layer(spec)
    w = (np.random.default_rng(3).random((1, 64)) * 2 - 1).astype(np.float32)
    scores = torch.full((1, 1, 800), 7.0, device="cuda")
    L.index_score(dev_q(inp["q_idx"].reshape(1, 1, 64, 128), "bf16"), torch.from_numpy(w.reshape(1, 1, 64)).cuda(),
                  dev_kv(inp["keys"]), 777, scores=scores)
    got = scores.cpu().numpy()
    ref, cond = oracle.index_score(inp["q_idx"].reshape(1, 1, 64, 128), w, inp["keys"], 1, 1, 64, 777,
                                   want_cond=True)
    assert_scores_close(got[..., :777], ref, cond)
    assert np.all(got[..., 777:] == 7.0)


def test_score_f16_refused():
    spec = synth.scaled(synth.DECODE_64K, N=64)
    inp = synth.decode_layer(spec)
    keys = dev_kv(inp["keys"])
    keys.dtype = L.F16
    with pytest.raises(L.LidxError) as e:
        L.index_score(dev_q(inp["q_idx"].reshape(1, 1, 64, 128), "bf16"),
                      torch.from_numpy(inp["w"].reshape(1, 1, 64)).cuda(), keys, 64)
    assert e.value.status == L.ERR_UNSUPPORTED


# ------------------------------------------------------------------- top-k
def _topk_check(s, k, allowed=None):
    rows, N = s.shape
    st = torch.from_numpy(s).cuda().reshape(rows, 1, N)
    al = None if allowed is None else torch.from_numpy(allowed).cuda()
    ids, n_sel, mask, bits = L.topk_select(st, k, al, want_mask=True, want_bits=True)
    ids, n_sel, mask = ids.cpu().numpy(), n_sel.cpu().numpy(), mask.cpu().numpy()
    bits = bits.cpu().numpy().view(np.uint32)
    for r in range(rows):
        ref_ids, ref_n, _ = oracle.topk(s[r], k, None if allowed is None else allowed[r])
        assert n_sel[r, 0] == ref_n
        assert np.array_equal(ids[r, 0], ref_ids), f"row {r}"
        dense = np.zeros(N, dtype=np.uint8)
        dense[ref_ids[:ref_n]] = 1
        assert np.array_equal(mask[r, 0], dense)
        assert np.array_equal(bits[r, 0], synth.pack_bits(dense.astype(bool))[0])


@pytest.mark.parametrize("kind", ["normal", "ties", "signed", "const"])
@pytest.mark.parametrize("N,k", [(1, 1), (37, 5), (1024, 64), (16384, 512), (16385, 512), (4000, 4000),
                                 (300, 1000), (60001, 1024)])
def test_topk_bit_exact(kind, N, k):
    """Identical fp32 inputs: ids, n_sel, mask and bits match exactly."""
    s = synth.random_scores(21, 2, N, kind)
    _topk_check(s, k)


def test_topk_large_row():
    s = synth.random_scores(22, 1, 125000, "normal")
    _topk_check(s, 1024)


@pytest.mark.parametrize("N,k,rows,kind", [(600000, 1024, 1, "normal"), (600000, 1024, 2, "ties"),
                                           (1000003, 512, 1, "signed"), (524289, 64, 3, "const")])
def test_topk_rows_beyond_one_cluster(N, k, rows, kind):
    """Rows longer than one thread-block cluster holds (524,288 entries on
    16-CTA clusters) take the segmented path: bit-exact ids, n_sel, mask and
    bits all the same."""
    s = synth.random_scores(27, rows, N, kind)
    _topk_check(s, k)


@pytest.mark.parametrize("N,n_expected", [(16384, 1), (524288, 1), (524289, 4)])
def test_topk_launch_count_matches_graph(N, n_expected):
    """One cluster select up to 524,288 entries a row (16-CTA clusters); four
    kernels beyond."""
    st = torch.from_numpy(synth.random_scores(28, 2, N, "normal")).cuda().reshape(2, 1, N)
    ids = torch.empty((2, 1, 512), dtype=torch.int32, device="cuda")
    n_sel = torch.empty((2, 1), dtype=torch.int32, device="cuda")
    a = L.topk_args(st, 512, None, ids, n_sel)
    assert L.launch_count(L.OP_TOPK, a) == n_expected
    ws = L.workspace(L.workspace_size(L.OP_TOPK, a))
    assert graph_kernel_count(lambda s: L.topk_select(st, 512, ids=ids, n_sel=n_sel, ws=ws, stream=s)) == n_expected


def test_topk_rows_beyond_one_cluster_masked_and_nan():
    N, k = 400000, 1024
    s = synth.random_scores(28, 2, N, "ties")
    s[0, ::1001] = np.nan
    allowed = (np.random.default_rng(29).random((2, N)) < 0.2).astype(np.uint8)
    _topk_check(s, k, allowed)


def test_topk_allowed_mask_and_nan():
    N = 5000
    s = synth.random_scores(23, 3, N, "ties")
    s[1, ::97] = np.nan
    g = np.random.default_rng(23)
    allowed = (g.random((3, N)) < 0.3).astype(np.uint8)
    allowed[2] = 0  # nothing allowed
    st = torch.from_numpy(s).cuda().reshape(3, 1, N)
    ids = torch.empty((3, 1, 256), dtype=torch.int32, device="cuda")
    ws = L.workspace(L.workspace_size(L.OP_TOPK, L.topk_args(st, 256, torch.from_numpy(allowed).cuda(), ids)))
    L.topk_select(st, 256, torch.from_numpy(allowed).cuda(), ws=ws)
    _topk_check(s, 256, allowed)
    # NaN raises the device status flag (row 1 has NaN among allowed entries)
    assert L.read_device_status(ws) & L.DEV_NAN
    assert L.read_device_status(ws) == 0


@pytest.mark.parametrize("N,k,density", [(5000, 256, 0.3), (16384, 512, 0.05), (16384, 512, 0.5), (777, 64, 0.0)])
def test_topk_allowed_bits(N, k, density):
    """A bit-set of eligible entries (the gate's fetched set): the top-k
    inside it, bit-exact against the oracle with the same set as a mask."""
    rows = 3
    s = synth.random_scores(24, rows, N, "ties")
    bits = synth.random_bits(25, rows, N, density)
    allowed = synth.unpack_bits(bits, N).astype(np.uint8)
    st = torch.from_numpy(s).cuda().reshape(rows, 1, N)
    bt = torch.from_numpy(bits.view(np.int32)).cuda()
    ids, n_sel, _, _ = L.topk_select(st, k, allowed_bits=bt)
    ids, n_sel = ids.cpu().numpy(), n_sel.cpu().numpy()
    for r in range(rows):
        ref_ids, ref_n, _ = oracle.topk(s[r], k, allowed[r])
        assert n_sel[r, 0] == ref_n and np.array_equal(ids[r, 0], ref_ids), f"row {r}"
    # both restrictions at once: the eligible entries are their intersection
    al2 = (np.random.default_rng(26).random((rows, N)) < 0.5).astype(np.uint8)
    ids, n_sel, _, _ = L.topk_select(st, k, torch.from_numpy(al2).cuda(), allowed_bits=bt)
    ids = ids.cpu().numpy()
    for r in range(rows):
        ref_ids, _, _ = oracle.topk(s[r], k, allowed[r] & al2[r])
        assert np.array_equal(ids[r, 0], ref_ids), f"row {r}"


# --------------------------------------------------------------- attention
def _attn_case(spec, n_sel=None, swa_len=None, ids=None, layer=0):
    inp = synth.decode_layer(spec, layer)
    B, H, N, k = spec.B, spec.H, spec.N, spec.k
    g = np.random.default_rng(31 + layer)
    if ids is None:
        ids = np.full((B, k), -1, dtype=np.int32)
        for b in range(B):
            m = k if n_sel is None else n_sel[b]
            ids[b, :m] = np.sort(g.choice(N, m, replace=False))
    sl = spec.swa if swa_len is None else swa_len
    kv, swa = dev_kv(inp["kv"], batch_rows=N), dev_kv(inp["swa"], batch_rows=spec.swa)
    q = dev_q(inp["q_attn"], spec.q_dtype)
    ns = None if n_sel is None else torch.tensor(n_sel, dtype=torch.int32, device="cuda")
    out, lse = L.sparse_attn_decode(q, kv, N, torch.from_numpy(ids).cuda(), ns, swa, sl, spec.scale)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        m = k if n_sel is None else n_sel[b]
        ro, rl = oracle.attn(inp["q_attn"][b], inp["kv"].slice(b * N, (b + 1) * N), N, ids[b, :m],
                             swa=inp["swa"].slice(b * spec.swa, (b + 1) * spec.swa), swa_len=sl, scale=spec.scale)
        if np.all(np.isneginf(rl)):
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        assert_attn_close(out[b], ro)
        np.testing.assert_allclose(lse[b], rl, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("spec", [
    synth.TINY_1K_F32,
    synth.scaled(synth.DECODE_64K, N=3000),
    synth.scaled(synth.DECODE_500K_FP8, N=5000, B=2),
    synth.scaled(synth.DECODE_128K_B32, N=4000, B=3, plant=False),
    # batches whose 16-head grid needs more than one wave: 64 heads per CTA
    synth.scaled(synth.DECODE_128K_B32, N=2000, B=8, plant=False),
    synth.scaled(synth.DECODE_500K_FP8, N=3000, B=8, k=512),
], ids=lambda s: f"{s.name}-B{s.B}")
def test_attn_parity(spec):
    _attn_case(spec)


@pytest.mark.parametrize("fmt,B,n_sel,swa_len", [
    ("bf16", 32, None, 128),
    ("e4m3", 32, None, 128),
    ("bf16", 40, "mixed", 37),
    ("bf16", 37, "mixed", 128),
])
def test_attn_wide_several_chunks_per_cta(fmt, B, n_sel, swa_len):
    """Batches past 148 / chunks sequences: each CTA folds several 64-row
    chunks with the online softmax (the accumulated O rescaled when a chunk
    raises a head's maximum), including CTAs whose chunks hold no row."""
    base = synth.DECODE_128K_B32 if fmt == "bf16" else synth.DECODE_500K_FP8
    kw = dict(plant=False) if fmt == "bf16" else {}
    spec = synth.scaled(base, N=1500, B=B, k=512, **kw)
    ns = None
    if n_sel == "mixed":
        ns = [[512, 0, 77, 511, 1, 300, 64, 200][b % 8] for b in range(B)]
    _attn_case(spec, n_sel=ns, swa_len=swa_len)


def test_attn_wide_partial_selection_and_short_window():
    """The 64-head layout (10 sequences x 9 chunks) with partial and empty
    selections and a window shorter than a chunk."""
    spec = synth.scaled(synth.DECODE_64K, N=2000, B=10, k=512)
    _attn_case(spec, n_sel=[512, 100, 0, 512, 511, 1, 64, 300, 0, 450], swa_len=37)


@pytest.mark.parametrize("fmt", ["bf16", "e4m3"])
@pytest.mark.parametrize("k,swa_len", [(20, 37), (64, 128), (384, 128), (448, 128), (512, 128), (896, 128),
                                       (960, 128), (1024, 128)])
def test_attn_split_counts(fmt, k, swa_len):
    """1 to 18 splits of 64 rows (window rows first, then ids), bf16 and E4M3
    rows, against the oracle; the kernel count the library reports against
    the captured graph."""
    base = synth.DECODE_64K if fmt == "bf16" else synth.DECODE_500K_FP8
    spec = synth.scaled(base, N=3000, B=2, k=k)
    _attn_case(spec, swa_len=swa_len)
    inp = synth.decode_layer(spec, 0)
    kv, swa = dev_kv(inp["kv"], batch_rows=spec.N), dev_kv(inp["swa"], batch_rows=spec.swa)
    q = dev_q(inp["q_attn"], spec.q_dtype)
    ids = torch.from_numpy(np.tile(np.arange(k, dtype=np.int32), (spec.B, 1))).cuda()
    out = torch.empty(spec.B, 64, 512, device="cuda")
    a = L.attn_args(q, kv, spec.N, ids, None, swa, swa_len, spec.scale, out, None)
    n = L.launch_count(L.OP_ATTN, a)
    assert n == 2
    ws = L.workspace(L.workspace_size(L.OP_ATTN, a))  # (allocated outside the captured call)
    assert graph_kernel_count(lambda s: L.sparse_attn_decode(q, kv, spec.N, ids, None, swa, swa_len, spec.scale,
                                                              out=out, want_lse=False, ws=ws, stream=s)) == n


def test_attn_partial_selection_and_short_window():
    spec = synth.scaled(synth.DECODE_64K, N=2000, B=3, k=512)
    _attn_case(spec, n_sel=[512, 100, 0], swa_len=37)


def test_attn_no_window_and_empty():
    spec = synth.scaled(synth.DECODE_64K, N=900, B=2, k=64)
    _attn_case(spec, swa_len=0)
    _attn_case(spec, n_sel=[0, 3], swa_len=0)


def test_attn_out_of_range_id_flags_bounds():
    spec = synth.scaled(synth.DECODE_64K, N=500, B=1, k=8)
    inp = synth.decode_layer(spec)
    ids = np.array([[1, 5, 499, 500, 7, -1, 1000, 2]], dtype=np.int32)
    kv, swa = dev_kv(inp["kv"]), dev_kv(inp["swa"])
    ws = L.workspace(L.workspace_size(L.OP_ATTN, L.attn_args(
        dev_q(inp["q_attn"], "bf16"), kv, 500, torch.from_numpy(ids).cuda(), None, swa, 128, spec.scale,
        torch.empty(1, 64, 512, device="cuda"), None)))
    out, _ = L.sparse_attn_decode(dev_q(inp["q_attn"], "bf16"), kv, 500, torch.from_numpy(ids).cuda(), None, swa,
                                  128, spec.scale, ws=ws)
    assert L.read_device_status(ws) & L.DEV_BOUNDS
    keep = np.array([1, 5, 499, 7, 2], dtype=np.int32)
    ro, _ = oracle.attn(inp["q_attn"][0], inp["kv"], 500, keep, swa=inp["swa"], swa_len=128, scale=spec.scale)
    assert_attn_close(out.cpu().numpy()[0], ro)


# ------------------------------------------------------------- end to end
def test_chain_tiny_config():
    """The tiny fp32 case end to end: score -> top-64 -> attention, against the
    oracle chain."""
    spec = synth.TINY_1K_F32
    inp, got, ref, cond = _score_case(spec)
    scores = torch.from_numpy(got).cuda()
    ids, n_sel, _, _ = L.topk_select(scores, spec.k)
    ids_ref, _, _ = oracle.topk(ref[0, 0], spec.k)
    assert topk_sets_equivalent(ids.cpu().numpy()[0, 0], ids_ref, ref[0, 0], score_bound(ref[0, 0], cond[0, 0]))
    kv, swa = dev_kv(inp["kv"]), dev_kv(inp["swa"])
    out, _ = L.sparse_attn_decode(dev_q(inp["q_attn"], "f32"), kv, spec.N, ids[:, 0], n_sel[:, 0], swa, spec.swa,
                                  spec.scale)
    ro, _ = oracle.attn(inp["q_attn"][0], inp["kv"], spec.N, ids_ref, swa=inp["swa"], swa_len=spec.swa,
                        scale=spec.scale)
    assert_attn_close(out.cpu().numpy()[0], ro)


# ------------------------------------------------------------------- eval
@pytest.mark.parametrize("Lq,T,N", [(2, 3, 1100), (1, 4, 32768), (1, 1, 1)])
def test_golden_index_parity(Lq, T, N):
    """probs = the softmax of each score row (LIDX_EVAL_GOLDEN_INDEX), on
    rows with NaN and -inf entries, a row of -inf only, and a padded row
    stride: within 2e-5 relative of the oracle (fp32 exp and a sum over the
    row against double), zeros where the oracle has zeros, NaN flagged."""
    g = np.random.default_rng(40 + N)
    s = (g.standard_normal((Lq * T, N + 5)) * 3).astype(np.float32)
    if Lq * T > 1:
        s[0, ::13] = np.nan
        s[0, 1::17] = -np.inf
        s[1, :] = -np.inf
    st = torch.from_numpy(s).cuda()[:, :N]
    probs = torch.full((Lq, T, N), 7.0, device="cuda")
    ws = L.workspace(4096)
    L.selection_eval(L.EVAL_GOLDEN_INDEX, L=Lq, T=T, N=N, index_scores=st, probs=probs, ws=ws)
    got = probs.cpu().numpy().reshape(Lq * T, N)
    ref = oracle.golden_index(s[:, :N])
    np.testing.assert_allclose(got, ref, rtol=2e-5, atol=1e-30)
    assert np.array_equal(got == 0, ref == 0)
    assert bool(L.read_device_status(ws) & L.DEV_NAN) == bool(np.isnan(s[:, :N]).any())


def test_golden_index_excludes_golden():
    st = torch.zeros((1, 8), device="cuda")
    probs = torch.empty((1, 1, 8), device="cuda")
    with pytest.raises(L.LidxError) as e:
        L.selection_eval(L.EVAL_GOLDEN | L.EVAL_GOLDEN_INDEX, L=1, T=1, H=1, N=8, index_scores=st, probs=probs)
    assert e.value.status == L.ERR_INVALID_ARG


def test_golden_probs_parity():
    spec = synth.scaled(synth.EVAL_WINDOW, L=2, T=3, H=8, N=1100)
    qa = np.stack([synth.eval_layer(spec, l)["qa"][:, :spec.H] for l in range(spec.L)])
    kvs = [synth.eval_layer(spec, l)["kv"] for l in range(spec.L)]
    kv = synth.concat_kv(kvs)
    probs = torch.empty((spec.L, spec.T, spec.N), device="cuda")
    L.selection_eval(L.EVAL_GOLDEN, L=spec.L, T=spec.T, H=spec.H, N=spec.N, qa=dev_q(qa, "bf16"),
                     kv=dev_kv(kv, batch_rows=spec.N), scale=spec.scale, probs=probs)
    got = probs.cpu().numpy()
    for l in range(spec.L):
        ref = oracle.golden(qa[l], kvs[l], spec.T, spec.H, spec.N, spec.scale)
        np.testing.assert_allclose(got[l], ref, rtol=1e-4, atol=1e-10)


@pytest.mark.parametrize("T,N", [(3, 1100), (2, 256), (5, 2000)])
def test_golden_probs_tensor_core(T, N):
    """64 heads, bf16: the tcgen05 path (two queries per 128-row tile, 256-key
    blocks); odd T leaves padding rows in the last tile, N a partial block."""
    spec = synth.scaled(synth.EVAL_WINDOW, L=2, T=T, H=64, N=N)
    qa = np.stack([synth.eval_layer(spec, l)["qa"] for l in range(spec.L)])
    kvs = [synth.eval_layer(spec, l)["kv"] for l in range(spec.L)]
    kv = synth.concat_kv(kvs)
    probs = torch.full((spec.L, spec.T, spec.N), -1.0, device="cuda")
    L.selection_eval(L.EVAL_GOLDEN, L=spec.L, T=spec.T, H=spec.H, N=spec.N, qa=dev_q(qa, "bf16"),
                     kv=dev_kv(kv, batch_rows=spec.N), scale=spec.scale, probs=probs)
    got = probs.cpu().numpy()
    for l in range(spec.L):
        ref = oracle.golden(qa[l], kvs[l], spec.T, spec.H, spec.N, spec.scale)
        np.testing.assert_allclose(got[l], ref, rtol=1e-4, atol=1e-10)


@pytest.mark.parametrize("N,conc", [(1, 1.0), (100, 0.5), (4097, 2.0), (32768, 1.0), (32768, 6.0), (60000, 1.0)])
def test_topp_bit_exact(N, conc):
    rows = 4
    p = synth.random_probs(41, rows, N, conc)
    W = (N + 31) // 32
    bits = torch.zeros((rows, W), dtype=torch.int32, device="cuda")
    L.selection_eval(L.EVAL_TOPP, L=rows, T=1, N=N, probs=torch.from_numpy(p).cuda(), topp_bits=bits)
    got = bits.cpu().numpy().view(np.uint32)
    for r in range(rows):
        ref, _ = oracle.topp(p[r])
        assert np.array_equal(got[r], ref), f"row {r}"


@pytest.mark.parametrize("case", ["uniform", "just_below_split", "at_split"])
def test_topp_unnormalised_rows(case):
    """Rows whose entries lie in [0, 1] but do not sum to 1: a total mass of
    2^43 or more takes the 64-bit digit sums, below it the split 32-bit sums."""
    rng = np.random.default_rng(7)
    if case == "uniform":
        p = rng.random((3, 4097), dtype=np.float32)
    elif case == "just_below_split":
        p = np.full((2, 10), 0.79, dtype=np.float32)
        p[1, 3] = 0.5
    else:
        p = np.full((2, 16), 0.5, dtype=np.float32)
        p[1, ::3] = 0.25
    rows, N = p.shape
    bits = torch.zeros((rows, (N + 31) // 32), dtype=torch.int32, device="cuda")
    L.selection_eval(L.EVAL_TOPP, L=rows, T=1, N=N, probs=torch.from_numpy(p).cuda(), topp_bits=bits)
    got = bits.cpu().numpy().view(np.uint32)
    for r in range(rows):
        ref, _ = oracle.topp(p[r])
        assert np.array_equal(got[r], ref), f"row {r}"


def test_topp_hand_examples_on_gpu():
    import json, os
    ex = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))["topp"]
    for e in ex:
        p = np.array([e["p"]], dtype=np.float32)
        bits = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
        L.selection_eval(L.EVAL_TOPP, L=1, T=1, N=p.shape[1], probs=torch.from_numpy(p).cuda(), topp_bits=bits)
        got = synth.unpack_bits(bits.cpu().numpy().view(np.uint32), p.shape[1])[0]
        assert got.nonzero()[0].tolist() == e["set"]


@pytest.mark.parametrize("N", [31, 32, 1000, 32768])
def test_vote_union_lsa_overlap_bit_exact(N):
    Lyr, T = 21, 5
    W = (N + 31) // 32
    sets = synth.random_bits(51, Lyr * T, N, 0.15).reshape(Lyr, T, W)
    vote = torch.zeros((T, W), dtype=torch.int32, device="cuda")
    win = torch.zeros(W, dtype=torch.int32, device="cuda")
    logits = (np.random.default_rng(52).standard_normal((3, N)) - 1.0).astype(np.float32)
    logits[0, ::11] = 0.0
    fetched = torch.zeros(W, dtype=torch.int32, device="cuda")
    A = synth.random_bits(53, 6, N, 0.3)
    B = synth.random_bits(54, 6, N, 0.5)
    counts = torch.zeros((6, 3), dtype=torch.int64, device="cuda")
    L.selection_eval(L.EVAL_VOTE | L.EVAL_LSA | L.EVAL_OVERLAP, L=Lyr, T=T, N=N,
                     topp_bits=torch.from_numpy(sets.view(np.int32)).cuda(), min_votes=3, vote_bits=vote,
                     window_bits=win, gate_logits=torch.from_numpy(logits).cuda(), gate_bias=-0.0,
                     fetched_bits=fetched, set_a=torch.from_numpy(A.view(np.int32)).cuda(),
                     set_b=torch.from_numpy(B.view(np.int32)).cuda(), n_pairs=6, counts=counts)
    vote_np = vote.cpu().numpy().view(np.uint32)
    for t in range(T):
        assert np.array_equal(vote_np[t], oracle.vote(sets[:, t], N, 3))
    assert np.array_equal(win.cpu().numpy().view(np.uint32), oracle.union(vote_np, N))
    assert np.array_equal(fetched.cpu().numpy().view(np.uint32), oracle.lsa_gate(logits, -0.0))
    c = counts.cpu().numpy()
    for p in range(6):
        assert tuple(c[p]) == oracle.overlap(A[p], B[p], N)


# ------------------------------------------------------ dense (HCA) layers
@pytest.mark.parametrize("spec,swa_len", [
    (synth.scaled(synth.DECODE_64K, N=512, k=512), 128),
    (synth.scaled(synth.DECODE_64K, N=512, k=512, B=3), 77),
    (synth.scaled(synth.DECODE_64K, N=300, k=300, B=2), 0),
    (synth.scaled(synth.DECODE_500K_FP8, N=3907, k=3907, B=2), 128),
    (synth.scaled(synth.TINY_1K_F32, N=32, k=32), 128),
    # many sequences: the wide kernel (several chunks per CTA)
    (synth.scaled(synth.DECODE_64K, N=512, k=512, B=40), 128),
    (synth.scaled(synth.DECODE_500K_FP8, N=700, k=700, B=36), 77),
], ids=lambda x: f"{x.name}-N{x.N}-B{x.B}" if hasattr(x, "name") else f"swa{x}")
def test_attn_dense_rows_hca(spec, swa_len):
    """The HCA layers of the architecture post (section (A): 128:1
    compression, about 512 entries at 64K, every entry read, no top-k): the
    attention with no ids reads rows 0..N-1 of every sequence; the oracle
    attends over ids = 0..N-1."""
    inp = synth.decode_layer(spec)
    B, N = spec.B, spec.N
    kv, swa = dev_kv(inp["kv"], batch_rows=N), dev_kv(inp["swa"], batch_rows=spec.swa)
    q = dev_q(inp["q_attn"], spec.q_dtype)
    out, lse = L.sparse_attn_decode(q, kv, N, None, None, swa, swa_len, spec.scale, n_dense=N)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        ro, rl = oracle.attn(inp["q_attn"][b], inp["kv"].slice(b * N, (b + 1) * N), N,
                             np.arange(N, dtype=np.int32), swa=inp["swa"].slice(b * spec.swa, (b + 1) * spec.swa),
                             swa_len=swa_len, scale=spec.scale)
        assert_attn_close(out[b], ro)
        np.testing.assert_allclose(lse[b], rl, rtol=1e-5, atol=1e-5)


def test_attn_dense_rows_with_n_sel():
    """Dense rows with a per-sequence count: sequence b reads rows 0..n_b-1."""
    spec = synth.scaled(synth.DECODE_64K, N=512, k=512, B=3)
    inp = synth.decode_layer(spec)
    N = spec.N
    n_b = [512, 100, 0]
    kv, swa = dev_kv(inp["kv"], batch_rows=N), dev_kv(inp["swa"], batch_rows=spec.swa)
    ns = torch.tensor(n_b, dtype=torch.int32, device="cuda")
    out, lse = L.sparse_attn_decode(dev_q(inp["q_attn"], "bf16"), kv, N, None, ns, swa, 64, spec.scale, n_dense=N)
    out = out.cpu().numpy()
    for b in range(3):
        ro, _ = oracle.attn(inp["q_attn"][b], inp["kv"].slice(b * N, (b + 1) * N), N,
                            np.arange(n_b[b], dtype=np.int32), swa=inp["swa"].slice(b * spec.swa, (b + 1) * spec.swa),
                            swa_len=64, scale=spec.scale)
        assert_attn_close(out[b], ro)
